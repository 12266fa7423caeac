// Grouped SwiGLU expert GEMMs with 4-bit expert weights, and the quantiser
// that writes those weights.
//
// Sources: "How Mixtral 8x7B uses mixture of experts", "Deployment tradeoffs
// you'll actually hit" / "Quantization asymmetry" (router kept in 16-bit,
// experts in 4 bits) and "Mixtral 8x7B — MoE Complete Guide", "4-bit
// Quantization for Single GPU" (4-bit weights, bf16 arithmetic).  The expert
// itself is the one of "Mixtral", "MoE Layer": w2(silu(w1 x) * w3 x).
//
// Weight format (one matrix W [E, R, K], K a multiple of 64):
//   codes  [E, R, K/2] bytes; the codes of inputs 8g .. 8g+7 of a row fill one
//          little-endian 32-bit word, nibble m holding input 8g + 2m and
//          nibble m + 4 input 8g + 2m + 1 (m = 0..3);
//   scales [E, K/64, R] bf16, one per 64 consecutive inputs of a row;
//   w = (code - 8) * scale.
// The nibble order lets one AND/OR turn a word into two bf16 pairs of
// adjacent inputs: (word >> 4m) & 0x000F000F | 0x43004300 is the bf16 pair
// (128 + code(8g+2m), 128 + code(8g+2m+1)).
//
// The GEMMs use the streaming schedule of the bf16 kernels (weights are the
// MMA's M operand, the expert's tokens its N operand), with the weight
// operand taken from tensor memory instead of shared memory:
//   warp 0      TMA: per stage of 128 inputs, the 4-bit codes of 128 weight
//               rows (64-byte swizzle), their scales and the tokens' bf16
//               tile (128-byte swizzle);
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               kind::f16 with A read from tensor memory, B from shared memory;
//   warps 2-5   epilogue (SiLU * mul, or fp32 split-K partials);
//   warps 6-9   dequantise: thread i of warp w owns weight row 32 (w % 4) + i
//               (its tensor-memory lane) and the stage's 128 inputs of it; it
//               turns the codes into bf16, multiplies by the block scales and
//               writes 64 columns of the A buffer with tcgen05.st.
// The MMA-issuing thread shares its scheduler with one epilogue and one
// dequantising warp (TMEM lane quarters fix which warps run where); small-N
// MMAs are bound by how fast that thread issues, so the dequantisation uses
// as few warps as keep up (4; 8 and 16 measured slower) and the issue loop
// is kept short.
// Four A buffers of 64 columns sit behind the two accumulators.  An A buffer
// is reused once the MMAs of the stage that last read it have completed,
// which the one commit per stage that frees the stage's shared memory also
// reports (a commit costs about as much to issue as an MMA).  Reading the
// 4-bit codes moves a quarter of the bf16 bytes from HBM; the bf16 weights
// never pass through shared memory.
#include <cstdint>
#include <cstdio>

#include <cuda_bf16.h>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int KQ = 128;                  // inputs per stage (two scale blocks)
constexpr int kDeqWarp0 = 6;             // first dequantising warp
constexpr int kDeqWarps = 4;
constexpr int kDeqParts = kDeqWarps / 4;    // warps per TMEM lane quarter
constexpr int kDeqChunks = 4 / kDeqParts;   // 16-byte code chunks (32 inputs) per thread and stage
constexpr int kQ4Threads = (kDeqWarp0 + kDeqWarps) * 32;
constexpr int kCodeBytes = 128 * KQ / 2;  // 128 rows x 64 bytes
constexpr int kScaleBytes = 1024;         // 2 blocks x 128 rows x bf16 = 512, padded
constexpr int kABufs = 4;
constexpr int kACols = KQ / 2;            // TMEM columns of one bf16 A buffer
constexpr int kACol0 = 256;               // A buffers start here; accumulators below
constexpr int kTmemCols = 512;

enum : int { Q4_SWIGLU = 0, Q4_PARTIAL = 1 };

template <int EPI, int BN>
struct Q4Cfg {
  static constexpr int B_BYTES = BN * KQ * 2;  // two 64-input chunks of BN token rows
  static constexpr int STAGE_BYTES = B_BYTES + kCodeBytes + kScaleBytes;
  static constexpr int STAGES = (212 * 1024) / STAGE_BYTES > 12 ? 12 : (212 * 1024) / STAGE_BYTES;
  static constexpr int XBUF_BYTES = (EPI == Q4_SWIGLU) ? 64 * 16 * 4 : 0;
  static constexpr int BAR_BYTES = (2 * STAGES + kABufs + 5) * 8;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + XBUF_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = make_idesc_bf16(128, BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 128, "MMA N");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(2 * BN <= kACol0, "accumulators overlap the A buffers");
  static_assert(STAGES > kABufs, "A-buffer reuse is read from the stage barriers");
  static_assert(STAGES >= 3 && SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Q4Params {
  const int32_t* offsets;
  uint32_t* status;
  void* out;            // bf16 h, or fp32 partials
  int64_t out_ld;
  int64_t part_stride;
  int32_t E;
  int32_t num_kq;       // stages over K (K / 128, rounded up)
  int32_t n_out;        // output columns (d_ff or d_model)
  int32_t n_blocks;     // weight blocks per expert (64 rows of W1 and W3, or 128 of W2)
  int32_t splits;
  int32_t kq_per_split;
  int64_t S;            // rows of the activation and output buffers (T * k)
  uint64_t* clock_probe;  // profiled calls: CTA 0 writes {clock64, globaltimer} at entry and exit
};

struct Q4Tile {
  int32_t e, row0, m_valid, n0, split, kq0, kq1;
};

template <int EPI, int BN>
__device__ __forceinline__ void q4_decode_tile(const Q4Params& p, const int32_t* s_off, const int32_t* s_base,
                                               int32_t tile, Q4Tile& t) {
  int e = 0;
  while (e < p.E && tile >= s_base[e + 1]) ++e;
  const int32_t local = tile - s_base[e];
  const int32_t M_e = s_off[e + 1] - s_off[e];
  const int32_t tb_count = (M_e + BN - 1) / BN;
  const int32_t tb = local % tb_count;
  const int32_t rest = local / tb_count;
  t.e = e;
  t.split = rest % p.splits;
  const int32_t wb = rest / p.splits;
  t.row0 = s_off[e] + tb * BN;
  t.m_valid = min(BN, M_e - tb * BN);
  t.n0 = wb * (EPI == Q4_SWIGLU ? 64 : 128);
  t.kq0 = t.split * p.kq_per_split;
  t.kq1 = min(p.num_kq, t.kq0 + p.kq_per_split);
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A is 128 lanes x 16 bf16 (8 columns).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 16 consecutive columns from registers: thread i writes lane
// (base lane + i).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}


// (code - 8) * s for the two codes in bits 0..3 and 16..19 of `bits`.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t bits, __nv_bfloat162 s2) {
  const uint32_t b = (bits & 0x000F000Fu) | 0x43004300u;  // 128 + code, exact
  const uint32_t k136 = 0x43084308u;                       // 136 in both halves
  const __nv_bfloat162 w = __hmul2(__hsub2(*reinterpret_cast<const __nv_bfloat162*>(&b),
                                           *reinterpret_cast<const __nv_bfloat162*>(&k136)),
                                   s2);
  return *reinterpret_cast<const uint32_t*>(&w);
}

template <int EPI, int BN>
__global__ void __launch_bounds__(kQ4Threads, 1)
    expert_gemm_q4_kernel(const __grid_constant__ CUtensorMap map_act,
                          const __grid_constant__ CUtensorMap map_ca,  // codes: W1 or W2
                          const __grid_constant__ CUtensorMap map_cb,  // codes: W3
                          const __grid_constant__ CUtensorMap map_sa,  // scales: W1 or W2
                          const __grid_constant__ CUtensorMap map_sb,  // scales: W3
                          Q4Params p) {
  using C = Q4Cfg<EPI, BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_epi_fail;
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_base[33];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [B tile | codes | scales], 1024-byte aligned pieces
  float* xbuf = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::XBUF_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* afull_bar = bars + 2 * STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES + kABufs;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tfull_bar + 4;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe);

  if (tid == 0) {
    tma_prefetch_desc(&map_act);
    tma_prefetch_desc(&map_ca);
    tma_prefetch_desc(&map_sa);
    if (EPI == Q4_SWIGLU) {
      tma_prefetch_desc(&map_cb);
      tma_prefetch_desc(&map_sb);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < kABufs; ++a) mbar_init(&afull_bar[a], kDeqWarps);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();     // offsets and activations of the kernels before this one
  pdl_trigger();  // the next kernel may start its own set-up
  if (tid == 64) {
    s_abort = 0;
    s_epi_fail = 0;
    int32_t acc = 0;
    s_base[0] = 0;
    for (int e = 0; e <= p.E; ++e) s_off[e] = p.offsets[e];
#ifdef MOE_DEBUG
    {  // offsets must start at 0, not decrease and stay within the S rows
      bool bad = s_off[0] != 0 || (int64_t)s_off[p.E] > p.S;
      for (int e = 0; e < p.E; ++e) bad = bad || s_off[e + 1] < s_off[e];
      if (bad) {
        record_status(p.status, kStatusBounds);
        for (int e = 0; e <= p.E; ++e) s_off[e] = 0;
      }
    }
#endif
    for (int e = 0; e < p.E; ++e) {
      const int32_t M_e = s_off[e + 1] - s_off[e];
      acc += M_e > 0 ? ((M_e + BN - 1) / BN) * p.n_blocks * p.splits : 0;
      s_base[e + 1] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const int32_t total = s_base[p.E];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        Q4Tile t;
        q4_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
        for (int32_t kq = t.kq0; kq < t.kq1; ++kq) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          uint8_t* b_dst = st;
          uint8_t* c_dst = st + C::B_BYTES;
          uint8_t* s_dst = c_dst + kCodeBytes;
          mbar_arrive_expect_tx(&full_bar[stage], C::B_BYTES + kCodeBytes + 512);
          const int32_t kx = kq * KQ;
          tma_load_2d(&map_act, &full_bar[stage], b_dst, kx, t.row0);
          tma_load_2d(&map_act, &full_bar[stage], b_dst + BN * 128, kx + 64, t.row0);
          if (EPI == Q4_SWIGLU) {
            tma_load_3d(&map_ca, &full_bar[stage], c_dst, kx / 2, t.n0, t.e);
            tma_load_3d(&map_cb, &full_bar[stage], c_dst + 64 * 64, kx / 2, t.n0, t.e);
            tma_load_3d(&map_sa, &full_bar[stage], s_dst, t.n0, 2 * kq, t.e);
            tma_load_3d(&map_sb, &full_bar[stage], s_dst + 256, t.n0, 2 * kq, t.e);
          } else {
            tma_load_3d(&map_ca, &full_bar[stage], c_dst, kx / 2, t.n0, t.e);
            tma_load_3d(&map_sa, &full_bar[stage], s_dst, t.n0, 2 * kq, t.e);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      for (int s = 0; s < STAGES; ++s) {
        if (s < issued) {
          const int64_t uses = (issued - s + STAGES - 1) / STAGES;
          mbar_wait(&full_bar[s], (uint32_t)((uses - 1) & 1), nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      uint32_t iter = 0;
      bool ok = true;
      for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++iter) {
        Q4Tile t;
        q4_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
        const uint32_t acc = iter & 1, use = iter >> 1;
        if (!mbar_wait(&tempty_bar[acc], (use & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int32_t kq = t.kq0; kq < t.kq1; ++kq) {
          if (!mbar_wait(&full_bar[stage], phase, &s_abort) || !mbar_wait(&afull_bar[abuf], aphase, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // The issuing thread shares its scheduler with dequantising warps
          // (TMEM lane quarters fix which warps run where), so its stream is
          // kept short: the B descriptor is built once per stage and moved by
          // constant offsets (the start-address field counts 16 bytes).
          const uint64_t b_desc = make_sdesc_sw128(smem_u32(smem + stage * C::STAGE_BYTES));
          const uint32_t a_tmem = tmem_base + kACol0 + abuf * kACols;
          umma_bf16_ts(d_tmem, a_tmem, b_desc, C::IDESC, kq > t.kq0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < KQ / 16; ++kk)
            umma_bf16_ts(d_tmem, a_tmem + kk * 8, b_desc + (uint64_t)(((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4),
                         C::IDESC, 1u);
          umma_commit(&empty_bar[stage]);  // frees the stage and its A buffer
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
          if (++abuf == kABufs) {
            abuf = 0;
            aphase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr);
    }
  } else if (warp >= kDeqWarp0) {
    // ------------------------------------------------ dequantise (warps 6..)
    const int q = warp & 3;                      // TMEM lane quarter
    const int part = (warp - kDeqWarp0) >> 2;    // chunks kDeqChunks*part .. of the stage
    const int r = q * 32 + lane;                 // weight row of the A tile
    // codes: row r is 64 bytes; 16-byte chunk c (inputs 32c .. 32c+31) sits at
    // chunk c ^ ((r >> 1) & 3) (64-byte swizzle); its scale is block c / 2
    uint32_t c_off[kDeqChunks], s_off_b[kDeqChunks];
#pragma unroll
    for (int c = 0; c < kDeqChunks; ++c) {
      const int chunk = part * kDeqChunks + c;
      const int blk = chunk >> 1;
      c_off[c] = (uint32_t)r * 64 + (((uint32_t)chunk ^ (uint32_t)((r >> 1) & 3)) << 4);
      s_off_b[c] = kCodeBytes + 2 * ((EPI == Q4_SWIGLU) ? ((r >> 6) * 128 + blk * 64 + (r & 63)) : (blk * 128 + r));
    }
    const uint32_t t_col = tmem_base + ((uint32_t)(q * 32) << 16) + kACol0 + part * kDeqChunks * 16;
    int stage = 0, abuf = 0;
    uint32_t phase = 0;
    int64_t i = 0;  // stages dequantised so far
    bool ok = true;
    for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      Q4Tile t;
      q4_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
      for (int32_t kq = t.kq0; kq < t.kq1; ++kq, ++i) {
        bool w_ok = mbar_wait(&full_bar[stage], phase, &s_abort);
        if (w_ok && i >= kABufs) {
          // the A buffer was last read by the MMAs of stage i - kABufs; the
          // barrier cannot have moved on further, since that needs stage
          // i - kABufs + STAGES, which this warp has not dequantised yet
          const int64_t j = i - kABufs;
          w_ok = mbar_wait(&empty_bar[j % STAGES], (uint32_t)((j / STAGES) & 1), &s_abort);
        }
        if (!w_ok) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + stage * C::STAGE_BYTES + C::B_BYTES;
#pragma unroll
        for (int c = 0; c < kDeqChunks; ++c) {
          const uint4 w4 = *reinterpret_cast<const uint4*>(st + c_off[c]);
          const uint16_t sb = *reinterpret_cast<const uint16_t*>(st + s_off_b[c]);
          const uint32_t s2u = uint32_t(sb) | (uint32_t(sb) << 16);
          const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
          const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
          uint32_t v[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int m = 0; m < 4; ++m) v[4 * k + m] = dequant_pair(words[k] >> (4 * m), s2);
          }
          tmem_st_32x32b_x16(t_col + abuf * kACols + c * 16, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull_bar[abuf]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
        if (++abuf == kABufs) abuf = 0;
      }
    }
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      s_abort = 1;
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint32_t iter = 0;
    for (int32_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++iter) {
      Q4Tile t;
      q4_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
      const uint32_t acc = iter & 1, use = iter >> 1;
      if (!mbar_wait(&tfull_bar[acc], use & 1, &s_abort)) s_epi_fail = 1;
      named_bar_sync(2, 128);
      if (s_epi_fail) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_acc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      if (EPI == Q4_SWIGLU) {
        // lanes 0..63: W1 projection of column n0 + r; lanes 64..127: W3 of column n0 + r - 64
        uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_acc + c0, v);
          tmem_ld_wait();
          if (r >= 64) {
#pragma unroll
            for (int j = 0; j < 16; ++j) xbuf[j * 64 + (r - 64)] = __uint_as_float(v[j]);
          }
          named_bar_sync(1, 128);
          if (r < 64 && t.n0 + r < p.n_out) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int tok = c0 + j;
              if (tok < t.m_valid && MOE_DCHECK(p.status, t.row0 + tok < p.S)) {
                const float hv = silu_f32(__uint_as_float(v[j])) * xbuf[j * 64 + r];
                out[(int64_t)(t.row0 + tok) * p.out_ld + t.n0 + r] = (uint16_t)(pack_bf16x2(hv, 0.f) & 0xFFFFu);
              }
            }
          }
          named_bar_sync(1, 128);
        }
      } else {
        float* out = reinterpret_cast<float*>(p.out) + (int64_t)t.split * p.part_stride;
        const bool col_ok = t.n0 + r < p.n_out;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_acc + c0, v);
          tmem_ld_wait();
          if (col_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int tok = c0 + j;
              if (tok < t.m_valid && MOE_DCHECK(p.status, t.row0 + tok < p.S))
                out[(int64_t)(t.row0 + tok) * p.out_ld + t.n0 + r] = __uint_as_float(v[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe + 2);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ quantiser
// One thread per code word (8 inputs); the 8 threads of a 64-input block
// share its absmax through shuffles.  s = bf16(absmax / 7) and
// q = clamp(round_half_even(w / s), -8, 7), both divisions IEEE fp32.
__global__ void __launch_bounds__(256) quantize_q4_kernel(const uint4* __restrict__ W, uint32_t* __restrict__ codes,
                                                          uint16_t* __restrict__ scales, int64_t words, int32_t R,
                                                          int32_t K) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= words) return;  // words is a multiple of 8: a block's 8 threads exit together
  const int lane = threadIdx.x & 31;
  const unsigned gmask = 0xFFu << (lane & ~7);
  const uint4 raw = W[i];
  const uint32_t pr[4] = {raw.x, raw.y, raw.z, raw.w};
  float w[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[2 * j] = __uint_as_float(pr[j] << 16);
    w[2 * j + 1] = __uint_as_float(pr[j] & 0xFFFF0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(w[j]));
  amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 4));
  const uint32_t sbits = pack_bf16x2(__fdiv_rn(amax, 7.0f), 0.f) & 0xFFFFu;
  const float s = __uint_as_float(sbits << 16);
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int qv = 0;
    if (s != 0.f) qv = (int)fminf(fmaxf(rintf(__fdiv_rn(w[j], s)), -8.f), 7.f);
    const int nib = j / 2 + 4 * (j % 2);
    word |= (uint32_t)(qv + 8) << (4 * nib);
  }
  codes[i] = word;
  if ((i & 7) == 0) {
    const int64_t wpr = K / 8;  // words per row
    const int64_t row = i / wpr;
    const int64_t blk = (i % wpr) / 8;
    const int64_t e = row / R, r = row % R;
    scales[(e * (K / 64) + blk) * R + r] = (uint16_t)sbits;
  }
}

}  // namespace

// codes [E, R, K/2] as a 3-D uint8 map, box {64 bytes, box_rows, 1}, 64-byte swizzle
bool encode_codes(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)R, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)(R * (K / 2))};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// scales [E, K/64, R] as a 3-D bf16 map, box {box_rows, 2, 1}
bool encode_scales(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)R, (cuuint64_t)(K / 64), (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(R * 2), (cuuint64_t)((K / 64) * R * 2)};
  cuuint32_t box[3] = {(cuuint32_t)box_rows, 2, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// token tile [S, K] bf16, box {64, box_rows}, 128-byte swizzle
namespace {

bool encode_tokens(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int BN>
cudaError_t launch_q4_one(const CUtensorMap& act, const CUtensorMap& ca, const CUtensorMap& cb,
                          const CUtensorMap& sa, const CUtensorMap& sb, const Q4Params& p, int num_sms,
                          cudaStream_t s, bool pdl) {
  using C = Q4Cfg<EPI, BN>;
  cudaError_t err =
      cudaFuncSetAttribute(expert_gemm_q4_kernel<EPI, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_k(expert_gemm_q4_kernel<EPI, BN>, dim3(num_sms), dim3(kQ4Threads), C::SMEM_BYTES, s, pdl, act, ca,
                  cb, sa, sb, p);
}

template <int BN>
cudaError_t launch_q4(const ExpertGemmQ4Args& a, cudaStream_t s) {
  CUtensorMap mx, mc1, mc3, ms1, ms3, mh, mc2, ms2;
  if (!encode_tokens(&mx, a.x_perm, a.S, a.d, BN) || !encode_codes(&mc1, a.W1c, a.E, a.f, a.d, 64) ||
      !encode_codes(&mc3, a.W3c, a.E, a.f, a.d, 64) || !encode_scales(&ms1, a.W1s, a.E, a.f, a.d, 64) ||
      !encode_scales(&ms3, a.W3s, a.E, a.f, a.d, 64) || !encode_tokens(&mh, a.h, a.S, a.f, BN) ||
      !encode_codes(&mc2, a.W2c, a.E, a.d, a.f, 128) || !encode_scales(&ms2, a.W2s, a.E, a.d, a.f, 128))
    return cudaErrorInvalidValue;
  Q4Params p1{};
  p1.offsets = a.offsets;
  p1.status = a.status;
  p1.S = a.S;
  p1.clock_probe = a.clock_probe;
  p1.out = a.h;
  p1.out_ld = a.f;
  p1.E = a.E;
  p1.num_kq = (a.d + KQ - 1) / KQ;
  p1.n_out = a.f;
  p1.n_blocks = a.f / 64;
  p1.splits = 1;
  p1.kq_per_split = p1.num_kq;
  cudaError_t err = launch_q4_one<Q4_SWIGLU, BN>(mx, mc1, mc3, ms1, ms3, p1, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  if (a.between && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;
  Q4Params p2{};
  p2.offsets = a.offsets;
  p2.status = a.status;
  p2.S = a.S;
  p2.clock_probe = a.clock_probe ? a.clock_probe + 4 : nullptr;
  p2.out = a.partials;
  p2.out_ld = a.d;
  p2.part_stride = a.S * (int64_t)a.d;
  p2.E = a.E;
  p2.num_kq = (a.f + KQ - 1) / KQ;
  p2.n_out = a.d;
  p2.n_blocks = (a.d + 127) / 128;
  p2.kq_per_split = (p2.num_kq + a.splits - 1) / a.splits;
  p2.splits = (p2.num_kq + p2.kq_per_split - 1) / p2.kq_per_split;
  return launch_q4_one<Q4_PARTIAL, BN>(mh, mc2, mc2, ms2, ms2, p2, a.num_sms, s, a.pdl && !a.between);
}

}  // namespace

void q4_params(int64_t T, int32_t k, int32_t d, int32_t f, int32_t E, int num_sms, int32_t* bn, int32_t* splits) {
  // token tile: 16 while the mean slots per expert fit it, 32 up to a mean
  // of 22, else twice the mean, so that an expert's slots usually fit one
  // tile (a second tile streams the expert's weights again).  The
  // integer-MMA kernel costs far less per weight byte at 16 tokens than at
  // 32, enough that re-reading the weights of experts that spill into a
  // second 16-token tile still wins: 0.371 -> 0.227 ms at T = 40, 0.371 ->
  // 0.320 ms at T = 64 (8 experts, top-2); 32-token integer-MMA tiles beat
  // 64-token dequantising ones by 2-3 % from T = 65 to 88 and lose at 96.
  const int64_t mean = (T * k + E - 1) / E;
  int64_t b = mean <= 16 ? 16 : mean <= 22 ? 32 : ((2 * mean + 15) / 16) * 16;
  if (b < 16) b = 16;
  if (b > 64) b = 128;
  else if (b > 32) b = 64;
  else if (b > 16) b = 32;
  *bn = (int32_t)b;
  // split K of the down projection as the bf16 streaming schedule does
  // (fewest waves x (stages per tile + 1) + one stage per partial plane); K
  // goes in stages of the kernel the token tile selects
  const int32_t kq_inputs = b <= 32 ? q4i8_stage_inputs((int32_t)b) : KQ;
  const int32_t num_kq = (f + kq_inputs - 1) / kq_inputs;
  const int64_t touched = T * k < E ? T * k : E;
  const int64_t base = touched * ((d + 127) / 128);
  int32_t best = 1;
  int64_t best_cost = INT64_MAX;
  for (int32_t sp = 1; sp <= 16 && sp <= num_kq; ++sp) {
    const int32_t kps = (num_kq + sp - 1) / sp;
    const int32_t real = (num_kq + kps - 1) / kps;
    const int64_t waves = (base * real + num_sms - 1) / num_sms;
    const int64_t cost = waves * (kps + 1) + real;
    if (cost < best_cost) {
      best_cost = cost;
      best = real;
    }
  }
  *splits = best;
}

int32_t q4_effective_splits(int32_t f, int32_t splits, int32_t bn) {
  const int32_t kq_inputs = bn <= 32 ? q4i8_stage_inputs(bn) : KQ;
  const int32_t num_kq = (f + kq_inputs - 1) / kq_inputs;
  const int32_t kps = (num_kq + splits - 1) / splits;
  return (num_kq + kps - 1) / kps;
}

cudaError_t launch_expert_gemms_q4(const ExpertGemmQ4Args& a, cudaStream_t s) {
  // token tiles of 16 and 32: the integer-MMA kernels (expert_gemm_q4i8.cu)
  if (a.act_q && a.bn <= 32) return launch_expert_gemms_q4i8(a, s);
  switch (a.bn) {
    case 16: return launch_q4<16>(a, s);
    case 32: return launch_q4<32>(a, s);
    case 64: return launch_q4<64>(a, s);
    default: return launch_q4<128>(a, s);
  }
}

cudaError_t launch_quantize_q4(const uint16_t* W, int32_t E, int32_t R, int32_t K, uint8_t* codes, uint16_t* scales,
                               cudaStream_t s) {
  const int64_t words = (int64_t)E * R * (K / 8);
  const int64_t blocks = (words + 255) / 256;
  quantize_q4_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(W),
                                                       reinterpret_cast<uint32_t*>(codes), scales, words, R, K);
  return cudaGetLastError();
}

}  // namespace moe
