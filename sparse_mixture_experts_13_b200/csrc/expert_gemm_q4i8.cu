// 4-bit expert GEMMs on the integer tensor-core MMA (tcgen05.mma kind::i8),
// for token tiles of 16 and 32 -- the decode regime, where the bf16
// dequantising kernels are bound by how fast MMAs are issued, not by HBM.
//
// Sources: as expert_gemm_q4.cu ("How Mixtral 8x7B uses mixture of experts",
// "Quantization asymmetry"; "Mixtral 8x7B — MoE Complete Guide", "4-bit
// Quantization for Single GPU"; the expert of "Mixtral", "MoE Layer").  Same
// weight format and the same function; only the arithmetic route differs.
//
// A 64-input block of a 4-bit weight row and a token's activations give an
// exact integer product, scaled afterwards:
//   w[r, i] = (c[r, i] - 8) * s[r, b]                   b = i / 64 (the format)
//   x[t, i] = q[t, i] * a[t] (+ rounding),  |q| <= 32639,  a[t] = max|x[t]| / 32639
//   q = 256 * qh + ql,  qh, ql signed bytes in [-127, 127]
//   sum_i w x = a[t] * sum_b s[r, b] * (256 * H[r, t, b] + L[r, t, b])
//   H = sum_{i in b} (c - 8) * qh,  L = sum_{i in b} (c - 8) * ql   (int32, exact)
// |256 H + L| < 2^24, so its conversion to fp32 is exact; the quantisation of
// x costs at most half a step, a[t] / 2, per element (relative 1.5e-5 of the
// row's largest value).
//
// quantize_act_kernel writes q as two planes of signed bytes (high, low),
// one row per token slot, with each group of 8 inputs stored in the order
// 0 4 1 5 2 6 3 7: the order in which a 32-bit code word's low nibbles, then
// its high nibbles, land in tensor memory (nibble m of the word is input
// 2m, nibble m + 4 input 2m + 1).
//
// expert_gemm_q4i8_kernel: the streaming schedule of the 4-bit kernels
// (weights = M operand, 128 rows; tokens = N operand), per stage of 128
// inputs:
//   warp 0       TMA: the codes of 128 weight rows (64-byte swizzle), their
//                scales, and the tokens' high and low rows (N = 2 BN rows of
//                128 bytes, 128-byte swizzle);
//   warps 1-4    one per tensor-memory lane quarter (warp w owns rows
//                32 (w % 4) .. +31): expand the row's codes to signed bytes
//                (c - 8) in its lanes of the stage's A buffer, then -- once
//                the stage's MMAs are done -- read the two blocks'
//                accumulators, scale them by s[r, b] and add them into fp32
//                registers; at the tile's end multiply by a[t] and store
//                (SiLU * mul through shared memory for the gate/up GEMM,
//                fp32 split-K partials for the down GEMM).
// The MMAs of block 0 are issued by warp 4 and those of block 1 by warp 1
// (2 MMAs of K = 32 into the block's own accumulator each, then a commit):
// an MMA's issue slows several-fold when another ALU-busy warp shares the
// issuing thread's scheduler, so each issuer only shares it with its own
// work (warp 0, the TMA producer, is nearly idle).  Accumulators are
// double-buffered by stage parity and A buffers four deep, so the tensor
// core runs a stage's MMAs while the workers scale the previous stage and
// expand the next.
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int KQ8 = 128;                    // inputs per stage (two 64-input scale blocks)
constexpr int kI8Threads = 160;             // warp 0 producer, warps 1-4 workers
constexpr int kI8Workers = 128;
constexpr int kI8ABufs = 4;
constexpr int kI8ACols = KQ8 / 4;           // TMEM columns of one stage's A (4 signed bytes each)
constexpr int kI8ACol0 = 256;               // A buffers start here; accumulators below
constexpr int kI8TmemCols = 512;
constexpr int kI8CodeBytes = 128 * KQ8 / 2;  // 128 rows x 64 bytes
constexpr int kI8ScaleBytes = 1024;          // 2 blocks x 128 rows x bf16 = 512, padded
constexpr int kQMax = 32639;                 // largest |q|: high and low bytes stay in [-127, 127]

enum : int { I8_SWIGLU = 0, I8_PARTIAL = 1 };

__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                          // D: s32
         | (1u << 7)                        // A: signed 8-bit
         | (1u << 10)                       // B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int EPI, int BN>
struct I8Cfg {
  static constexpr int N = 2 * BN;                       // MMA N: the tokens' high bytes, then low bytes
  static constexpr int B_BYTES = N * KQ8;                // N rows x 128 signed bytes
  static constexpr int STAGE_BYTES = B_BYTES + kI8CodeBytes + kI8ScaleBytes;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 12 ? 12 : (200 * 1024) / STAGE_BYTES;
  static constexpr int XBUF_BYTES = (EPI == I8_SWIGLU) ? BN * 64 * 4 : 0;
  static constexpr int BAR_BYTES = (2 * STAGES + kI8ABufs + 2) * 8;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + XBUF_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_i8(128, N);
  static_assert(BN == 16 || BN == 32, "token tile");
  static_assert(STAGES > kI8ABufs, "an A buffer is reused before its stage's barrier can move on twice");
  static_assert(B_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "1024-byte aligned pieces");
  static_assert(4 * N + kI8ABufs * kI8ACols <= kI8TmemCols && 4 * N <= kI8ACol0, "tensor memory");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct I8Params {
  const int32_t* offsets;
  uint32_t* status;
  void* out;            // bf16 h, or fp32 partials
  const float* act_scale;  // [S] a[t] of the quantised activations
  int64_t out_ld;
  int64_t part_stride;
  int32_t E;
  int32_t num_kq;       // stages over K (K / 128, rounded up)
  int32_t n_out;        // output columns (d_ff or d_model)
  int32_t n_blocks;     // weight blocks per expert (64 rows of W1 and W3, or 128 of W2)
  int32_t splits;
  int32_t kq_per_split;
  int64_t S;
  uint64_t* clock_probe;
};

struct I8Tile {
  int32_t row0, m_valid, n0, split, kq0, kq1, e;
};

template <int EPI, int BN>
__device__ __forceinline__ void i8_decode_tile(const I8Params& p, const int32_t* s_off, const int32_t* s_base,
                                               int32_t tile, I8Tile& t) {
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
  t.n0 = wb * (EPI == I8_SWIGLU ? 64 : 128);
  t.kq0 = t.split * p.kq_per_split;
  t.kq1 = min(p.num_kq, t.kq0 + p.kq_per_split);
}

// D[tmem] (+)= A[tmem] * B[smem]^T, signed 8-bit A and B, int32 D.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive columns from registers: thread i writes lane
// (base lane + i).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Four 4-bit codes (the low nibbles of the bytes of x) -> the signed bytes c - 8:
// c ^ 8 is the 4-bit two's complement of c - 8; bit 3 then fills bits 4-7.
__device__ __forceinline__ uint32_t codes_to_s8(uint32_t x) {
  const uint32_t y = (x & 0x0F0F0F0Fu) ^ 0x08080808u;
  return y | ((y & 0x08080808u) * 30u);  // 8 * 30 = 0xF0 per byte, no carries
}

template <int EPI, int BN>
__global__ void __launch_bounds__(kI8Threads, 1)
    expert_gemm_q4i8_kernel(const __grid_constant__ CUtensorMap map_act,  // [2][S][K] signed bytes
                            const __grid_constant__ CUtensorMap map_ca,   // codes: W1 or W2
                            const __grid_constant__ CUtensorMap map_cb,   // codes: W3
                            const __grid_constant__ CUtensorMap map_sa,   // scales: W1 or W2
                            const __grid_constant__ CUtensorMap map_sb,   // scales: W3
                            I8Params p) {
  using C = I8Cfg<EPI, BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int N = C::N;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_base[33];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [B tile (high rows, low rows) | codes | scales]
  float* xbuf = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::XBUF_BYTES);
  uint64_t* full_bar = bars;              // TMA bytes of a stage
  uint64_t* done_bar = bars + STAGES;     // both blocks' MMAs of a stage completed (2 commits)
  uint64_t* afull_bar = bars + 2 * STAGES;  // the 4 workers wrote an A buffer
  uint64_t* dfree_bar = afull_bar + kI8ABufs;  // the 4 workers read an accumulator set

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe);

  if (tid == 0) {
    tma_prefetch_desc(&map_act);
    tma_prefetch_desc(&map_ca);
    tma_prefetch_desc(&map_sa);
    if (EPI == I8_SWIGLU) {
      tma_prefetch_desc(&map_cb);
      tma_prefetch_desc(&map_sb);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&done_bar[s], 2);
    }
    for (int a = 0; a < kI8ABufs; ++a) mbar_init(&afull_bar[a], 4);
    for (int a = 0; a < 2; ++a) mbar_init(&dfree_bar[a], 4);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kI8TmemCols);
    tmem_relinquish();
  }
  pdl_wait();     // offsets, quantised activations and their scales of the kernels before this one
  pdl_trigger();  // the next kernel may start its own set-up
  if (tid == 64) {
    s_abort = 0;
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
        I8Tile t;
        i8_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
        for (int32_t kq = t.kq0; kq < t.kq1; ++kq) {
          if (!mbar_wait(&done_bar[stage], phase ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          uint8_t* c_dst = st + C::B_BYTES;
          uint8_t* s_dst = c_dst + kI8CodeBytes;
          mbar_arrive_expect_tx(&full_bar[stage], C::B_BYTES + kI8CodeBytes + 512);
          const int32_t kx = kq * KQ8;
          tma_load_3d(&map_act, &full_bar[stage], st, kx, t.row0, 0);               // high bytes
          tma_load_3d(&map_act, &full_bar[stage], st + BN * KQ8, kx, t.row0, 1);    // low bytes
          if (EPI == I8_SWIGLU) {
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
      // Let every load this thread issued land before the CTA may exit.
      for (int s = 0; s < STAGES; ++s) {
        if (s < issued) {
          const int64_t uses = (issued - s + STAGES - 1) / STAGES;
          mbar_wait(&full_bar[s], (uint32_t)((uses - 1) & 1), nullptr);
        }
      }
    }
  } else {
    // ------------------------------------------------ workers (warps 1..4)
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int r = q * 32 + lane;            // weight row of the A tile
    const bool issuer = (warp == 4 || warp == 1);
    const int my_block = warp == 4 ? 0 : 1;
    // codes of row r: 64 bytes; 16-byte chunk c (inputs 32c .. 32c+31) at
    // chunk c ^ ((r >> 1) & 3) (64-byte swizzle); scale of block b
    uint32_t c_off[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) c_off[c] = (uint32_t)r * 64 + (((uint32_t)c ^ (uint32_t)((r >> 1) & 3)) << 4);
    uint32_t s_off_b[2];
#pragma unroll
    for (int b = 0; b < 2; ++b)
      s_off_b[b] = kI8CodeBytes + 2 * ((EPI == I8_SWIGLU) ? ((r >> 6) * 128 + b * 64 + (r & 63)) : (b * 128 + r));
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);

    float acc[BN];
#pragma unroll
    for (int t = 0; t < BN; ++t) acc[t] = 0.f;
    float sc_prev[2] = {0.f, 0.f};
    I8Tile t_prev{};
    bool ok = true;
    int64_t i = 0;  // stages expanded so far

    // Scale stage j (its accumulator set j & 1) into acc with that stage's
    // block scales; release the set.
    auto scale_stage = [&](int64_t j, const float (&sc)[2], bool go) -> bool {
      bool w_ok = go && mbar_wait(&done_bar[j % STAGES], (uint32_t)((j / STAGES) & 1), &s_abort);
      tc_fence_after();
      if (w_ok) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint32_t d = lane_base + (uint32_t)((j & 1) * 2 * N + b * N);
          uint32_t hi[BN], lo[BN];
          if constexpr (BN == 16) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(d, v);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              hi[t] = v[t];
              lo[t] = v[16 + t];
            }
          } else {
            tmem_ld_32x32b_x32(d, hi);
            tmem_ld_32x32b_x32(d + 32, lo);
            tmem_ld_wait();
          }
#pragma unroll
          for (int t = 0; t < BN; ++t) {
            const int32_t vi = (int32_t)hi[t] * 256 + (int32_t)lo[t];
            acc[t] = fmaf(__int2float_rn(vi), sc[b], acc[t]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dfree_bar[j & 1]);
      return w_ok;
    };

    // The tile's outputs: a[t] * acc, SiLU * mul or fp32 partials.
    auto epilogue = [&](const I8Tile& t) {
      float a[BN];
#pragma unroll
      for (int tk = 0; tk < BN; ++tk) a[tk] = tk < t.m_valid ? p.act_scale[t.row0 + tk] * acc[tk] : 0.f;
      if (EPI == I8_SWIGLU) {
        // rows 0..63: W1 projection of column n0 + r; rows 64..127: W3 of column n0 + r - 64
        uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
        if (r >= 64) {
#pragma unroll
          for (int tk = 0; tk < BN; ++tk) xbuf[tk * 64 + (r - 64)] = a[tk];
        }
        named_bar_sync(1, kI8Workers);
        if (r < 64 && t.n0 + r < p.n_out) {
#pragma unroll
          for (int tk = 0; tk < BN; ++tk) {
            if (tk < t.m_valid && MOE_DCHECK(p.status, t.row0 + tk < p.S)) {
              const float hv = silu_f32(a[tk]) * xbuf[tk * 64 + r];
              out[(int64_t)(t.row0 + tk) * p.out_ld + t.n0 + r] = (uint16_t)(pack_bf16x2(hv, 0.f) & 0xFFFFu);
            }
          }
        }
        named_bar_sync(1, kI8Workers);
      } else {
        float* out = reinterpret_cast<float*>(p.out) + (int64_t)t.split * p.part_stride;
        if (t.n0 + r < p.n_out) {
#pragma unroll
          for (int tk = 0; tk < BN; ++tk)
            if (tk < t.m_valid && MOE_DCHECK(p.status, t.row0 + tk < p.S))
              out[(int64_t)(t.row0 + tk) * p.out_ld + t.n0 + r] = a[tk];
        }
      }
#pragma unroll
      for (int tk = 0; tk < BN; ++tk) acc[tk] = 0.f;
    };

    // Every worker runs the same stages and epilogues even after a wait gave
    // up (it then skips tensor-memory and MMA work), so the workers' named
    // barriers always match; waits return at once once s_abort is set.
    for (int32_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
      I8Tile t;
      i8_decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
      for (int32_t kq = t.kq0; kq < t.kq1; ++kq, ++i) {
        const int stage = (int)(i % STAGES);
        // ---- expand stage i into A buffer i % 4 (free once stage i - 4's MMAs are done)
        bool w_ok = ok && mbar_wait(&full_bar[stage], (uint32_t)((i / STAGES) & 1), &s_abort);
        if (w_ok && i >= kI8ABufs) {
          const int64_t j = i - kI8ABufs;
          w_ok = mbar_wait(&done_bar[j % STAGES], (uint32_t)((j / STAGES) & 1), &s_abort);
        }
        tc_fence_after();
        const uint8_t* st = smem + stage * C::STAGE_BYTES;
        float sc_cur[2] = {0.f, 0.f};
        if (w_ok) {
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(st + C::B_BYTES + c_off[c]);
            const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              v[8 * c + 2 * k] = codes_to_s8(words[k]);             // inputs 0 4 1 5 of the group
              v[8 * c + 2 * k + 1] = codes_to_s8(words[k] >> 4);    // inputs 2 6 3 7
            }
          }
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint16_t sb = *reinterpret_cast<const uint16_t*>(st + C::B_BYTES + s_off_b[b]);
            sc_cur[b] = __uint_as_float((uint32_t)sb << 16);
          }
          tmem_st_32x32b_x32(lane_base + kI8ACol0 + (uint32_t)((i % kI8ABufs) * kI8ACols), v);
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull_bar[i % kI8ABufs]);
        // ---- this warp's block of stage i on the tensor core
        if (issuer && w_ok) {
          w_ok = mbar_wait(&afull_bar[i % kI8ABufs], (uint32_t)((i / kI8ABufs) & 1), &s_abort);
          if (w_ok && i >= 2) w_ok = mbar_wait(&dfree_bar[i & 1], (uint32_t)(((i - 2) / 2) & 1), &s_abort);
          tc_fence_after();
          if (w_ok && lane == 0) {
            const uint32_t d = tmem_base + (uint32_t)((i & 1) * 2 * N + my_block * N);
            const uint32_t a0 = tmem_base + kI8ACol0 + (uint32_t)((i % kI8ABufs) * kI8ACols + my_block * 16);
            // K step kk of the stage: 32 bytes into the 128-byte swizzled rows
            const uint64_t b_desc = make_sdesc_sw128(smem_u32(st));
            umma_i8_ts(d, a0, b_desc + (uint64_t)((my_block * 64) >> 4), C::IDESC, 0u);
            umma_i8_ts(d, a0 + 8, b_desc + (uint64_t)((my_block * 64 + 32) >> 4), C::IDESC, 1u);
            umma_commit(&done_bar[stage]);
          }
          __syncwarp();
        }
        // ---- scale the previous stage (and finish its tile when this stage starts a new one)
        if (i >= 1) {
          w_ok = scale_stage(i - 1, sc_prev, w_ok) && w_ok;
          if (kq == t.kq0) epilogue(t_prev);
        }
        sc_prev[0] = sc_cur[0];
        sc_prev[1] = sc_cur[1];
        t_prev = t;
        if (!w_ok) {
          ok = false;
          s_abort = 1;
        }
      }
    }
    if (i >= 1) {
      if (!scale_stage(i - 1, sc_prev, ok)) ok = false;
      epilogue(t_prev);
    }
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      s_abort = 1;
    }
    // Every MMA this CTA issued has completed before tensor memory is freed:
    // each stage's two commits arrive on its done barrier, waited for here
    // (bounded) for the last STAGES stages.
    if (issuer && lane == 0) {
      for (int64_t j = (i > STAGES ? i - STAGES : 0); j < i; ++j)
        mbar_wait(&done_bar[j % STAGES], (uint32_t)((j / STAGES) & 1), nullptr, kWaitLimitNs / 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe + 2);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kI8TmemCols);
  }
}

// One warp per row r < offsets[E] of `in` [S, K] bf16: a = max |x[r]|,
// q = clamp(rint(x * 32639 / a), -32639, 32639), low byte ((q + 128) & 255) - 128,
// high byte (q - low) / 256, written to planes [2][S][K] in the MMA's K order
// (0 4 1 5 2 6 3 7 per group of 8); scale[r] = a / 32639.
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ in,
                                                           const int32_t* __restrict__ offsets, int32_t E, int32_t K,
                                                           int64_t plane, int8_t* __restrict__ q8,
                                                           float* __restrict__ scale) {
  pdl_wait();  // the rows (and offsets) of the kernels before this one
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t rows = offsets[E];
  const int nvec = K >> 3;
  for (int64_t row = w0; row < rows; row += nw) {
    const uint4* src = reinterpret_cast<const uint4*>(in + row * (int64_t)K);
    float amax = 0.f;
    for (int v = lane; v < nvec; v += 32) {
      const uint4 x = src[v];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float inv = amax > 0.f ? (float)kQMax / amax : 0.f;
    if (lane == 0) scale[row] = amax / (float)kQMax;
    for (int v = lane; v < nvec; v += 32) {
      const uint4 x = src[v];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      int qv[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qv[2 * j] = max(-kQMax, min(kQMax, __float2int_rn(__uint_as_float(w[j] << 16) * inv)));
        qv[2 * j + 1] = max(-kQMax, min(kQMax, __float2int_rn(__uint_as_float(w[j] & 0xFFFF0000u) * inv)));
      }
      constexpr int kPerm[8] = {0, 4, 1, 5, 2, 6, 3, 7};
      uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
      for (int pos = 0; pos < 8; ++pos) {
        const int qq = qv[kPerm[pos]];
        const int lo = ((qq + 128) & 255) - 128;
        const int hi = (qq - lo) / 256;
        hw[pos >> 2] |= ((uint32_t)hi & 0xFFu) << (8 * (pos & 3));
        lw[pos >> 2] |= ((uint32_t)lo & 0xFFu) << (8 * (pos & 3));
      }
      const int64_t at = row * (int64_t)K + 8 * (int64_t)v;
      *reinterpret_cast<uint2*>(q8 + at) = make_uint2(hw[0], hw[1]);
      *reinterpret_cast<uint2*>(q8 + plane + at) = make_uint2(lw[0], lw[1]);
    }
  }
}

// [2][S][K] signed bytes as a 3-D map, box {128 bytes, box_rows, 1}, 128-byte swizzle
bool encode_act_planes(CUtensorMap* m, const void* base, int64_t S, int64_t K, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)S, 2};
  cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)(S * K)};
  cuuint32_t box[3] = {(cuuint32_t)KQ8, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_quantize_act(const uint16_t* in, const int32_t* offsets, int32_t E, int64_t S, int32_t K,
                                int8_t* q8, float* scale, int num_sms, cudaStream_t s, bool pdl) {
  int64_t blocks = (S + 7) / 8;  // 8 warps per block
  if (blocks > 8 * (int64_t)num_sms) blocks = 8 * (int64_t)num_sms;
  if (blocks < 1) blocks = 1;
  return launch_k(quantize_act_kernel, dim3((unsigned)blocks), dim3(256), 0, s, pdl, in, offsets, E, K, S * (int64_t)K,
                  q8, scale);
}

template <int EPI, int BN>
cudaError_t launch_i8_one(const CUtensorMap& act, const CUtensorMap& ca, const CUtensorMap& cb, const CUtensorMap& sa,
                          const CUtensorMap& sb, const I8Params& p, int num_sms, cudaStream_t s, bool pdl) {
  using C = I8Cfg<EPI, BN>;
  cudaError_t err =
      cudaFuncSetAttribute(expert_gemm_q4i8_kernel<EPI, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_k(expert_gemm_q4i8_kernel<EPI, BN>, dim3(num_sms), dim3(kI8Threads), C::SMEM_BYTES, s, pdl, act, ca,
                  cb, sa, sb, p);
}

template <int BN>
cudaError_t launch_i8(const ExpertGemmQ4Args& a, cudaStream_t s) {
  const int64_t S = a.S;
  CUtensorMap mx, mc1, mc3, ms1, ms3, mh, mc2, ms2;
  if (!encode_act_planes(&mx, a.act_q, S, a.d, BN) || !encode_codes(&mc1, a.W1c, a.E, a.f, a.d, 64) ||
      !encode_codes(&mc3, a.W3c, a.E, a.f, a.d, 64) || !encode_scales(&ms1, a.W1s, a.E, a.f, a.d, 64) ||
      !encode_scales(&ms3, a.W3s, a.E, a.f, a.d, 64) || !encode_act_planes(&mh, a.act_q, S, a.f, BN) ||
      !encode_codes(&mc2, a.W2c, a.E, a.d, a.f, 128) || !encode_scales(&ms2, a.W2s, a.E, a.d, a.f, 128))
    return cudaErrorInvalidValue;
  // x_perm -> planes (K = d)
  cudaError_t err = launch_quantize_act(a.x_perm, a.offsets, a.E, S, a.d, a.act_q, a.act_scale, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  I8Params p1{};
  p1.offsets = a.offsets;
  p1.status = a.status;
  p1.out = a.h;
  p1.act_scale = a.act_scale;
  p1.out_ld = a.f;
  p1.E = a.E;
  p1.num_kq = (a.d + KQ8 - 1) / KQ8;
  p1.n_out = a.f;
  p1.n_blocks = a.f / 64;
  p1.splits = 1;
  p1.kq_per_split = p1.num_kq;
  p1.S = S;
  p1.clock_probe = a.clock_probe;
  err = launch_i8_one<I8_SWIGLU, BN>(mx, mc1, mc3, ms1, ms3, p1, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  if (a.between && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;
  const bool pdl2 = a.pdl && !a.between;
  // h -> planes (K = f), reusing the buffer once the gate/up GEMM is done
  err = launch_quantize_act(a.h, a.offsets, a.E, S, a.f, a.act_q, a.act_scale, a.num_sms, s, pdl2);
  if (err != cudaSuccess) return err;
  I8Params p2{};
  p2.offsets = a.offsets;
  p2.status = a.status;
  p2.out = a.partials;
  p2.act_scale = a.act_scale;
  p2.out_ld = a.d;
  p2.part_stride = S * (int64_t)a.d;
  p2.E = a.E;
  p2.num_kq = (a.f + KQ8 - 1) / KQ8;
  p2.n_out = a.d;
  p2.n_blocks = (a.d + 127) / 128;
  p2.kq_per_split = (p2.num_kq + a.splits - 1) / a.splits;
  p2.splits = (p2.num_kq + p2.kq_per_split - 1) / p2.kq_per_split;
  p2.S = S;
  p2.clock_probe = a.clock_probe ? a.clock_probe + 4 : nullptr;
  return launch_i8_one<I8_PARTIAL, BN>(mh, mc2, mc2, ms2, ms2, p2, a.num_sms, s, pdl2);
}

}  // namespace

cudaError_t launch_expert_gemms_q4i8(const ExpertGemmQ4Args& a, cudaStream_t s) {
  return a.bn <= 16 ? launch_i8<16>(a, s) : launch_i8<32>(a, s);
}

}  // namespace moe
