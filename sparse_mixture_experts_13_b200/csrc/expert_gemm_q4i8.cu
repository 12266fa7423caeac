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
//   q = 256 * qh + ql,  qh in [-127, 127], ql in [-128, 127] (signed bytes)
//   sum_i w x = a[t] / 16 * sum_b s[r, b] * (256 * H[r, t, b] + L[r, t, b])
//   H = sum_{i in b} 16 (c - 8) * qh,  L = sum_{i in b} 16 (c - 8) * ql   (int32, exact)
// The weights enter the MMA as 16 (c - 8), a signed byte that one mask and
// one XOR make from a nibble.  |256 H + L| < 2^29; its conversion to fp32
// rounds at 2^-24 relative, below the fp32 sums that follow.  The
// quantisation of x costs at most half a step, a[t] / 2, per element
// (relative 1.5e-5 of the row's largest value).
//
// quantize_act_kernel writes q, one token slot per row, straight into the
// shared-memory image of the GEMMs' token operand, so that one bulk copy
// loads a stage's: per token tile (BN slots of one expert) and stage of KS
// inputs, KS / 128 slices of [2 BN rows (the high bytes of the BN slots,
// then the low bytes) x 128 bytes], with the 128-byte swizzle of the MMA's
// K-major layout (16-byte chunk c of row n at chunk c ^ (n % 8)).  Each
// group of 8 inputs is stored in the order 0 4 1 5 2 6 3 7: the order in
// which a 32-bit code word's low nibbles, then its high nibbles, land in
// tensor memory (nibble m of the word is input 2m, nibble m + 4 input 2m + 1).
//
// expert_gemm_q4i8_kernel: the streaming schedule of the 4-bit kernels
// (weights = M operand, 128 rows; tokens = N operand), per stage of KS
// inputs (256 for 16-token tiles, 128 for 32), with one role per warp so
// that no warp waits on its own previous step:
//   warp 0       loads: the token operand (one bulk copy), the codes of 128
//                weight rows (TMA, rows of KS / 2 bytes, swizzled to match)
//                and their scales;
//   warps 1, 14  MMA issue, each for half of a stage's scale blocks (on
//                different schedulers): per block two K = 32 MMAs (A from
//                tensor memory) into its own accumulator columns, then one
//                commit per stage;
//   warps 2-5    expanders, one per tensor-memory lane quarter (warp w owns
//                rows 32 (w % 4) .. +31): the row's codes -> 16 (c - 8) into
//                its lanes of the stage's A buffer;
//   warps 6-13   scalers, two per lane quarter (one per half of the token
//                tile): read the stage's block accumulators, scale them by
//                s[r, b] into fp32 registers (two tokens per packed FMA) and,
//                at the tile's end, multiply by a[t] / 16 and store (SiLU *
//                mul through shared memory for the gate/up GEMM, fp32 split-K
//                partials for the down GEMM).
// A stage's shared memory is refilled once its scalers have read its scales
// (after its MMAs, which read its codes' expansion and token rows).  Wide
// stages keep the per-stage work of every role (barrier round trips, load
// and MMA issue) small against the bytes it moves.
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

// warps: 0 loads, 1 and 14 MMA issuers (the first and the second half of a
// stage's scale blocks), 2-5 expanders, 6-13 scalers (two per lane quarter,
// one per half of the token tile); warp w runs on scheduler w % 4 and
// reaches tensor-memory lanes 32 (w % 4) .. +31.  Measured slower at
// 16-token tiles: one issuer per block (four, twice the commits per stage)
// and two expanders per lane quarter (four more warps on the schedulers).
constexpr int kI8FirstScaler = 6;
constexpr int kI8FirstExtraIssuer = 14;
constexpr int kI8Scalers = 256;
constexpr int kI8ACol0 = 256;               // A buffers start here; accumulators below
constexpr int kI8TmemCols = 512;
constexpr int kQMax = 32639;                 // largest |q|: high byte in [-127, 127], low byte in [-128, 127]

enum : int { I8_SWIGLU = 0, I8_PARTIAL = 1 };

__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                          // D: s32
         | (1u << 7)                        // A: signed 8-bit
         | (1u << 10)                       // B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// inputs per stage for a token tile (the tiled token operand is laid out by it)
__host__ __device__ constexpr int i8_stage_inputs(int bn) { return bn <= 16 ? 256 : 128; }

template <int EPI, int BN>
struct I8Cfg {
  static constexpr int KS = i8_stage_inputs(BN);         // inputs per stage
  static constexpr int NB = KS / 64;                     // scale blocks per stage
  static constexpr int KH = KS / 128;                    // 128-byte slices of a token row per stage
  static constexpr int ISSUERS = 2;
  static constexpr int THREADS = 32 * (kI8FirstExtraIssuer + ISSUERS - 1);
  static constexpr int N = 2 * BN;                       // MMA N: the tokens' high bytes, then low bytes
  static constexpr int B_BYTES = KH * N * 128;           // token operand of a stage
  static constexpr int ROW_BYTES = KS / 2;               // codes of one weight row per stage
  static constexpr int CODE_BYTES = 128 * ROW_BYTES;
  static constexpr int SCALE_BYTES = 128 * NB * 2;
  static constexpr int STAGE_BYTES = B_BYTES + CODE_BYTES + 1024;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 16 ? 16 : (200 * 1024) / STAGE_BYTES;
  static constexpr int ACOLS = KS / 4;                   // TMEM columns of a stage's A (4 signed bytes each)
  static constexpr int ABUFS = (kI8TmemCols - kI8ACol0) / ACOLS;
  static constexpr int DCOLS = NB * N;                   // accumulator columns of a stage
  static constexpr int DBUFS = kI8ACol0 / DCOLS;
  static constexpr int XBUF_BYTES = (EPI == I8_SWIGLU) ? BN * 64 * 4 : 0;
  static constexpr int BAR_BYTES = (3 * STAGES + ABUFS + DBUFS) * 8;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + XBUF_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_i8(128, N);
  static_assert(BN == 16 || BN == 32, "token tile");
  static_assert(SCALE_BYTES <= 1024, "scales of a stage");
  static_assert(ABUFS >= 2 && DBUFS >= 2, "double-buffered tensor memory");
  static_assert(STAGES > ABUFS && STAGES > DBUFS,
                "a stage's barrier must not move on twice while an A buffer or accumulator set waits on it");
  static_assert(B_BYTES % 1024 == 0 && CODE_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0,
                "1024-byte aligned pieces (swizzle atoms)");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct I8Params {
  const int32_t* offsets;
  uint32_t* status;
  void* out;            // bf16 h, or fp32 partials
  const uint8_t* act;   // the tiled token operand: [tile][stage] of B_BYTES
  const float* act_scale;  // [S] a[t] of the quantised activations
  int64_t out_ld;
  int64_t part_stride;
  int32_t E;
  int32_t num_kq;       // stages over K (K / KS, rounded up)
  int32_t n_out;        // output columns (d_ff or d_model)
  int32_t n_blocks;     // weight blocks per expert (64 rows of W1 and W3, or 128 of W2)
  int32_t splits;
  int32_t kq_per_split;
  int64_t S;
  uint64_t* clock_probe;
};

struct I8Tile {
  int32_t row0, m_valid, n0, split, kq0, kq1, e, tau;  // tau: token tile over all experts
};

template <int EPI, int BN>
__device__ __forceinline__ void i8_decode_tile(const I8Params& p, const int32_t* s_off, const int32_t* s_base,
                                               const int32_t* s_tau, int32_t tile, I8Tile& t) {
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
  t.tau = s_tau[e] + tb;
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

// 32 lanes x 16 consecutive columns from registers: thread i writes lane
// (base lane + i).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Position in a ring of N barrier-guarded slots: the slot and the parity of
// its current use (32-bit counters instead of divisions of a 64-bit index).
template <int N>
struct RingPos {
  uint32_t slot = 0, phase = 0;
  __device__ __forceinline__ void next() {
    if (++slot == (uint32_t)N) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// 32 lanes x W consecutive columns into registers (W = 8 or 16).
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
  if constexpr (W == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    static_assert(W == 8, "column count");
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  }
}

// Wait for this thread's tensor-memory loads; the registers they filled are
// passed through an empty asm after the wait so that no use of them is
// scheduled before it.
template <int W>
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t* a, uint32_t* b) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < W; ++j) asm volatile("" : "+r"(a[j]), "+r"(b[j]));
}

// Eight 4-bit codes of a word -> 16 (c - 8) as signed bytes, in two words:
// 16 c ^ 0x80 reads as 16 (c - 8) in two's complement, so masking a nibble
// into the high half of its byte and flipping the top bit is the whole
// conversion.  lo: the low nibbles (inputs 0 4 1 5 of the group of 8), hi:
// the high nibbles (inputs 2 6 3 7).  The factor 16 is taken out of the scale.
__device__ __forceinline__ uint32_t codes_lo_s8x16(uint32_t x) { return ((x << 4) & 0xF0F0F0F0u) ^ 0x80808080u; }
__device__ __forceinline__ uint32_t codes_hi_s8x16(uint32_t x) { return (x & 0xF0F0F0F0u) ^ 0x80808080u; }

template <int EPI, int BN>
__global__ void __launch_bounds__(I8Cfg<EPI, BN>::THREADS, 1)
    expert_gemm_q4i8_kernel(const __grid_constant__ CUtensorMap map_ca,   // codes: W1 or W2
                            const __grid_constant__ CUtensorMap map_cb,   // codes: W3
                            const __grid_constant__ CUtensorMap map_sa,   // scales: W1 or W2
                            const __grid_constant__ CUtensorMap map_sb,   // scales: W3
                            I8Params p) {
  using C = I8Cfg<EPI, BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int N = C::N;
  constexpr int NB = C::NB;
  constexpr int ABUFS = C::ABUFS;
  constexpr int DBUFS = C::DBUFS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_base[33];
  __shared__ int32_t s_tau[33];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [token operand | codes | scales]
  float* xbuf = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::XBUF_BYTES);
  uint64_t* full_bar = bars;                  // the loads of a stage
  uint64_t* mma_bar = bars + STAGES;          // the stage's MMAs completed (one commit per issuer)
  uint64_t* free_bar = bars + 2 * STAGES;     // the 8 scalers read the stage's scales
  uint64_t* afull_bar = bars + 3 * STAGES;    // the 4 expanders wrote an A buffer
  uint64_t* dfree_bar = afull_bar + ABUFS;    // the 8 scalers read an accumulator set

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe);

  if (tid == 0) {
    tma_prefetch_desc(&map_ca);
    tma_prefetch_desc(&map_sa);
    if (EPI == I8_SWIGLU) {
      tma_prefetch_desc(&map_cb);
      tma_prefetch_desc(&map_sb);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&mma_bar[s], C::ISSUERS);
      mbar_init(&free_bar[s], 8);
    }
    for (int a = 0; a < ABUFS; ++a) mbar_init(&afull_bar[a], 4);
    for (int a = 0; a < DBUFS; ++a) mbar_init(&dfree_bar[a], 8);
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
    int32_t acc = 0, taus = 0;
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
      const int32_t tiles_e = M_e > 0 ? (M_e + BN - 1) / BN : 0;
      s_tau[e] = taus;
      taus += tiles_e;
      acc += tiles_e * p.n_blocks * p.splits;
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
      // ------------------------------------------------ loads
      int64_t i = 0;
      RingPos<STAGES> sp;
      bool ok = true;
      for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        I8Tile t;
        i8_decode_tile<EPI, BN>(p, s_off, s_base, s_tau, tile, t);
        for (int32_t kq = t.kq0; kq < t.kq1; ++kq, ++i, sp.next()) {
          const int stage = (int)sp.slot;
          // the slot's previous use (parity phase ^ 1) must have been read
          if (i >= STAGES && !mbar_wait(&free_bar[stage], sp.phase ^ 1u, &s_abort)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          uint8_t* c_dst = st + C::B_BYTES;
          uint8_t* s_dst = c_dst + C::CODE_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], C::B_BYTES + C::CODE_BYTES + C::SCALE_BYTES);
          bulk_load(st, p.act + ((int64_t)t.tau * p.num_kq + kq) * C::B_BYTES, C::B_BYTES, &full_bar[stage]);
          const int32_t kx = kq * C::KS;
          if (EPI == I8_SWIGLU) {
            tma_load_3d(&map_ca, &full_bar[stage], c_dst, kx / 2, t.n0, t.e);
            tma_load_3d(&map_cb, &full_bar[stage], c_dst + 64 * C::ROW_BYTES, kx / 2, t.n0, t.e);
            tma_load_3d(&map_sa, &full_bar[stage], s_dst, t.n0, NB * kq, t.e);
            tma_load_3d(&map_sb, &full_bar[stage], s_dst + 64 * NB * 2, t.n0, NB * kq, t.e);
          } else {
            tma_load_3d(&map_ca, &full_bar[stage], c_dst, kx / 2, t.n0, t.e);
            tma_load_3d(&map_sa, &full_bar[stage], s_dst, t.n0, NB * kq, t.e);
          }
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      // Let every load this thread issued land before the CTA may exit.
      for (int s = 0; s < STAGES; ++s) {
        if (s < i) {
          const int64_t uses = (i - s + STAGES - 1) / STAGES;
          mbar_wait(&full_bar[s], (uint32_t)((uses - 1) & 1), nullptr);
        }
      }
    }
  } else if (warp == 1 || warp >= kI8FirstExtraIssuer) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuers
      // per stage: block b's two K = 32 MMAs into accumulator columns
      // (i % DBUFS) DCOLS + b N, then one commit; the two issuers (on
      // different schedulers) take the first and the second half of the blocks
      const int b_lo = warp == 1 ? 0 : NB / 2, b_hi = warp == 1 ? NB / 2 : NB;
      int64_t i = 0;
      RingPos<STAGES> sp;
      RingPos<ABUFS> ap;
      RingPos<DBUFS> dp;
      bool ok = true;
      for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        I8Tile t;
        i8_decode_tile<EPI, BN>(p, s_off, s_base, s_tau, tile, t);
        for (int32_t kq = t.kq0; kq < t.kq1; ++kq, ++i, sp.next(), ap.next(), dp.next()) {
          const int stage = (int)sp.slot;
          const int ab = (int)ap.slot, db = (int)dp.slot;
          ok = mbar_wait(&full_bar[stage], sp.phase, &s_abort) && mbar_wait(&afull_bar[ab], ap.phase, &s_abort) &&
               (i < DBUFS || mbar_wait(&dfree_bar[db], dp.phase ^ 1u, &s_abort));
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(db * C::DCOLS);
          const uint32_t a0 = tmem_base + kI8ACol0 + (uint32_t)(ab * C::ACOLS);
          const uint32_t b0 = smem_u32(smem + stage * C::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b < b_lo || b >= b_hi) continue;
            // block b: 128-byte slice b / 2 of the token rows, 64 bytes into it
            const uint64_t b_desc = make_sdesc_sw128(b0 + (uint32_t)((b >> 1) * N * 128));
            umma_i8_ts(d + b * N, a0 + b * 16, b_desc + (uint64_t)(((b & 1) * 64) >> 4), C::IDESC, 0u);
            umma_i8_ts(d + b * N, a0 + b * 16 + 8, b_desc + (uint64_t)(((b & 1) * 64 + 32) >> 4), C::IDESC, 1u);
          }
          umma_commit(&mma_bar[stage]);
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      // every MMA issued here completes before tensor memory is freed
      for (int64_t j = (i > STAGES ? i - STAGES : 0); j < i; ++j)
        mbar_wait(&mma_bar[j % STAGES], (uint32_t)((j / STAGES) & 1), nullptr, kWaitLimitNs / 8);
    }
  } else if (warp < kI8FirstScaler) {
    // ------------------------------------------------ expanders (one per lane quarter)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row of the A tile
    // codes of row r: ROW_BYTES bytes; its 16-byte chunk c (inputs 32c ..
    // 32c+31) sits at chunk c ^ (r % 8) (128-byte rows) or c ^ ((r / 2) % 4)
    // (64-byte rows), the TMA swizzle of the row width
    constexpr int CHUNKS = C::ROW_BYTES / 16;
    const uint32_t row_base = (uint32_t)r * C::ROW_BYTES;
    const uint32_t cx = CHUNKS == 8 ? (uint32_t)(r & 7) : (uint32_t)((r >> 1) & 3);
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    int64_t i = 0;
    RingPos<STAGES> sp, lag;  // lag: the stage ABUFS before this one
    RingPos<ABUFS> ap;
    bool ok = true;
    for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      I8Tile t;
      i8_decode_tile<EPI, BN>(p, s_off, s_base, s_tau, tile, t);
      for (int32_t kq = t.kq0; kq < t.kq1; ++kq, ++i, sp.next(), ap.next()) {
        const int stage = (int)sp.slot;
        // A buffer ap.slot is free once stage i - ABUFS's MMAs are done
        ok = mbar_wait(&full_bar[stage], sp.phase, &s_abort) &&
             (i < ABUFS || mbar_wait(&mma_bar[lag.slot], lag.phase, &s_abort));
        if (i >= ABUFS) lag.next();
        if (!ok) break;  // the issuer then stops at its own wait for this buffer
        tc_fence_after();
        const uint8_t* codes = smem + stage * C::STAGE_BYTES + C::B_BYTES + row_base;
        const uint32_t acol = lane_base + kI8ACol0 + ap.slot * (uint32_t)C::ACOLS;
#pragma unroll
        for (int half = 0; half < CHUNKS / 2; ++half) {
          // chunks 2 half, 2 half + 1: 64 inputs -> 16 columns
          uint32_t v[16];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t c = (uint32_t)(2 * half + cc);
            const uint4 w4 = *reinterpret_cast<const uint4*>(codes + ((c ^ cx) << 4));
            const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              v[8 * cc + 2 * k] = codes_lo_s8x16(words[k]);      // inputs 0 4 1 5 of the group
              v[8 * cc + 2 * k + 1] = codes_hi_s8x16(words[k]);  // inputs 2 6 3 7
            }
          }
          tmem_st_32x32b_x16(acol + (uint32_t)(half * 16), v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull_bar[ap.slot]);
      }
    }
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      s_abort = 1;
    }
  } else {
    // ------------------------------------------------ scalers (two per lane quarter)
    constexpr int TPW = BN / 2;               // tokens of this warp: t_half * TPW ..
    const int q = warp & 3;
    const int t_half = (warp - kI8FirstScaler) >> 2;
    const int r = q * 32 + lane;
    // scale of row r, block b: [W1 blocks x 64 rows | W3 blocks x 64 rows] or [blocks x 128 rows]
    const uint32_t s_row = C::B_BYTES + C::CODE_BYTES +
                           2 * ((EPI == I8_SWIGLU) ? ((r >> 6) * (NB * 64) + (r & 63)) : r);
    constexpr uint32_t s_blk = 2 * ((EPI == I8_SWIGLU) ? 64 : 128);
    // accumulator columns of block b: [BN high-byte sums | BN low-byte sums]
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(t_half * TPW);
    uint64_t acc[TPW / 2];                    // token pairs
#pragma unroll
    for (int j = 0; j < TPW / 2; ++j) acc[j] = 0ull;
    bool ok = true;
    RingPos<STAGES> sp;
    RingPos<DBUFS> dp;

    // The tile's outputs: a[t] * acc / 16, SiLU * mul or fp32 partials.
    auto epilogue = [&](const I8Tile& t) {
      float a[TPW];
#pragma unroll
      for (int j = 0; j < TPW / 2; ++j) unpack_f32x2(acc[j], a[2 * j], a[2 * j + 1]);
#pragma unroll
      for (int j = 0; j < TPW; ++j) {
        const int tk = t_half * TPW + j;
        a[j] = tk < t.m_valid ? p.act_scale[t.row0 + tk] * (a[j] * 0.0625f) : 0.f;
      }
      if (EPI == I8_SWIGLU) {
        // rows 0..63: W1 projection of column n0 + r; rows 64..127: W3 of column n0 + r - 64
        uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
        if (r >= 64) {
#pragma unroll
          for (int j = 0; j < TPW; ++j) xbuf[(t_half * TPW + j) * 64 + (r - 64)] = a[j];
        }
        named_bar_sync(1, kI8Scalers);
        if (r < 64 && t.n0 + r < p.n_out) {
#pragma unroll
          for (int j = 0; j < TPW; ++j) {
            const int tk = t_half * TPW + j;
            if (tk < t.m_valid && MOE_DCHECK(p.status, t.row0 + tk < p.S)) {
              const float hv = silu_f32(a[j]) * xbuf[tk * 64 + r];
              out[(int64_t)(t.row0 + tk) * p.out_ld + t.n0 + r] = (uint16_t)(pack_bf16x2(hv, 0.f) & 0xFFFFu);
            }
          }
        }
        named_bar_sync(1, kI8Scalers);
      } else {
        float* out = reinterpret_cast<float*>(p.out) + (int64_t)t.split * p.part_stride;
        if (t.n0 + r < p.n_out) {
#pragma unroll
          for (int j = 0; j < TPW; ++j) {
            const int tk = t_half * TPW + j;
            if (tk < t.m_valid && MOE_DCHECK(p.status, t.row0 + tk < p.S))
              out[(int64_t)(t.row0 + tk) * p.out_ld + t.n0 + r] = a[j];
          }
        }
      }
#pragma unroll
      for (int j = 0; j < TPW / 2; ++j) acc[j] = 0ull;
    };
    // acc += s * (256 hi + lo) over this warp's tokens
    auto add_block = [&](const uint32_t* hi, const uint32_t* lo, float s_b) {
      const uint64_t s2 = pack_f32x2(s_b, s_b);
#pragma unroll
      for (int j = 0; j < TPW / 2; ++j) {
        const int32_t v0 = (int32_t)hi[2 * j] * 256 + (int32_t)lo[2 * j];
        const int32_t v1 = (int32_t)hi[2 * j + 1] * 256 + (int32_t)lo[2 * j + 1];
        fma_f32x2(acc[j], pack_f32x2(__int2float_rn(v0), __int2float_rn(v1)), s2);
      }
    };

    // Every scaler runs the same stages and epilogues even after a wait gave
    // up (it then skips tensor-memory work), so their named barriers match;
    // waits return at once once s_abort is set.
    for (int32_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
      I8Tile t;
      i8_decode_tile<EPI, BN>(p, s_off, s_base, s_tau, tile, t);
      for (int32_t kq = t.kq0; kq < t.kq1; ++kq, sp.next(), dp.next()) {
        const int stage = (int)sp.slot;
        const int db = (int)dp.slot;
        ok = ok && mbar_wait(&mma_bar[stage], sp.phase, &s_abort);
        tc_fence_after();
        if (ok) {
          const uint8_t* st = smem + stage * C::STAGE_BYTES;
          float sc[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b)
            sc[b] = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(st + s_row + b * s_blk)) << 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(&free_bar[stage]);
          const uint32_t dcol = lane_base + (uint32_t)(db * C::DCOLS);
          // block b + 1's columns load while block b is scaled
          uint32_t hi[2][TPW], lo[2][TPW];
          tmem_ld_cols<TPW>(dcol, hi[0]);
          tmem_ld_cols<TPW>(dcol + BN, lo[0]);
          tmem_ld_wait_regs<TPW>(hi[0], lo[0]);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b + 1 < NB) {
              tmem_ld_cols<TPW>(dcol + (b + 1) * N, hi[(b + 1) & 1]);
              tmem_ld_cols<TPW>(dcol + (b + 1) * N + BN, lo[(b + 1) & 1]);
            } else {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&dfree_bar[db]);
            }
            add_block(hi[b & 1], lo[b & 1], sc[b]);
            if (b + 1 < NB) tmem_ld_wait_regs<TPW>(hi[(b + 1) & 1], lo[(b + 1) & 1]);
          }
        }
        if (kq + 1 == t.kq1) epilogue(t);
      }
    }
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      s_abort = 1;
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

// One block per row r < offsets[E] of `in` [S, K] bf16 (8 warps share the
// row): a = max |x[r]|, q = clamp(rint(x * 32639 / a), -32639, 32639), low
// byte ((q + 128) & 255) - 128, high byte (q - low) / 256, in the MMA's K
// order (0 4 1 5 2 6 3 7 per group of 8), written into the tiled token
// operand (layout at the top of this file; inputs from K up to the last
// stage's end are zero); scale[r] = a / 32639.
constexpr int kQuantThreads = 256;
__global__ void __launch_bounds__(kQuantThreads) quantize_act_kernel(const uint16_t* __restrict__ in,
                                                                     const int32_t* __restrict__ offsets, int32_t E,
                                                                     int32_t K, int32_t bn, int32_t ks, int32_t num_kq,
                                                                     uint8_t* __restrict__ q8,
                                                                     float* __restrict__ scale) {
  __shared__ float s_amax[kQuantThreads / 32];
  pdl_wait();  // the rows (and offsets) of the kernels before this one
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t rows = offsets[E];
  const int nvec = K >> 3;
  const int nvec_all = (num_kq * ks) >> 3;
  const int n_rows = 2 * bn;  // rows of a 128-byte slice: high bytes, then low bytes
  const int64_t tile_bytes = (int64_t)(ks / 128) * n_rows * 128;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    // token tile of the row: its expert's tiles follow those of the experts before it
    int e = 0;
    int64_t tau = 0;
    while (e + 1 < E && row >= offsets[e + 1]) {
      const int64_t m = offsets[e + 1] - offsets[e];
      tau += (m + bn - 1) / bn;
      ++e;
    }
    const int64_t local = row - offsets[e];
    tau += local / bn;
    const int tl = (int)(local % bn);
    uint8_t* tile = q8 + tau * num_kq * tile_bytes;

    const uint4* src = reinterpret_cast<const uint4*>(in + row * (int64_t)K);
    float amax = 0.f;
    for (int v = tid; v < nvec; v += kQuantThreads) {
      const uint4 x = src[v];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) s_amax[warp] = amax;
    __syncthreads();
    amax = s_amax[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, s_amax[w]);
    __syncthreads();  // s_amax is rewritten for the next row
    const float inv = amax > 0.f ? (float)kQMax / amax : 0.f;
    if (tid == 0) scale[row] = amax / (float)kQMax;
    for (int v = tid; v < nvec_all; v += kQuantThreads) {
      uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
      if (v < nvec) {
        const uint4 x = src[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        int qv[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          qv[2 * j] = max(-kQMax, min(kQMax, __float2int_rn(__uint_as_float(w[j] << 16) * inv)));
          qv[2 * j + 1] = max(-kQMax, min(kQMax, __float2int_rn(__uint_as_float(w[j] & 0xFFFF0000u) * inv)));
        }
        constexpr int kPerm[8] = {0, 4, 1, 5, 2, 6, 3, 7};
#pragma unroll
        for (int pos = 0; pos < 8; ++pos) {
          const int qq = qv[kPerm[pos]];
          const int lo = ((qq + 128) & 255) - 128;
          const int hi = (qq - lo) / 256;
          hw[pos >> 2] |= ((uint32_t)hi & 0xFFu) << (8 * (pos & 3));
          lw[pos >> 2] |= ((uint32_t)lo & 0xFFu) << (8 * (pos & 3));
        }
      }
      // input 8v: stage kq, 128-byte slice h, group g of 8 in the slice's row
      const int i0 = 8 * v;
      const int kq = i0 / ks, h = (i0 % ks) >> 7, g = (i0 & 127) >> 3;
      uint8_t* slice = tile + kq * tile_bytes + (int64_t)h * n_rows * 128;
      const int c = g >> 1, part = (g & 1) * 8;
      const int nh = tl, nl = bn + tl;
      *reinterpret_cast<uint2*>(slice + nh * 128 + ((c ^ (nh & 7)) << 4) + part) = make_uint2(hw[0], hw[1]);
      *reinterpret_cast<uint2*>(slice + nl * 128 + ((c ^ (nl & 7)) << 4) + part) = make_uint2(lw[0], lw[1]);
    }
  }
}

// codes [E, R, K/2] as a 3-D map, box {row_bytes, box_rows, 1}, swizzled to the row width
bool encode_codes_i8(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows, int row_bytes) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)R, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)(R * (K / 2))};
  cuuint32_t box[3] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// scales [E, K/64, R] as a 3-D bf16 map, box {box_rows, blocks, 1}
bool encode_scales_i8(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows, int blocks) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)R, (cuuint64_t)(K / 64), (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(R * 2), (cuuint64_t)((K / 64) * R * 2)};
  cuuint32_t box[3] = {(cuuint32_t)box_rows, (cuuint32_t)blocks, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_quantize_act(const uint16_t* in, const int32_t* offsets, int32_t E, int64_t S, int32_t K, int bn,
                                uint8_t* q8, float* scale, int num_sms, cudaStream_t s, bool pdl) {
  int64_t blocks = S;  // a block per row
  if (blocks > 8 * (int64_t)num_sms) blocks = 8 * (int64_t)num_sms;
  if (blocks < 1) blocks = 1;
  const int ks = i8_stage_inputs(bn);
  const int num_kq = (K + ks - 1) / ks;
  return launch_k(quantize_act_kernel, dim3((unsigned)blocks), dim3(kQuantThreads), 0, s, pdl, in, offsets, E, K, bn,
                  ks, num_kq, q8, scale);
}

template <int EPI, int BN>
cudaError_t launch_i8_one(const CUtensorMap& ca, const CUtensorMap& cb, const CUtensorMap& sa, const CUtensorMap& sb,
                          const I8Params& p, int num_sms, cudaStream_t s, bool pdl) {
  using C = I8Cfg<EPI, BN>;
  cudaError_t err =
      cudaFuncSetAttribute(expert_gemm_q4i8_kernel<EPI, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_k(expert_gemm_q4i8_kernel<EPI, BN>, dim3(num_sms), dim3(C::THREADS), C::SMEM_BYTES, s, pdl, ca, cb,
                  sa, sb, p);
}

template <int BN>
cudaError_t launch_i8(const ExpertGemmQ4Args& a, cudaStream_t s) {
  using C1 = I8Cfg<I8_SWIGLU, BN>;
  using C2 = I8Cfg<I8_PARTIAL, BN>;
  const int64_t S = a.S;
  CUtensorMap mc1, mc3, ms1, ms3, mc2, ms2;
  if (!encode_codes_i8(&mc1, a.W1c, a.E, a.f, a.d, 64, C1::ROW_BYTES) ||
      !encode_codes_i8(&mc3, a.W3c, a.E, a.f, a.d, 64, C1::ROW_BYTES) ||
      !encode_scales_i8(&ms1, a.W1s, a.E, a.f, a.d, 64, C1::NB) ||
      !encode_scales_i8(&ms3, a.W3s, a.E, a.f, a.d, 64, C1::NB) ||
      !encode_codes_i8(&mc2, a.W2c, a.E, a.d, a.f, 128, C2::ROW_BYTES) ||
      !encode_scales_i8(&ms2, a.W2s, a.E, a.d, a.f, 128, C2::NB))
    return cudaErrorInvalidValue;
  // x_perm -> tiled token operand (K = d)
  cudaError_t err =
      launch_quantize_act(a.x_perm, a.offsets, a.E, S, a.d, BN, a.act_q, a.act_scale, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  I8Params p1{};
  p1.offsets = a.offsets;
  p1.status = a.status;
  p1.out = a.h;
  p1.act = a.act_q;
  p1.act_scale = a.act_scale;
  p1.out_ld = a.f;
  p1.E = a.E;
  p1.num_kq = (a.d + C1::KS - 1) / C1::KS;
  p1.n_out = a.f;
  p1.n_blocks = a.f / 64;
  p1.splits = 1;
  p1.kq_per_split = p1.num_kq;
  p1.S = S;
  p1.clock_probe = a.clock_probe;
  err = launch_i8_one<I8_SWIGLU, BN>(mc1, mc3, ms1, ms3, p1, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  if (a.between && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;
  const bool pdl2 = a.pdl && !a.between;
  // h -> tiled token operand (K = f), reusing the buffer once the gate/up GEMM is done
  err = launch_quantize_act(a.h, a.offsets, a.E, S, a.f, BN, a.act_q, a.act_scale, a.num_sms, s, pdl2);
  if (err != cudaSuccess) return err;
  I8Params p2{};
  p2.offsets = a.offsets;
  p2.status = a.status;
  p2.out = a.partials;
  p2.act = a.act_q;
  p2.act_scale = a.act_scale;
  p2.out_ld = a.d;
  p2.part_stride = S * (int64_t)a.d;
  p2.E = a.E;
  p2.num_kq = (a.f + C2::KS - 1) / C2::KS;
  p2.n_out = a.d;
  p2.n_blocks = (a.d + 127) / 128;
  p2.kq_per_split = (p2.num_kq + a.splits - 1) / a.splits;
  p2.splits = (p2.num_kq + p2.kq_per_split - 1) / p2.kq_per_split;
  p2.S = S;
  p2.clock_probe = a.clock_probe ? a.clock_probe + 4 : nullptr;
  return launch_i8_one<I8_PARTIAL, BN>(mc2, mc2, ms2, ms2, p2, a.num_sms, s, pdl2);
}

}  // namespace

int32_t q4i8_stage_inputs(int32_t bn) { return i8_stage_inputs(bn); }

size_t q4i8_act_bytes(int64_t S, int32_t E, int32_t d, int32_t f, int32_t bn) {
  const int64_t ks = i8_stage_inputs(bn);
  const int64_t K = d > f ? d : f;
  const int64_t tiles = (S + bn - 1) / bn + E;  // at most one partial tile per expert
  return (size_t)(tiles * ((K + ks - 1) / ks) * (ks / 128) * 2 * bn * 128);
}

cudaError_t launch_expert_gemms_q4i8(const ExpertGemmQ4Args& a, cudaStream_t s) {
  return a.bn <= 16 ? launch_i8<16>(a, s) : launch_i8<32>(a, s);
}

}  // namespace moe
