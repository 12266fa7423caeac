// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores.
//
// Source: "Mixtral", sections "MoE Layer" (MixtralExpert.forward:
// w2(silu(w1 x) * w3 x), bias-free) and "SwiGLU Experts"
// (SwiGLU(x) = SiLU(x W1) (.) (x W3), output = SwiGLU(x) W2).
//
// For each expert e the rows offsets[e] .. offsets[e+1]-1 of the grouped
// activations are multiplied by that expert's weights:
//   GEMM1: h[r]      = SiLU(x_perm[r] . W1[e]^T) * (x_perm[r] . W3[e]^T)
//   GEMM2: y_perm[r] = h[r] . W2[e]^T
// Both use one persistent, warp-specialised kernel (one CTA per SM):
//   warp 0     one thread issues TMA tile loads into a STAGES-deep ring of
//              shared-memory buffers (128-byte swizzle, K-major);
//   warp 1     allocates tensor memory and one thread issues
//              tcgen05.mma (kind::f16, bf16 in, fp32 accumulate, M = 128,
//              N = BN, K = 16) into one of two TMEM accumulators;
//   warps 2-5  epilogue: tcgen05.ld the accumulator, apply SiLU * mul or a
//              plain conversion, store bf16 (or fp32 split-K partials).
// The accumulators are double-buffered so the epilogue of one tile overlaps
// the main loop of the next.  Tiles are enumerated per expert from the
// device-resident offsets (no host synchronisation) and distributed
// round-robin over the CTAs.
//
// Two schedules compute the same function:
//   TILED  (token-rich): A = 128 activation rows, B = weight rows.  GEMM1's
//          B tile stacks 128 rows of W1 over the same 128 rows of W3 (N = 256)
//          so accumulator columns c and c + 128 hold the two projections of
//          one output column; GEMM2's B tile is 256 rows of W2.
//   STREAM (token-poor, bound by reading the weights): A = weight rows,
//          B = the expert's (up to BN) tokens.  GEMM1's A tile stacks 64 rows
//          of W1 over the same 64 rows of W3 (accumulator lanes r and r + 64);
//          GEMM2's A tile is 128 rows of W2 and its K range is split so that
//          there are enough tiles to stream the weights on every SM; the
//          fp32 partials are summed by the combine (or a reduce kernel).
// Rows past an expert's end (next expert's rows, or zero fill past the
// buffer) are computed but never stored; weight rows past d_ff / d_model are
// zero-filled by the 3-D tensor maps.
#include <cstdint>
#include <cstdio>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

constexpr int BM = 128;  // MMA M: rows of the A operand
constexpr int BK = 64;   // K elements per stage: 128 bytes of bf16, one swizzle span
constexpr int kGemmThreads = 192;
constexpr int A_BYTES = BM * BK * 2;

// EPI_STREAM_GU_PARTIAL: the gate/up GEMM split along K (few tokens): fp32
// partials of both projections, [splits][S][2 f] (W1 columns, then W3),
// summed and passed through SiLU * mul by swiglu_splitk_kernel.
enum : int {
  EPI_TILED_SWIGLU = 0,
  EPI_TILED_STORE = 1,
  EPI_STREAM_SWIGLU = 2,
  EPI_STREAM_PARTIAL = 3,
  EPI_STREAM_GU_PARTIAL = 4
};
__host__ __device__ constexpr bool epi_is_gate_up(int epi) {
  return epi == EPI_STREAM_SWIGLU || epi == EPI_STREAM_GU_PARTIAL;
}

struct GemmParams {
  const int32_t* offsets;
  uint32_t* status;
  void* out;            // bf16 h / y_perm, or fp32 partials
  int64_t out_ld;       // elements between output rows
  int64_t part_stride;  // elements between split-K partial buffers
  int32_t E;
  int32_t num_kb;       // K / 64
  int32_t n_out;        // valid output columns (d_ff or d_model)
  int32_t n_blocks;     // weight blocks per expert
  int32_t splits;       // K splits (STREAM partial), else 1
  int32_t kb_per_split;
  uint32_t* tile_counter;  // CTA-pair kernels: next tile id (zero before the launch)
  int64_t S;               // rows of the activation and output buffers (T * k)
  uint64_t* clock_probe;   // profiled calls: CTA 0 writes {clock64, globaltimer} at entry and exit, else nullptr
  int32_t prefetch_kb;     // streaming kernels launched as dependents: K chunks of the
                           // first tile's weights to prefetch into L2 before waiting (0: none)
};

__host__ __device__ constexpr bool epi_is_tiled(int epi) { return epi <= EPI_TILED_STORE; }

template <int EPI, int BN>
struct GemmCfg {
  static constexpr bool kTiled = epi_is_tiled(EPI);
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = kTiled ? 4 : ((192 * 1024) / STAGE_BYTES > 10 ? 10 : (192 * 1024) / STAGE_BYTES);
  // TMEM columns: two accumulators of BN fp32 columns, power of two >= 32.
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr int XBUF_BYTES = (EPI == EPI_STREAM_SWIGLU) ? 64 * 16 * 4 : 0;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + XBUF_BYTES + BAR_BYTES;
  // rows of the weight operand per tile (n-extent of one weight block)
  static constexpr int W_ROWS = (EPI == EPI_TILED_SWIGLU) ? 128 : (EPI == EPI_TILED_STORE) ? 256 : epi_is_gate_up(EPI) ? 64 : 128;
  static constexpr uint32_t IDESC = make_idesc_bf16(BM, BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Tile {
  int32_t e, row0, m_valid, n0, split, kb0, kb1;
};

template <int EPI, int BN>
__device__ __forceinline__ bool decode_tile(const GemmParams& p, const int32_t* s_off,
                                            const int32_t* s_base, int32_t tile, Tile& t) {
  using C = GemmCfg<EPI, BN>;
  int e = 0;
  while (e < p.E && tile >= s_base[e + 1]) ++e;
  if (e >= p.E) return false;
  const int32_t local = tile - s_base[e];
  const int32_t M_e = s_off[e + 1] - s_off[e];
  t.e = e;
  if (C::kTiled) {
    const int32_t mb_count = (M_e + BM - 1) / BM;
    const int32_t nb = local / mb_count, mb = local % mb_count;
    t.row0 = s_off[e] + mb * BM;
    t.m_valid = min(BM, M_e - mb * BM);
    t.n0 = nb * C::W_ROWS;
    t.split = 0;
    t.kb0 = 0;
    t.kb1 = p.num_kb;
  } else {
    const int32_t tb_count = (M_e + BN - 1) / BN;
    const int32_t tb = local % tb_count;
    const int32_t rest = local / tb_count;
    t.split = rest % p.splits;
    const int32_t wb = rest / p.splits;
    t.row0 = s_off[e] + tb * BN;
    t.m_valid = min(BN, M_e - tb * BN);
    t.n0 = wb * C::W_ROWS;
    t.kb0 = t.split * p.kb_per_split;
    t.kb1 = min(p.num_kb, t.kb0 + p.kb_per_split);
  }
  return true;
}

template <int EPI, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap map_act,
                       const __grid_constant__ CUtensorMap map_wa,
                       const __grid_constant__ CUtensorMap map_wb, GemmParams p) {
  using C = GemmCfg<EPI, BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_epi_fail;
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_base[33];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  float* xbuf = reinterpret_cast<float*>(sB + STAGES * C::B_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * C::B_BYTES + C::XBUF_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe);

  if (tid == 0) {
    tma_prefetch_desc(&map_act);
    tma_prefetch_desc(&map_wa);
    if (EPI == EPI_TILED_SWIGLU || epi_is_gate_up(EPI)) tma_prefetch_desc(&map_wb);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (!C::kTiled && tid == 0 && p.prefetch_kb > 0) {
    // While the router and the grouping still run, start pulling into L2 the
    // weights of this CTA's first tile as it would be if every expert had one
    // block of tokens (the usual decode case).  A wrong guess costs only L2
    // traffic: nothing is written to shared memory and nothing waits.
    const int32_t per_e = p.n_blocks * p.splits;
    const int32_t e = (int32_t)blockIdx.x / per_e;
    if (e < p.E) {
      const int32_t rest = (int32_t)blockIdx.x % per_e;
      const int32_t kb0 = (rest % p.splits) * p.kb_per_split;
      const int32_t n0 = (rest / p.splits) * C::W_ROWS;
      const int32_t kb1 = min(p.num_kb, kb0 + min(p.kb_per_split, p.prefetch_kb));
      for (int32_t kb = kb0; kb < kb1; ++kb) {
        tma_prefetch_l2_3d(&map_wa, kb * BK, n0, e);
        if (epi_is_gate_up(EPI)) tma_prefetch_l2_3d(&map_wb, kb * BK, n0, e);
      }
    }
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
      int32_t n = 0;
      if (M_e > 0) {
        if (C::kTiled) n = ((M_e + BM - 1) / BM) * p.n_blocks;
        else n = ((M_e + BN - 1) / BN) * p.n_blocks * p.splits;
      }
      acc += n;
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
        Tile t;
        decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
        for (int32_t kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[stage], C::STAGE_BYTES);
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          const int32_t kx = kb * BK;
          if (EPI == EPI_TILED_SWIGLU) {
            tma_load_2d(&map_act, &full_bar[stage], a_dst, kx, t.row0);
            tma_load_3d(&map_wa, &full_bar[stage], b_dst, kx, t.n0, t.e);
            tma_load_3d(&map_wb, &full_bar[stage], b_dst + 128 * 128, kx, t.n0, t.e);
          } else if (EPI == EPI_TILED_STORE) {
            tma_load_2d(&map_act, &full_bar[stage], a_dst, kx, t.row0);
            tma_load_3d(&map_wa, &full_bar[stage], b_dst, kx, t.n0, t.e);
          } else if (epi_is_gate_up(EPI)) {
            tma_load_3d(&map_wa, &full_bar[stage], a_dst, kx, t.n0, t.e);
            tma_load_3d(&map_wb, &full_bar[stage], a_dst + 64 * 128, kx, t.n0, t.e);
            tma_load_2d(&map_act, &full_bar[stage], b_dst, kx, t.row0);
          } else {
            tma_load_3d(&map_wa, &full_bar[stage], a_dst, kx, t.n0, t.e);
            tma_load_2d(&map_act, &full_bar[stage], b_dst, kx, t.row0);
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
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t iter = 0;
      bool ok = true;
      for (int32_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++iter) {
        Tile t;
        decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
        const uint32_t acc = iter & 1, use = iter >> 1;
        if (!mbar_wait(&tempty_bar[acc], (use & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
        for (int32_t kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16(d_tmem, make_sdesc_sw128(a_addr + kk * 32), make_sdesc_sw128(b_addr + kk * 32),
                      C::IDESC, (kb > t.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      // Wait for every MMA this thread issued before tensor memory is freed.
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;      // accumulator lane (row of the MMA's M)
    uint32_t iter = 0;
    for (int32_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++iter) {
      Tile t;
      decode_tile<EPI, BN>(p, s_off, s_base, tile, t);
      const uint32_t acc = iter & 1, use = iter >> 1;
      // The four epilogue warps decide together whether to go on, so that a
      // wait that gives up in one warp never leaves the others at a barrier.
      if (!mbar_wait(&tfull_bar[acc], use & 1, &s_abort)) s_epi_fail = 1;
      named_bar_sync(2, 128);
      if (s_epi_fail) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_acc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;

      if (EPI == EPI_TILED_SWIGLU) {
        uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
        const bool row_ok = r < t.m_valid;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t va[32], vb[32];
          tmem_ld_32x32b_x32(t_acc + c0, va);
          tmem_ld_32x32b_x32(t_acc + 128 + c0, vb);
          tmem_ld_wait();
          if (row_ok && t.n0 + c0 < p.n_out && MOE_DCHECK(p.status, t.row0 + r < p.S)) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(va[2 * i])) * __uint_as_float(vb[2 * i]);
              const float h1 = silu_f32(__uint_as_float(va[2 * i + 1])) * __uint_as_float(vb[2 * i + 1]);
              packed[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(t.row0 + r) * p.out_ld + t.n0 + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      } else if (EPI == EPI_TILED_STORE) {
        uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
        const bool row_ok = r < t.m_valid;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_acc + c0, v);
          tmem_ld_wait();
          if (row_ok && t.n0 + c0 < p.n_out && MOE_DCHECK(p.status, t.row0 + r < p.S)) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(t.row0 + r) * p.out_ld + t.n0 + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      } else if (EPI == EPI_STREAM_SWIGLU) {
        // lanes 0..63: W1 projection of output column n0 + r; lanes 64..127:
        // W3 projection of column n0 + r - 64.  Columns of TMEM are tokens.
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
                out[(int64_t)(t.row0 + tok) * p.out_ld + t.n0 + r] =
                    (uint16_t)(pack_bf16x2(hv, 0.f) & 0xFFFFu);
              }
            }
          }
          named_bar_sync(1, 128);
        }
      } else {
        // fp32 split-K partial; TMEM columns are tokens.  Down projection:
        // lane r is output column n0 + r.  Gate/up: lanes 0..63 are W1
        // column n0 + r, lanes 64..127 W3 column n0 + r - 64, stored f later.
        float* out = reinterpret_cast<float*>(p.out) + (int64_t)t.split * p.part_stride +
                     (EPI == EPI_STREAM_GU_PARTIAL && r >= 64 ? (int64_t)p.n_out - 64 : 0);
        const bool col_ok = t.n0 + (EPI == EPI_STREAM_GU_PARTIAL ? (r & 63) : r) < p.n_out;
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
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA pairs
//
// The token-rich schedule on CTA pairs: a cluster of two CTAs on neighbouring
// SMs shares each tcgen05.mma (cta_group::2, M = 256 over the pair).  The
// weights are the M operand and the tokens the N operand, so the MMA's N can
// shrink to an expert's last, partial block of tokens (a multiple of 16)
// instead of computing a full tile of rows that belong to the next expert.
// A pair tile is 256 weight rows x up to 256 tokens:
//   GEMM1: CTA r holds W1 rows n0 + 64r .. +63 over the same W3 rows (its
//          accumulator lanes l and l + 64 are the two projections of output
//          column n0 + 64r + l), so SiLU * mul pairs lanes inside one CTA;
//   GEMM2: CTA r holds W2 rows n0 + 128r .. +127 (accumulator lane l is
//          output column n0 + 128r + l).
// The tokens are split between the CTAs: CTA r loads token rows
// row0 + r*N/2 .. and the accumulator column n of both CTAs is token row0 + n.
// Each CTA moves 32 KB per 64-element K chunk (16 KB of weights, 16 KB of
// tokens) for the MMA work of 48 KB on a single-CTA 128 x 256 tile; a stage
// holds two chunks (8 MMAs per full/empty handshake) and three stages fit.  The
// leader CTA (rank 0) counts both CTAs' bytes on its full barrier, issues the
// MMAs and commits to the barriers of both CTAs with one multicast commit;
// each CTA's epilogue reads its own accumulator and arrives on the leader's
// accumulator-empty barrier.
// Tiles are handed out dynamically: the leader's producer takes the next tile
// id from a global counter and publishes it to every role of both CTAs
// through a small ring in shared memory.  Tile ids run over (expert, weight
// block, token block), so the pairs working at the same time share each
// weight block through L2 and it is read from HBM once.
constexpr int kPairStagesMax = 6;
constexpr int kPairHalf = 128 * BK * 2;              // one 128-row operand half
constexpr int kPairStageBytes = 2 * kPairHalf;       // A half + B half per CTA
// Epilogue transpose buffers: two 16-token x 128-lane fp32 tiles, rows padded
// to 132 floats.
constexpr int kXsStride = 132;
constexpr int kPairXbuf = 2 * 16 * kXsStride * 4;
constexpr int kRing = 4;            // tile ids in flight
constexpr int kRingConsumers = 10;  // leader MMA + 4 epilogue warps per CTA + peer producer
constexpr int kPairBarBytes = (2 * kPairStagesMax + 5 + 2 * kRing) * 8;
// Stage ring: 192 KB per CTA, as 6 stages of one 64-element K chunk or 3 stages
// of two chunks (fewer full/empty handshakes per MMA).
constexpr int kPairRingBytes = 6 * kPairStageBytes;
constexpr int kPairSmem = 1024 + kPairRingBytes + kPairXbuf + kPairBarBytes;
static_assert(kPairSmem <= 227 * 1024, "shared memory");

struct PairTile {
  int32_t e, row0, m_valid, n_mma, n0;
};

template <int EPI>
__device__ __forceinline__ void decode_pair_tile(const GemmParams& p, const int32_t* s_off, const int32_t* s_base,
                                                 int32_t tile, PairTile& t) {
  int e = 0;
  while (e < p.E - 1 && tile >= s_base[e + 1]) ++e;
  const int32_t local = tile - s_base[e];
  const int32_t M_e = s_off[e + 1] - s_off[e];
  const int32_t tb_count = (M_e + 255) / 256;
  const int32_t tb = local % tb_count, wb = local / tb_count;
  t.e = e;
  t.row0 = s_off[e] + tb * 256;
  t.m_valid = min(256, M_e - tb * 256);
  t.n_mma = (t.m_valid + 15) & ~15;
  t.n0 = wb * (EPI == EPI_TILED_SWIGLU ? 128 : 256);
}

template <int EPI, int CHUNKS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_act, const __grid_constant__ CUtensorMap map_wa,
                            const __grid_constant__ CUtensorMap map_wb, GemmParams p) {
  constexpr int STAGES = kPairStagesMax / CHUNKS;
  constexpr int SHALF = CHUNKS * kPairHalf;  // bytes of one operand half per stage
  constexpr int ACC_COLS = 256;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_epi_fail;
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_base[33];
  __shared__ volatile int32_t s_ring[kRing];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * SHALF;
  float* xbuf = reinterpret_cast<float*>(sB + STAGES * SHALF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * SHALF + kPairXbuf);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint64_t* ring_full = bars + 2 * STAGES + 5;
  uint64_t* ring_empty = ring_full + kRing;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe);
  const uint32_t rank = cluster_ctarank();

  if (tid == 0) {
    tma_prefetch_desc(&map_act);
    tma_prefetch_desc(&map_wa);
    if (EPI == EPI_TILED_SWIGLU) tma_prefetch_desc(&map_wb);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);
    }
    mbar_init(drain_bar, 1);
    for (int q = 0; q < kRing; ++q) {
      mbar_init(&ring_full[q], 1);
      mbar_init(&ring_empty[q], kRingConsumers);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem, 512);
    tmem_relinquish_pair();
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
      acc += (M_e > 0) ? ((M_e + 255) / 256) * p.n_blocks : 0;
      s_base[e + 1] = acc;
    }
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const int32_t total = s_base[p.E];

  // Tile-id ring.  The leader's producer publishes; everyone else consumes
  // and releases the slot on the leader right after reading it.
  auto ring_get = [&](uint32_t n, int32_t& tile) -> bool {
    const uint32_t q = n % kRing, par = (n / kRing) & 1;
    if (!mbar_wait_cluster(&ring_full[q], par, &s_abort)) return false;
    tile = s_ring[q];
    mbar_arrive_cluster(map_to_rank(smem_u32(&ring_empty[q]), 0));
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        int32_t tile;
        if (rank == 0) {
          const uint32_t q = n % kRing, par = (n / kRing) & 1;
          if (!mbar_wait_cluster(&ring_empty[q], par ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          tile = (int32_t)atomicAdd(p.tile_counter, 1u);
          if (tile >= total) tile = -1;
          s_ring[q] = tile;
          st_cluster_u32(map_to_rank(smem_u32((const void*)&s_ring[q]), 1), (uint32_t)tile);
          mbar_arrive(&ring_full[q]);
          mbar_arrive_cluster(map_to_rank(smem_u32(&ring_full[q]), 1));
        } else if (!ring_get(n, tile)) {
          ok = false;
          break;
        }
        if (tile < 0) break;
        PairTile t;
        decode_pair_tile<EPI>(p, s_off, s_base, tile, t);
        const int32_t tok_row = t.row0 + (int32_t)rank * (t.n_mma >> 1);
        const int32_t n_steps = (p.num_kb + CHUNKS - 1) / CHUNKS;
        for (int32_t ks = 0; ks < n_steps; ++ks) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = map_to_rank(smem_u32(&full_bar[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * CHUNKS * kPairStageBytes);
#pragma unroll
          for (int c = 0; c < CHUNKS; ++c) {
            // a chunk past the end of K is zero-filled by the tensor maps
            uint8_t* a_dst = sA + stage * SHALF + c * kPairHalf;
            uint8_t* b_dst = sB + stage * SHALF + c * kPairHalf;
            const int32_t kx = (ks * CHUNKS + c) * BK;
            if (EPI == EPI_TILED_SWIGLU) {
              const int32_t wrow = t.n0 + (int32_t)rank * 64;
              tma_load_3d_pair(&map_wa, full_leader, a_dst, kx, wrow, t.e);
              tma_load_3d_pair(&map_wb, full_leader, a_dst + 64 * 128, kx, wrow, t.e);
            } else {
              tma_load_3d_pair(&map_wa, full_leader, a_dst, kx, t.n0 + (int32_t)rank * 128, t.e);
            }
            tma_load_2d_pair(&map_act, full_leader, b_dst, kx, tok_row);
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
      if (rank == 0) {
        // The leader's full barriers count both CTAs' bytes: wait for every
        // stage this pair filled before the pair may exit.
        for (int s = 0; s < STAGES; ++s) {
          if (s < issued) {
            const int64_t uses = (issued - s + STAGES - 1) / STAGES;
            mbar_wait_cluster(&full_bar[s], (uint32_t)((uses - 1) & 1), nullptr);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        int32_t tile;
        if (!ring_get(n, tile)) {
          ok = false;
          break;
        }
        if (tile < 0) break;
        PairTile t;
        decode_pair_tile<EPI>(p, s_off, s_base, tile, t);
        const uint32_t idesc = make_idesc_bf16(256, t.n_mma);
        const uint32_t acc = n & 1, use = n >> 1;
        if (!mbar_wait_cluster(&tempty_bar[acc], (use & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        const int32_t n_steps = (p.num_kb + CHUNKS - 1) / CHUNKS;
        for (int32_t ks = 0; ks < n_steps; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * SHALF);
          const uint32_t b_addr = smem_u32(sB + stage * SHALF);
#pragma unroll
          for (int c = 0; c < CHUNKS; ++c)
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16_pair(d_tmem, make_sdesc_sw128(a_addr + c * kPairHalf + kk * 32),
                             make_sdesc_sw128(b_addr + c * kPairHalf + kk * 32), idesc,
                             (ks > 0 || c > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair_both(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_both(&tfull_bar[acc]);
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
      }
      umma_commit_pair(map_to_rank(smem_u32(drain_bar), 0));
      mbar_wait_cluster(drain_bar, 0, nullptr);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator lane
    const int tid_epi = tid - 64;  // 0..127
    uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
    for (uint32_t n = 0;; ++n) {
      int32_t tile = -1;
      if (lane == 0 && !ring_get(n, tile)) s_epi_fail = 1;
      tile = __shfl_sync(0xffffffffu, tile, 0);
      const uint32_t acc = n & 1, use = n >> 1;
      // The four epilogue warps decide together whether to go on, so that a
      // wait that gives up in one warp never leaves the others at a barrier.
      if (tile >= 0 && !mbar_wait(&tfull_bar[acc], use & 1, &s_abort)) s_epi_fail = 1;
      named_bar_sync(2, 128);
      if (s_epi_fail) {
        record_status(p.status, kStatusTimeout);
        s_abort = 1;
        break;
      }
      if (tile < 0) break;
      PairTile t;
      decode_pair_tile<EPI>(p, s_off, s_base, tile, t);
      tc_fence_after();
      const uint32_t t_acc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
      // Per chunk of 16 tokens: every thread writes its lane's 16 values into
      // xs[token][lane], then thread i produces 8 consecutive outputs of token
      // i / 8 and stores them as one 16-byte vector.
      const int jt = tid_epi >> 3, g = tid_epi & 7;
#pragma unroll 1
      for (int c0 = 0, buf = 0; c0 < t.n_mma; c0 += 16, buf ^= 1) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(t_acc + c0, v);
        tmem_ld_wait();
        float* xs = xbuf + buf * 16 * kXsStride;
#pragma unroll
        for (int j = 0; j < 16; ++j) xs[j * kXsStride + r] = __uint_as_float(v[j]);
        named_bar_sync(1, 128);
        const int n = c0 + jt;
        const float* row = xs + jt * kXsStride;
        if (EPI == EPI_TILED_SWIGLU) {
          // lanes 0..63: W1 projection of columns n0 + 64*rank + lane;
          // lanes 64..127: the W3 projection of the same columns.
          const int32_t col = t.n0 + (int32_t)rank * 64 + 8 * g;
          if (n < t.m_valid && col < p.n_out && MOE_DCHECK(p.status, t.row0 + n < p.S)) {
            const float4 a0 = *reinterpret_cast<const float4*>(row + 8 * g);
            const float4 a1 = *reinterpret_cast<const float4*>(row + 8 * g + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(row + 64 + 8 * g);
            const float4 b1 = *reinterpret_cast<const float4*>(row + 64 + 8 * g + 4);
            uint4 o;
            o.x = pack_bf16x2(silu_f32(a0.x) * b0.x, silu_f32(a0.y) * b0.y);
            o.y = pack_bf16x2(silu_f32(a0.z) * b0.z, silu_f32(a0.w) * b0.w);
            o.z = pack_bf16x2(silu_f32(a1.x) * b1.x, silu_f32(a1.y) * b1.y);
            o.w = pack_bf16x2(silu_f32(a1.z) * b1.z, silu_f32(a1.w) * b1.w);
            *reinterpret_cast<uint4*>(out + (int64_t)(t.row0 + n) * p.out_ld + col) = o;
          }
        } else {
          // lane l: output column n0 + 128*rank + l; thread i writes 16 columns.
          const int32_t col = t.n0 + (int32_t)rank * 128 + 16 * g;
          if (n < t.m_valid && col < p.n_out && MOE_DCHECK(p.status, t.row0 + n < p.S)) {
            const float4 q0 = *reinterpret_cast<const float4*>(row + 16 * g);
            const float4 q1 = *reinterpret_cast<const float4*>(row + 16 * g + 4);
            const float4 q2 = *reinterpret_cast<const float4*>(row + 16 * g + 8);
            const float4 q3 = *reinterpret_cast<const float4*>(row + 16 * g + 12);
            uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(t.row0 + n) * p.out_ld + col);
            dst[0] = make_uint4(pack_bf16x2(q0.x, q0.y), pack_bf16x2(q0.z, q0.w), pack_bf16x2(q1.x, q1.y),
                                pack_bf16x2(q1.z, q1.w));
            dst[1] = make_uint4(pack_bf16x2(q2.x, q2.y), pack_bf16x2(q2.z, q2.w), pack_bf16x2(q3.x, q3.y),
                                pack_bf16x2(q3.z, q3.w));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty_bar[acc]), 0));
    }
  }

  tc_fence_before();
  cluster_sync();
  if (p.clock_probe && blockIdx.x == 0 && tid == 0) probe_clock(p.clock_probe + 2);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host side

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D bf16 map over a [rows, cols] row-major matrix, box {64, box_rows}.
static bool encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over [E, rows, cols] row-major, box {64, box_rows, 1}.
static bool encode_3d(CUtensorMap* m, const void* base, int64_t E, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)(rows * cols * 2)};
  cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int BN>
static cudaError_t launch_one(const CUtensorMap& act, const CUtensorMap& wa, const CUtensorMap& wb,
                              const GemmParams& p, int num_sms, cudaStream_t s, bool pdl) {
  using C = GemmCfg<EPI, BN>;
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_kernel<EPI, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_k(expert_gemm_kernel<EPI, BN>, dim3(num_sms), dim3(kGemmThreads), C::SMEM_BYTES, s, pdl, act, wa,
                  wb, p);
}

template <int EPI, int CHUNKS>
static cudaError_t launch_pair(const CUtensorMap& act, const CUtensorMap& wa, const CUtensorMap& wb,
                               const GemmParams& p, int num_sms, cudaStream_t s, bool pdl) {
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_pair_kernel<EPI, CHUNKS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kPairSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  // As many pairs as can be resident at once (persistent kernel).
  cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
  int clusters = 0;
  cudaLaunchConfig_t occ = cfg;
  occ.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&clusters, expert_gemm_pair_kernel<EPI, CHUNKS>, &occ) == cudaSuccess &&
      clusters > 0 &&
      2 * clusters < (int)cfg.gridDim.x)
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  return cudaLaunchKernelEx(&cfg, expert_gemm_pair_kernel<EPI, CHUNKS>, act, wa, wb, p);
}

// K chunks (16 KB of weights each) of its first tile that a streaming CTA
// prefetches into L2 while the kernels before it finish: about 64 MB over all
// CTAs, half of L2.
static int32_t prefetch_chunks(int num_sms) {
  const int64_t budget = 64ll << 20, chunk = 16 << 10;
  const int64_t n = budget / ((int64_t)(num_sms > 0 ? num_sms : 1) * chunk);
  return (int32_t)(n < 1 ? 1 : n);
}

void stream_params(int64_t T, int32_t k, int32_t d, int32_t f, int32_t E, int num_sms, int32_t* bn, int32_t* splits,
                   int32_t* splits1) {
  // token tile: twice the mean slots per expert, rounded up to 16 (an
  // expert's slots usually fit one tile; smaller tiles mean smaller stages,
  // more of them in flight, and a shorter epilogue)
  int64_t b = ((2 * ((T * k + E - 1) / E) + 15) / 16) * 16;
  if (b < 16) b = 16;
  if (b > 128) b = 128;
  if (b > 64) b = 128;
  else if (b > 32) b = 64;
  else if (b > 16) b = 32;
  *bn = (int32_t)b;
  // Split K of the down projection: the count that minimises the waves of
  // (experts x 128-row blocks x splits) tiles times the K chunks of a tile
  // plus one (a tile's start-up and epilogue), plus one chunk per split for
  // the partial plane the combine reads.  At most T * k experts receive
  // tokens, which bounds the tile count for few tokens.
  const int32_t num_kb = f / BK;
  const int64_t touched = T * k < E ? T * k : E;
  const int64_t base = touched * ((d + 127) / 128);
  int32_t best = 1;
  int64_t best_cost = INT64_MAX;
  for (int32_t sp = 1; sp <= 16 && sp <= num_kb; ++sp) {
    const int32_t kbps = (num_kb + sp - 1) / sp;
    const int32_t real = (num_kb + kbps - 1) / kbps;
    const int64_t waves = (base * real + num_sms - 1) / num_sms;
    const int64_t cost = waves * (kbps + 1) + real;
    if (cost < best_cost) {
      best_cost = cost;
      best = real;
    }
  }
  *splits = best;
  // Split K of the gate/up projection (2 ways) only where it shortens the
  // last, partly filled wave of (experts x 64-row blocks) tiles enough (by
  // 3 %) to pay for its fp32 partials and the extra reduction launch
  // (counted as 8 chunk-waves).  4 ways was measured 1 % slower than 2 at
  // one and two Mixtral tokens, where the model preferred it.
  const int32_t num_kb1 = d / BK;
  const int64_t base1 = touched * (f / 64);
  const int64_t plane = (T * k * 2 * (int64_t)f * 8 + 16384LL * num_sms - 1) / (16384LL * num_sms);
  const int64_t cost1 = ((base1 + num_sms - 1) / num_sms) * (num_kb1 + 1);
  int32_t best1 = 1;
  int64_t best1_cost = cost1;
  for (int32_t sp = 2; sp <= 2 && sp <= num_kb1; sp *= 2) {
    const int32_t kbps = (num_kb1 + sp - 1) / sp;
    const int32_t real = (num_kb1 + kbps - 1) / kbps;
    const int64_t waves = (base1 * real + num_sms - 1) / num_sms;
    const int64_t c = waves * (kbps + 1) + real * plane + 8;
    if (c * 100 <= cost1 * 97 && c < best1_cost) {
      best1_cost = c;
      best1 = real;
    }
  }
  *splits1 = best1;
}

// h[r, c] = bf16(SiLU(a) * b), a and b the sums over splits (in split order)
// of the gate/up partials of row r < offsets[E]: columns c and f + c.
__global__ void __launch_bounds__(256) swiglu_splitk_kernel(const float* __restrict__ partials, int32_t splits,
                                                            int64_t part_stride, const int32_t* __restrict__ offsets,
                                                            int32_t E, int32_t f, uint16_t* __restrict__ h, int64_t S,
                                                            uint32_t* status) {
  pdl_wait();  // the gate/up partials
  pdl_trigger();
  int64_t rows = offsets[E];
  if (!MOE_DCHECK(status, rows >= 0 && rows <= S)) rows = 0;
  const int nvec = f >> 2;
  const int64_t total = rows * nvec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nvec;
    const int v = (int)(i % nvec);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int sp = 0; sp < splits; ++sp) {
      const float* row = partials + sp * part_stride + r * 2 * (int64_t)f;
      const float4 pa = reinterpret_cast<const float4*>(row)[v];
      const float4 pb = reinterpret_cast<const float4*>(row + f)[v];
      a.x += pa.x; a.y += pa.y; a.z += pa.z; a.w += pa.w;
      b.x += pb.x; b.y += pb.y; b.z += pb.z; b.w += pb.w;
    }
    reinterpret_cast<uint2*>(h + r * (int64_t)f)[v] =
        make_uint2(pack_bf16x2(silu_f32(a.x) * b.x, silu_f32(a.y) * b.y),
                   pack_bf16x2(silu_f32(a.z) * b.z, silu_f32(a.w) * b.w));
  }
}



template <int BN>
static cudaError_t launch_stream(const ExpertGemmArgs& a, cudaStream_t s) {
  CUtensorMap mx, mw1, mw3, mh, mw2;
  if (!encode_2d(&mx, a.x_perm, a.S, a.d, BN) || !encode_3d(&mw1, a.W1, a.E, a.f, a.d, 64) ||
      !encode_3d(&mw3, a.W3, a.E, a.f, a.d, 64) || !encode_2d(&mh, a.h, a.S, a.f, BN) ||
      !encode_3d(&mw2, a.W2, a.E, a.d, a.f, 128))
    return cudaErrorInvalidValue;
  GemmParams p1{};
  p1.offsets = a.offsets;
  p1.status = a.status;
  p1.S = a.S;
  p1.out = a.h;
  p1.out_ld = a.f;
  p1.part_stride = 0;
  p1.E = a.E;
  p1.num_kb = a.d / BK;
  p1.n_out = a.f;
  p1.n_blocks = a.f / 64;
  p1.splits = 1;
  p1.kb_per_split = p1.num_kb;
  p1.prefetch_kb = a.pdl ? prefetch_chunks(a.num_sms) : 0;
  p1.clock_probe = a.clock_probe;
  cudaError_t err;
  if (a.splits1 > 1) {
    // gate/up split along K: fp32 partials, then their sum through SiLU * mul
    p1.out = a.partials1;
    p1.out_ld = 2 * (int64_t)a.f;
    p1.part_stride = a.S * 2 * (int64_t)a.f;
    p1.kb_per_split = (p1.num_kb + a.splits1 - 1) / a.splits1;
    p1.splits = (p1.num_kb + p1.kb_per_split - 1) / p1.kb_per_split;
    err = launch_one<EPI_STREAM_GU_PARTIAL, BN>(mx, mw1, mw3, p1, a.num_sms, s, a.pdl);
    if (err != cudaSuccess) return err;
    int64_t blocks = (a.S * (a.f / 4) + 255) / 256;
    if (blocks > 4 * (int64_t)a.num_sms) blocks = 4 * (int64_t)a.num_sms;
    if (blocks < 1) blocks = 1;
    err = launch_k(swiglu_splitk_kernel, dim3((unsigned)blocks), dim3(256), 0, s, a.pdl, (const float*)a.partials1,
                   p1.splits, p1.part_stride, a.offsets, a.E, a.f, a.h, a.S, a.status);
  } else {
    err = launch_one<EPI_STREAM_SWIGLU, BN>(mx, mw1, mw3, p1, a.num_sms, s, a.pdl);
  }
  if (err != cudaSuccess) return err;
  if (a.between && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;
  GemmParams p2{};
  p2.offsets = a.offsets;
  p2.status = a.status;
  p2.S = a.S;
  p2.out = a.partials;
  p2.out_ld = a.d;
  p2.part_stride = a.S * (int64_t)a.d;
  p2.E = a.E;
  p2.num_kb = a.f / BK;
  p2.n_out = a.d;
  p2.n_blocks = (a.d + 127) / 128;
  p2.kb_per_split = (p2.num_kb + a.splits - 1) / a.splits;
  p2.splits = (p2.num_kb + p2.kb_per_split - 1) / p2.kb_per_split;
  const bool pdl2 = a.pdl && !a.between;
  p2.prefetch_kb = pdl2 ? prefetch_chunks(a.num_sms) : 0;
  p2.clock_probe = a.clock_probe ? a.clock_probe + 4 : nullptr;
  return launch_one<EPI_STREAM_PARTIAL, BN>(mh, mw2, mw2, p2, a.num_sms, s, pdl2);
}

static cudaError_t launch_tiled(const ExpertGemmArgs& a, cudaStream_t s) {
  CUtensorMap mx, mw1, mw3, mh, mw2;
  const int wbox = a.pair ? 64 : 128;
  if (!encode_2d(&mx, a.x_perm, a.S, a.d, 128) || !encode_3d(&mw1, a.W1, a.E, a.f, a.d, wbox) ||
      !encode_3d(&mw3, a.W3, a.E, a.f, a.d, wbox) || !encode_2d(&mh, a.h, a.S, a.f, 128) ||
      !encode_3d(&mw2, a.W2, a.E, a.d, a.f, a.pair ? 128 : 256))
    return cudaErrorInvalidValue;
  GemmParams p1{};
  p1.offsets = a.offsets;
  p1.status = a.status;
  p1.S = a.S;
  p1.out = a.h;
  p1.out_ld = a.f;
  p1.E = a.E;
  p1.num_kb = a.d / BK;
  p1.n_out = a.f;
  p1.n_blocks = (a.f + 127) / 128;
  p1.splits = 1;
  p1.kb_per_split = p1.num_kb;
  p1.tile_counter = a.tile_counters;
  p1.clock_probe = a.clock_probe;
  // two 64-element K chunks per pipeline stage (3 stages): half the handshakes
  cudaError_t err = a.pair ? launch_pair<EPI_TILED_SWIGLU, 2>(mx, mw1, mw3, p1, a.num_sms, s, a.pdl)
                           : launch_one<EPI_TILED_SWIGLU, 256>(mx, mw1, mw3, p1, a.num_sms, s, a.pdl);
  if (err != cudaSuccess) return err;
  if (a.between && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;
  GemmParams p2{};
  p2.offsets = a.offsets;
  p2.status = a.status;
  p2.S = a.S;
  p2.out = a.y_perm;
  p2.out_ld = a.d;
  p2.E = a.E;
  p2.num_kb = a.f / BK;
  p2.n_out = a.d;
  p2.n_blocks = (a.d + 255) / 256;
  p2.splits = 1;
  p2.kb_per_split = p2.num_kb;
  p2.tile_counter = a.tile_counters + 1;
  p2.clock_probe = a.clock_probe ? a.clock_probe + 4 : nullptr;
  const bool pdl2 = a.pdl && !a.between;
  return a.pair ? launch_pair<EPI_TILED_STORE, 2>(mh, mw2, mw2, p2, a.num_sms, s, pdl2)
                : launch_one<EPI_TILED_STORE, 256>(mh, mw2, mw2, p2, a.num_sms, s, pdl2);
}

cudaError_t launch_expert_gemms(const ExpertGemmArgs& a, cudaStream_t s) {
  if (a.variant == 1) return launch_tiled(a, s);
  switch (a.stream_bn) {
    case 16: return launch_stream<16>(a, s);
    case 32: return launch_stream<32>(a, s);
    case 64: return launch_stream<64>(a, s);
    default: return launch_stream<128>(a, s);
  }
}

}  // namespace moe
