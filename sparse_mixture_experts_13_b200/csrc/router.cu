// Router and top-k gate.
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (G(x) = Softmax(TopK(x . W_g)), logits outside the top-k at -inf), and
// "Mixtral", section "MoE Layer" (bias-free nn.Linear router, topk of the
// logits, softmax over the k kept logits).
//
// Logits are fp32 dot products of a token's bf16 row with the E rows of W_g.
// Two kernels compute them:
//
// router_reg_kernel (E <= 8, d <= 4096, the Mixtral shape): a persistent
//   block of d/8 threads holds all of W_g in registers, thread i owning inputs
//   [8i, 8i+8) of every expert row, so W_g is read once per block instead of
//   once per token.  Token rows stream through a ring of shared-memory slots
//   filled by bulk copies (one copy per group of TB consecutive rows), so many
//   rows are in flight per SM without costing registers.  Each thread forms
//   its 8 partial logits of a token, a warp reduce-scatter leaves one expert's
//   warp sum on every fourth lane, and the warp sums are added across warps in
//   shared memory in warp order.
// router_group_kernel (any other shape): a block takes a group of tokens and
//   splits d over its warps; every W_g vector a warp reads (from L2) serves
//   all tokens of the group.
//
// In both, the top-k (ties to the smaller expert index), the k-way softmax
// and the full-softmax probability of each chosen expert are computed
// redundantly per lane of one warp and lanes 0..k-1 write one slot each.  The
// per-expert histogram is aggregated in shared memory and added to global
// memory once per block.
#include <cfloat>
#include <cstdint>


#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Lane e < E holds the logit l of expert e for token t (other lanes: any
// value).  Every lane ranks its expert in the order (logit descending, index
// ascending), so the experts of rank < k are the top-k, rank 0 first, and
// ranks k .. 2k-1 are the next-best candidates.  With m the largest logit,
// the gate of a chosen expert is exp(l - m) over the sum of exp(l' - m) of the
// k chosen ones, and its full-softmax probability is exp(l - m) over the sum
// across all E experts.  The sums are butterflies over the first EMAX lanes
// (a fixed order).  Lane e writes the slot of its rank and counts it in *hist.
template <int EMAX>
__device__ __forceinline__ void finish_token(const RouterArgs& a, int64_t t, float l, int lane, int* hist) {
  const int E = a.E, k = a.k;
  const bool valid = lane < E;
  int rank = 0;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    const float le = __shfl_sync(0xffffffffu, l, e);
    if (e < E && (le > l || (le == l && e < lane))) ++rank;
  }
  float m = valid ? l : -FLT_MAX;
#pragma unroll
  for (int off = EMAX / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float ex = valid ? expf(l - m) : 0.f;
  float zE = ex, zk = (valid && rank < k) ? ex : 0.f;
#pragma unroll
  for (int off = EMAX / 2; off > 0; off >>= 1) {
    zE += __shfl_xor_sync(0xffffffffu, zE, off);
    zk += __shfl_xor_sync(0xffffffffu, zk, off);
  }
  if (valid && rank < k) {
    a.topk_idx[t * k + rank] = lane;
    a.topk_w[t * k + rank] = ex / zk;
    a.topk_p[t * k + rank] = ex / zE;
    atomicAdd(&hist[lane], 1);
  }
  if (a.logits && valid) a.logits[t * E + lane] = l;
  if (a.next_idx) {
    // ranks k .. 2k-1 (capacity fallback); ranks past E - 1 do not exist
    if (valid && rank >= k && rank < 2 * k) {
      a.next_idx[t * k + rank - k] = lane;
      a.next_p[t * k + rank - k] = ex / zE;
    }
    if (lane < k && k + lane >= E) {
      a.next_idx[t * k + lane] = -1;
      a.next_p[t * k + lane] = 0.f;
    }
  }
}

__device__ __forceinline__ float dot8(const float (&x)[8], const float4& w0, const float4& w1, float s) {
  s = fmaf(x[0], w0.x, s);
  s = fmaf(x[1], w0.y, s);
  s = fmaf(x[2], w0.z, s);
  s = fmaf(x[3], w0.w, s);
  s = fmaf(x[4], w1.x, s);
  s = fmaf(x[5], w1.y, s);
  s = fmaf(x[6], w1.z, s);
  s = fmaf(x[7], w1.w, s);
  return s;
}

// One block of 16 warps per group of G tokens.  Warp w takes the d-slice
// [w*d/16, (w+1)*d/16); each lane loads one 16-byte vector of that slice for
// every token of the group at once, then reads the matching vectors of the E
// rows of W_g (from L2) and applies each to the G tokens held in registers.
// The 16 partial sums per (token, expert) are added in shared memory in warp
// order; warp g then finishes token g.
constexpr int kGroupThreads = 512;
constexpr int kGroupWarps = kGroupThreads / 32;

template <int EMAX, int G>
__global__ void __launch_bounds__(kGroupThreads) router_group_kernel(RouterArgs a) {
  __shared__ float s_part[kGroupWarps][G][EMAX];
  __shared__ int s_count[32];
  pdl_trigger();  // the grouping kernel may launch now; it waits for this grid
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, d = a.d;
  const int64_t t0 = (int64_t)blockIdx.x * G;
  if (tid < 32) s_count[tid] = 0;
  const int nvec = d >> 3;  // 16-byte vectors per row
  const int per_warp = (nvec + kGroupWarps - 1) / kGroupWarps;
  const int v0 = warp * per_warp, v1 = min(nvec, v0 + per_warp);
  float acc[G][EMAX];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[g][e] = 0.f;
  for (int v = v0 + lane; v < v1; v += 32) {
    uint4 xr[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
      xr[g] = (t0 + g < a.T) ? __ldg(reinterpret_cast<const uint4*>(a.x + (t0 + g) * d) + v) : make_uint4(0, 0, 0, 0);
    float xf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) bf16x8_to_f32(xr[g], xf[g]);
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        const float4* w = reinterpret_cast<const float4*>(a.Wg + (int64_t)e * d + (int64_t)v * 8);
        const float4 w0 = __ldg(w), w1 = __ldg(w + 1);
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g][e] = dot8(xf[g], w0, w1, acc[g][e]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], off);
    }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EMAX; ++e) s_part[warp][g][e] = acc[g][e];
  }
  __syncthreads();
  if (warp < G && t0 + warp < a.T) {
    float v = 0.f;
    if (lane < EMAX) {
#pragma unroll
      for (int w = 0; w < kGroupWarps; ++w) v += s_part[w][warp][lane];
    }
    finish_token<EMAX>(a, t0 + warp, v, lane, s_count);
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

// ---------------------------------------------------------------- W_g in registers
constexpr int kRegMaxThreads = 512;  // d <= 8 * 512
constexpr int kRegSlots = 4;         // ring depth, in groups of TB token rows
constexpr int kRegMaxWarps = kRegMaxThreads / 32;

// a[V] (V a power of two, 8 <= V <= 32) of every lane -> the warp's sum of
// value lane >> log2(32 / V), exact on every lane.  Halving exchanges with
// masks 16, 8, ... (log2 V of them) hand the partner the half of the values
// this lane gives up; each step's V / 2^s exchanges are independent, so the
// steps pipeline.  Masks left below the last halving step are plain sums.
template <int V>
__device__ __forceinline__ float warp_transpose_reduce(float (&a)[V], int lane) {
  int m = 16;
#pragma unroll
  for (int n = V / 2; n >= 1; n /= 2, m /= 2) {
    const bool up = lane & m;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = up ? a[j] : a[j + n];
      const float keep = up ? a[j + n] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  float v = a[0];
#pragma unroll
  for (; m >= 1; m /= 2) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// Dynamic shared memory of router_reg_kernel<TB> for rows of d bf16.
__host__ __device__ constexpr size_t reg_ring_bytes(int TB, int d) { return (size_t)kRegSlots * TB * d * 2; }
__host__ __device__ constexpr size_t reg_smem_bytes(int TB, int d) {
  return reg_ring_bytes(TB, d) + sizeof(float) * 2 * TB * kRegMaxWarps * 8 + sizeof(uint64_t) * kRegSlots +
         sizeof(int) * 32;
}

// Block b takes token groups b, b + gridDim.x, ... (TB consecutive tokens
// each).  Thread 0 keeps up to kRegSlots groups in flight; a slot is refilled
// right after the block barrier that follows its last read.
template <int TB>
__global__ void __launch_bounds__(kRegMaxThreads, 1) router_reg_kernel(RouterArgs a, int64_t ngroups) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_trigger();  // the grouping kernel may launch now; it waits for this grid
  const int d = a.d, E = a.E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const size_t row_bytes = (size_t)d * 2;
  uint8_t* ring = smem;
  float* s_part = reinterpret_cast<float*>(smem + reg_ring_bytes(TB, d));  // [2][TB][kRegMaxWarps][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_part + 2 * TB * kRegMaxWarps * 8);
  int* s_count = reinterpret_cast<int*>(bars + kRegSlots);

  const int64_t g0 = blockIdx.x, gstride = gridDim.x;
  const int64_t my_groups = g0 < ngroups ? (ngroups - 1 - g0) / gstride + 1 : 0;
  if (tid < 32) s_count[tid] = 0;
  if (tid == 0) {
    for (int i = 0; i < kRegSlots; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int64_t i) {  // this block's i-th group into slot i % kRegSlots
    const int64_t t0 = (g0 + i * gstride) * TB;
    const int64_t nt = a.T - t0 < TB ? a.T - t0 : TB;
    const uint32_t bytes = (uint32_t)(nt * (int64_t)row_bytes);
    uint64_t* bar = &bars[i % kRegSlots];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(ring + (size_t)(i % kRegSlots) * TB * row_bytes, a.x + t0 * d, bytes, bar);
  };
  if (tid == 0)
    for (int64_t i = 0; i < my_groups && i < kRegSlots; ++i) issue(i);

  // inputs [8 tid, 8 tid + 8) of every expert row as pairs (2i, 2i+1); zero
  // past E and past d
  const bool active = tid < (d >> 3);
  uint64_t w2[8][4];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
    if (active && e < E) {
      const float4* src = reinterpret_cast<const float4*>(a.Wg + (int64_t)e * d + tid * 8);
      w0 = __ldg(src);
      w1 = __ldg(src + 1);
    }
    w2[e][0] = pack_f32x2(w0.x, w0.y);
    w2[e][1] = pack_f32x2(w0.z, w0.w);
    w2[e][2] = pack_f32x2(w1.x, w1.y);
    w2[e][3] = pack_f32x2(w1.z, w1.w);
  }

  bool ok = true;
  for (int64_t i = 0; i < my_groups; ++i) {
    const int slot = (int)(i % kRegSlots);
    const int64_t t0 = (g0 + i * gstride) * TB;
    const int nt = (int)(a.T - t0 < TB ? a.T - t0 : TB);
    if (ok) ok = mbar_wait(&bars[slot], (uint32_t)((i / kRegSlots) & 1), nullptr);
    float* part = s_part + (i & 1) * TB * kRegMaxWarps * 8;
    const uint8_t* rows = ring + (size_t)slot * TB * row_bytes;
    // this thread's partial logits of the group's tokens: value tb * 8 + e
    float acc[8 * TB];
#pragma unroll
    for (int j = 0; j < 8 * TB; ++j) acc[j] = 0.f;
    if (active) {
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        if (tb < nt) {
          // even and odd inputs accumulate in the two halves of a packed pair
          const uint4 v = *reinterpret_cast<const uint4*>(rows + tb * row_bytes + tid * 16);
          const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
          uint64_t acc2[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc2[e] = 0ull;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint64_t x2 = pack_f32x2(__uint_as_float(xw[i] << 16), __uint_as_float(xw[i] & 0xFFFF0000u));
#pragma unroll
            for (int e = 0; e < 8; ++e) fma_f32x2(acc2[e], x2, w2[e][i]);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float lo, hi;
            unpack_f32x2(acc2[e], lo, hi);
            acc[tb * 8 + e] = lo + hi;
          }
        }
      }
    }
    // the warp's sums of all TB x 8 values at once; value j on lanes j << shift
    {
      constexpr int kShift = TB == 4 ? 0 : (TB == 2 ? 1 : 2);
      const float r = warp_transpose_reduce<8 * TB>(acc, lane);
      const int j = lane >> kShift, tb = j >> 3;
      if ((lane & ((1 << kShift) - 1)) == 0 && tb < nt) part[(tb * kRegMaxWarps + warp) * 8 + (j & 7)] = r;
    }
    if (!__syncthreads_and(ok)) {
      // a row copy never arrived: report, let the copies still in flight land, leave
      if (tid == 0) {
        record_status(a.status, kStatusTimeout);
        for (int64_t j = i; j < my_groups && j < i + kRegSlots; ++j)
          mbar_wait(&bars[j % kRegSlots], (uint32_t)((j / kRegSlots) & 1), nullptr, kWaitLimitNs / 8);
      }
      return;
    }
    if (tid == 0 && i + kRegSlots < my_groups) issue(i + kRegSlots);
    // warp sums -> logits, in warp order: lane (q, e) adds warps q, q+4, q+8, q+12
    for (int tb = warp; tb < nt; tb += nwarps) {
      const int e = lane & 7, q = lane >> 3;
      float v = 0.f;
#pragma unroll
      for (int ww = 0; ww < kRegMaxWarps; ww += 4)
        if (q + ww < nwarps) v += part[(tb * kRegMaxWarps + q + ww) * 8 + e];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      finish_token<8>(a, t0 + tb, v, lane, s_count);  // lane e < 8 holds logit e
    }
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

template <int TB>
static cudaError_t launch_router_reg(const RouterArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = reg_smem_bytes(TB, a.d);
  cudaError_t err = cudaFuncSetAttribute(router_reg_kernel<TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (a.T + TB - 1) / TB;
  const int64_t grid = ngroups < num_sms ? ngroups : num_sms;
  const int threads = ((a.d / 8 + 31) / 32) * 32;
  router_reg_kernel<TB><<<(unsigned)grid, threads, smem, s>>>(a, ngroups);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- tensor-core router
// router_mma_kernel (E <= 8, d a multiple of 256 up to 4096): the logits of a
// tile of 8 tokens by mma.sync m16n8k16 (bf16 operands, fp32 accumulation).
// x is exact in bf16, and every fp32 weight is split exactly into three bf16
// terms, w = hi + mid + lo (8 + 8 + 8 significant bits, by truncation), so the three
// MMAs per 16 inputs multiply exactly by the fp32 weights and the products
// add up in fp32.  Each of the 16 warps owns d/16 inputs and keeps its slice
// of the three weight terms as MMA B fragments for the whole launch (hi and
// mid in registers, lo in shared memory); the token rows arrive by bulk
// copies, one per row, into a ring of two tiles with rows 16 bytes further
// apart than their length, and are read by ldmatrix.  The MMA's rows 8..15
// repeat rows 0..7 (ignored).  Per tile each warp leaves its 8 x 8
// partial logits in shared memory; the partials are added in warp order and
// warp t finishes token t.
constexpr int kMmaTile = 8;     // tokens per tile
constexpr int kMmaWarps = 16;
constexpr int kMmaSlots = 2;
constexpr int kMmaMaxSteps = 16;  // 16-input steps per warp (d <= 4096)
constexpr int64_t kMmaMinTokens = 1024;

// w -> (hi, mid, lo) bf16 bits with hi + mid + lo == w exactly: hi keeps the
// top 8 significant bits of w (truncation), mid the next 8 of the remainder,
// lo the rest (at most 8 bits, so bf16 holds it); both subtractions are exact
__device__ __forceinline__ void split3(float w, uint32_t& h, uint32_t& m, uint32_t& l) {
  const uint32_t wb = __float_as_uint(w);
  h = wb >> 16;
  const float r1 = w - __uint_as_float(wb & 0xFFFF0000u);
  const uint32_t rb = __float_as_uint(r1);
  m = rb >> 16;
  const float r2 = r1 - __uint_as_float(rb & 0xFFFF0000u);
  l = __float_as_uint(r2) >> 16;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// a tile's rows in shared memory, 16 bytes more apart than a row, so the 8
// rows that one ldmatrix reads fall in distinct bank groups
__host__ __device__ constexpr size_t mma_row_pitch(int d) { return (size_t)d * 2 + 16; }
__host__ __device__ constexpr size_t mma_slot_bytes(int d) { return (((size_t)kMmaTile * mma_row_pitch(d)) + 127) / 128 * 128; }
// lo fragments: [warp][step][lane] uint2
__host__ __device__ constexpr size_t mma_lo_bytes(int d) { return (size_t)kMmaWarps * (d / (16 * kMmaWarps)) * 32 * 8; }
__host__ __device__ constexpr size_t mma_smem_bytes(int d) {
  return 1024 + kMmaSlots * mma_slot_bytes(d) + mma_lo_bytes(d) + sizeof(float) * 2 * kMmaWarps * kMmaTile * 8 +
         sizeof(uint64_t) * kMmaSlots + sizeof(int) * 32;
}

__global__ void __launch_bounds__(kMmaWarps * 32, 1)
    router_mma_kernel(RouterArgs a, int64_t ntiles) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();  // the grouping kernel may launch now; it waits for this grid
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = a.d, E = a.E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t slot_bytes = mma_slot_bytes(d);
  uint2* s_lo = reinterpret_cast<uint2*>(smem + kMmaSlots * slot_bytes);     // [warps][steps][32]
  float* s_part = reinterpret_cast<float*>(smem + kMmaSlots * slot_bytes + mma_lo_bytes(d));  // [2][warps][8][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_part + 2 * kMmaWarps * kMmaTile * 8);
  int* s_count = reinterpret_cast<int*>(bars + kMmaSlots);

  const int64_t g0 = blockIdx.x, gstride = gridDim.x;
  const int64_t my_tiles = g0 < ntiles ? (ntiles - 1 - g0) / gstride + 1 : 0;
  if (tid < 32) s_count[tid] = 0;
  if (tid == 0) {
    for (int i = 0; i < kMmaSlots; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  const size_t row_pitch = mma_row_pitch(d);
  auto issue = [&](int64_t j) {  // this block's j-th tile into slot j % 2: one bulk copy per token row
    const int64_t t0 = (g0 + j * gstride) * kMmaTile;
    const int rows = (int)(a.T - t0 < kMmaTile ? a.T - t0 : kMmaTile);
    uint8_t* dst = smem + (size_t)(j % kMmaSlots) * slot_bytes;
    uint64_t* bar = &bars[j % kMmaSlots];
    mbar_arrive_expect_tx(bar, (uint32_t)(rows * d * 2));
    for (int r = 0; r < rows; ++r) bulk_load(dst + r * row_pitch, a.x + (t0 + r) * d, (uint32_t)(d * 2), bar);
  };
  if (tid == 0)
    for (int64_t j = 0; j < my_tiles && j < kMmaSlots; ++j) issue(j);

  // B fragments of this warp's inputs: lane l holds expert l / 4 at inputs
  // 2 (l % 4) + {0, 1} and + {8, 9} of each 16-input step
  const int steps = d / (16 * kMmaWarps);
  const int n = lane >> 2, kq = 2 * (lane & 3);
  uint32_t bh[kMmaMaxSteps][2], bm[kMmaMaxSteps][2];
  uint2* my_lo = s_lo + (size_t)warp * steps * 32 + lane;
  // W_g comes from HBM at every launch: the loads of half the steps are
  // issued together before any is split, so the warp waits for two memory
  // round trips rather than one per step
  constexpr int kHalf = kMmaMaxSteps / 2;
#pragma unroll
  for (int ph = 0; ph < 2; ++ph) {
    float2 u[kHalf], v[kHalf];
#pragma unroll
    for (int q = 0; q < kHalf; ++q) {
      const int ks = ph * kHalf + q;
      u[q] = v[q] = make_float2(0.f, 0.f);
      if (ks < steps && n < E) {
        const float* row = a.Wg + (int64_t)n * d + warp * (steps * 16) + ks * 16 + kq;
        u[q] = *reinterpret_cast<const float2*>(row);
        v[q] = *reinterpret_cast<const float2*>(row + 8);
      }
    }
#pragma unroll
    for (int q = 0; q < kHalf; ++q) {
      const int ks = ph * kHalf + q;
      const float w[4] = {u[q].x, u[q].y, v[q].x, v[q].y};
      uint32_t h[4], m[4], lo[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) split3(w[c], h[c], m[c], lo[c]);
      bh[ks][0] = h[0] | (h[1] << 16);
      bh[ks][1] = h[2] | (h[3] << 16);
      bm[ks][0] = m[0] | (m[1] << 16);
      bm[ks][1] = m[2] | (m[3] << 16);
      if (ks < steps) my_lo[ks * 32] = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
    }
  }
  __syncwarp();
  // ldmatrix rows: thread l addresses row l % 8 of matrix l / 8 (matrices 0, 1:
  // inputs 0..7 of the step, 2, 3: inputs 8..15; rows 8..15 of the MMA repeat
  // rows 0..7)
  const int lr = lane & 7, lhalf = (lane >> 4) & 1;

  bool ok = true;
  for (int64_t j = 0; j < my_tiles; ++j) {
    const int slot = (int)(j % kMmaSlots);
    const int64_t t0 = (g0 + j * gstride) * kMmaTile;
    if (ok) ok = mbar_wait(&bars[slot], (uint32_t)((j / kMmaSlots) & 1), nullptr);
    // three independent accumulators (one per weight term) keep the MMAs of
    // a step from waiting on each other; they are added at the end
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      float ch[4] = {}, cm[4] = {}, cl[4] = {};
      const uint32_t base = smem_u32(smem + (size_t)slot * slot_bytes);
#pragma unroll
      for (int ks = 0; ks < kMmaMaxSteps; ++ks) {
        if (ks < steps) {
          const int k0 = warp * (steps * 16) + ks * 16;     // first input of the step
          const uint32_t addr = base + (uint32_t)(lr * row_pitch + k0 * 2 + lhalf * 16);
          uint32_t af[4];
          ldmatrix_x4(addr, af);
          const uint2 bl = my_lo[ks * 32];
          mma_bf16_16816(ch, af, bh[ks][0], bh[ks][1]);
          mma_bf16_16816(cm, af, bm[ks][0], bm[ks][1]);
          mma_bf16_16816(cl, af, bl.x, bl.y);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) c[q] = (ch[q] + cm[q]) + cl[q];
    }
    // c[0], c[1]: token lane / 4, experts kq, kq + 1
    float* part = s_part + (j & 1) * kMmaWarps * kMmaTile * 8;
    *reinterpret_cast<float2*>(part + (warp * kMmaTile + n) * 8 + kq) = make_float2(c[0], c[1]);
    if (!__syncthreads_and(ok)) {
      // a tile never arrived: report, let the copies still in flight land, leave
      if (tid == 0) {
        record_status(a.status, kStatusTimeout);
        for (int64_t q = j; q < my_tiles && q < j + kMmaSlots; ++q)
          mbar_wait(&bars[q % kMmaSlots], (uint32_t)((q / kMmaSlots) & 1), nullptr, kWaitLimitNs / 8);
      }
      return;
    }
    if (tid == 0 && j + kMmaSlots < my_tiles) issue(j + kMmaSlots);
    // warp w < 8 finishes token t0 + w: lane e < 8 adds the 16 warps' partials in warp order
    if (warp < kMmaTile && t0 + warp < a.T) {
      float v = 0.f;
      if (lane < 8) {
#pragma unroll
        for (int ww = 0; ww < kMmaWarps; ++ww) v += part[(ww * kMmaTile + warp) * 8 + lane];
      }
      finish_token<8>(a, t0 + warp, v, lane, s_count);
    }
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

static cudaError_t launch_router_mma(const RouterArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = mma_smem_bytes(a.d);
  cudaError_t err = cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t ntiles = (a.T + kMmaTile - 1) / kMmaTile;
  const int64_t grid = ntiles < num_sms ? ntiles : num_sms;
  router_mma_kernel<<<(unsigned)grid, kMmaWarps * 32, smem, s>>>(a, ntiles);
  return cudaGetLastError();
}

constexpr int64_t kFewTokens = 512;

template <int EMAX>
static cudaError_t launch_router_e(const RouterArgs& a, cudaStream_t s) {
  constexpr int G = EMAX <= 8 ? 4 : (EMAX <= 16 ? 2 : 1);
  const int g = a.T <= kFewTokens ? 1 : G;
  const int64_t blocks = (a.T + g - 1) / g;
  if (g == 1)
    router_group_kernel<EMAX, 1><<<(unsigned)blocks, kGroupThreads, 0, s>>>(a);
  else
    router_group_kernel<EMAX, G><<<(unsigned)blocks, kGroupThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a, int num_sms, cudaStream_t s, bool counts_zeroed) {
  if (!counts_zeroed) {
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
    if (err != cudaSuccess) return err;
  }
  // Many tokens: tensor cores (fewer instructions per token); few tokens: the
  // register kernel, whose set-up (W_g into registers) is shorter.
  if (a.T >= kMmaMinTokens && a.E <= 8 && a.d % (16 * kMmaWarps) == 0 && a.d <= 16 * kMmaWarps * kMmaMaxSteps)
    return launch_router_mma(a, num_sms, s);
  if (a.E <= 8 && a.d <= 8 * kRegMaxThreads) {
    // tokens per SM decide how many rows one ring slot carries
    const int64_t per_sm = (a.T + num_sms - 1) / num_sms;
    if (per_sm >= 16) return launch_router_reg<4>(a, num_sms, s);
    if (per_sm >= 4) return launch_router_reg<2>(a, num_sms, s);
    return launch_router_reg<1>(a, num_sms, s);
  }
  if (a.E <= 8) return launch_router_e<8>(a, s);
  if (a.E <= 16) return launch_router_e<16>(a, s);
  return launch_router_e<32>(a, s);
}

}  // namespace moe
