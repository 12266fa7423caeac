// Router and top-k gate.
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (G(x) = Softmax(TopK(x . W_g)), logits outside the top-k at -inf), and
// "Mixtral", section "MoE Layer" (bias-free nn.Linear router, topk of the
// logits, softmax over the k kept logits).
//
// Logits are fp32 dot products of a token's bf16 row with the E rows of W_g.
// Three kernels compute them:
//
// router_mma_kernel (from 192 tokens, E <= 8, d a multiple of 512 up to
//   4096): tensor-core MMAs on W_g split exactly into three bf16 terms, in
//   clusters of 4 CTAs that split d (described at the kernel below).
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
// In all three, the top-k (ties to the smaller expert index), the k-way
// softmax and the full-softmax probability of each chosen expert are
// computed redundantly per lane of one warp (or of an 8-lane segment) and
// lanes 0..k-1 write one slot each.  The
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

// Lane e < E of a segment of SEG lanes holds the logit l of expert e for
// token t (other lanes of the segment: any value; `lane` is the index within
// the segment).  Every lane ranks its expert in the order (logit
// descending, index ascending), so the experts of rank < k are the top-k,
// rank 0 first, and ranks k .. 2k-1 are the next-best candidates.  With m
// the largest logit, the gate of a chosen expert is exp(l - m) over the sum
// of exp(l' - m) of the k chosen ones, and its full-softmax probability is
// exp(l - m) over the sum across all E experts.  The sums are butterflies
// over the first EMAX lanes of the segment (a fixed order).  Lane e writes
// the slot of its rank and counts it in *hist.  Every lane of the warp calls
// this (the shuffles span it); a segment with `active` false writes nothing.
template <int EMAX, int SEG = 32>
__device__ __forceinline__ void finish_token(const RouterArgs& a, int64_t t, float l, int lane, int* hist,
                                             bool active = true) {
  static_assert(EMAX <= SEG, "the experts of a token fit its segment");
  const int E = a.E, k = a.k;
  const bool valid = lane < E;
  int rank = 0;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    const float le = __shfl_sync(0xffffffffu, l, e, SEG);
    if (e < E && (le > l || (le == l && e < lane))) ++rank;
  }
  float m = valid ? l : -FLT_MAX;
#pragma unroll
  for (int off = EMAX / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off, SEG));
  const float ex = valid ? expf(l - m) : 0.f;
  float zE = ex, zk = (valid && rank < k) ? ex : 0.f;
#pragma unroll
  for (int off = EMAX / 2; off > 0; off >>= 1) {
    zE += __shfl_xor_sync(0xffffffffu, zE, off, SEG);
    zk += __shfl_xor_sync(0xffffffffu, zk, off, SEG);
  }
  if (!active) return;
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
// router_mma_kernel (E <= 8, d a multiple of 512 up to 4096): the logits of a
// tile of 16 tokens by mma.sync m16n8k16 (bf16 operands, fp32 accumulation),
// computed by a cluster of 4 CTAs that split d four ways.  x is exact in bf16,
// and every fp32 weight is split exactly into three bf16 terms, w = hi + mid
// + lo (8 + 8 + 8 significant bits, by truncation), so the three MMAs per 16
// inputs multiply exactly by the fp32 weights and the products add up in fp32.
//
// CTA c of a cluster owns inputs [c d/4, (c+1) d/4) and reads only that
// quarter of W_g; each of its 8 MMA warps owns d/32 of those inputs and keeps
// its slice of the three weight terms in registers as MMA B fragments for the
// whole launch.  The CTAs of a cluster walk the same token tiles.  A producer
// warp brings a CTA's quarter of each tile's 16 rows into a ring of
// shared-memory slots with one TMA load, viewed as (64 inputs, 16 rows, d/256
// chunks of 64) so that the slot holds chunk-major 128-byte rows with the
// 128-byte swizzle: the 8 token rows one ldmatrix reads fall in distinct bank
// groups.  Each MMA warp pushes its partial logits of tokens 4c' .. 4c'+3
// straight into CTA c''s receive ring with asynchronous remote stores
// counted on that CTA's mbarrier, and frees the slot.  Four finishing warps
// take the tiles in turn: for each of the CTA's four tokens of a tile (one
// 8-lane segment each) they add the 32 partials (CTA order, then warp order),
// finish the token and tell the senders that the ring entry was read (a
// relaxed remote arrive).  No step needs a cluster-wide fence, and loads,
// MMAs and finishing overlap across tiles.
constexpr int kMmaCtas = 4;       // cluster size: d split four ways
constexpr int kMmaWarps = 8;      // MMA warps
constexpr int kMmaTile = 16;      // tokens per tile (the MMA's M)
constexpr int kMmaSlots = 4;      // ring of token tiles per CTA
constexpr int kMmaMaxSteps = 8;   // 16-input steps per MMA warp (d <= 4096)
constexpr int kMmaRecv = 8;       // receive ring of a CTA's partial logits (tiles)
constexpr int kMmaPerCta = kMmaTile / kMmaCtas;  // tokens each CTA finishes per tile
constexpr int kMmaProducer = kMmaWarps;          // the warp that issues the tile loads
constexpr int kMmaFinishers = 4;                 // finishing warps, tiles in turn
constexpr int kMmaFinisher0 = kMmaProducer + 1;
constexpr int kMmaThreads = 32 * (kMmaFinisher0 + kMmaFinishers);
// one tile's partials into one CTA: [sender CTA][MMA warp][token][expert] fp32
constexpr uint32_t kMmaRecvFloats = kMmaCtas * kMmaWarps * kMmaPerCta * 8;
constexpr uint32_t kMmaRecvBytes = kMmaRecvFloats * 4;
constexpr int64_t kMmaMinTokens = 192;
static_assert(kMmaPerCta * 8 == 32, "a finishing warp holds one CTA's tokens of a tile, 8 lanes per token");
static_assert(kMmaRecv % kMmaFinishers == 0, "a ring entry is always finished by the same warp");

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

// 8-byte asynchronous store into a cluster peer's shared memory, counted (as
// transaction bytes) on the peer's mbarrier at `bar`
__device__ __forceinline__ void st_async_f32x2(uint32_t cluster_addr, float v0, float v1, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
                   cluster_addr),
               "f"(v0), "f"(v1), "r"(bar)
               : "memory");
}
// arrive on named barrier `id` (of `nthreads` threads) without waiting
__device__ __forceinline__ void named_bar_arrive(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// split-phase cluster barrier: a relaxed arrive (no ordering of this thread's
// memory operations) and an acquiring wait
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// arrive on a (possibly remote) mbarrier without ordering this thread's
// earlier memory operations: the reads it reports have been consumed already
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// a slot: a CTA's quarter of 16 token rows, chunk-major rows of 64 inputs
__host__ __device__ constexpr size_t mma_slot_bytes(int d) { return (size_t)kMmaTile * (d / kMmaCtas) * 2; }
__host__ __device__ constexpr size_t mma_smem_bytes(int d) {
  return 1024 + kMmaSlots * mma_slot_bytes(d) + (size_t)kMmaRecv * kMmaRecvBytes +
         sizeof(uint64_t) * 2 * (kMmaSlots + kMmaRecv) + sizeof(int) * 32;
}

__global__ void __launch_bounds__(kMmaThreads, 1)
    router_mma_kernel(const __grid_constant__ CUtensorMap xmap, RouterArgs a, int64_t ntiles, int64_t nclusters) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();  // the grouping kernel may launch now; it waits for this grid
  // the 128-byte swizzle repeats every 1024 bytes: slots start on that boundary
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = a.d, E = a.E;
  const int dq = d / kMmaCtas;                 // inputs of this CTA
  const int chunks = dq / 64;                  // 64-input chunks of this CTA
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int crank = (int)cluster_ctarank();
  const int64_t cl = blockIdx.x / kMmaCtas;    // the cluster (its CTAs are consecutive blocks)
  const size_t slot_bytes = mma_slot_bytes(d);
  float* s_recv = reinterpret_cast<float*>(smem + kMmaSlots * slot_bytes);    // [ring][kMmaRecvFloats]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_recv + kMmaRecv * kMmaRecvFloats);  // a slot is loaded
  uint64_t* empty = full + kMmaSlots;           // the MMA warps have read a slot
  uint64_t* recv_full = empty + kMmaSlots;      // a ring entry holds every partial of its tile
  uint64_t* recv_empty = recv_full + kMmaRecv;  // every CTA has read what this CTA sent to an entry
  int* s_count = reinterpret_cast<int*>(recv_empty + kMmaRecv);

  // every CTA of a cluster has the same tiles: cl, cl + nclusters, ...
  const int64_t my_tiles = cl < ntiles ? (ntiles - 1 - cl) / nclusters + 1 : 0;
  if (tid < 32) s_count[tid] = 0;
  auto issue = [&](int64_t j) {  // this CTA's quarter of tile j's rows into slot j % kMmaSlots
    uint64_t* bar = &full[j % kMmaSlots];
    mbar_arrive_expect_tx(bar, (uint32_t)slot_bytes);  // rows past T are zero-filled and counted
    tma_load_3d(&xmap, bar, smem + (size_t)(j % kMmaSlots) * slot_bytes, 0,
                (int32_t)((cl + j * nclusters) * kMmaTile), crank * chunks);
  };

  // B fragments of this warp's inputs: lane l holds expert l / 4 at inputs
  // 2 (l % 4) + {0, 1} and + {8, 9} of each 16-input step.  All of the
  // warp's W_g loads are issued before the first token tile is requested
  // (so they do not queue behind it) and before any is split.
  const int steps = dq / (16 * kMmaWarps);
  const int n = lane >> 2, kq = 2 * (lane & 3);
  uint32_t bh[kMmaMaxSteps][2], bm[kMmaMaxSteps][2], bl[kMmaMaxSteps][2];
  float2 u[kMmaMaxSteps], v[kMmaMaxSteps];
  if (warp < kMmaWarps) {
    const int k_warp = crank * dq + warp * steps * 16;  // first input of this warp
#pragma unroll
    for (int q = 0; q < kMmaMaxSteps; ++q) {
      u[q] = v[q] = make_float2(0.f, 0.f);
      if (q < steps && n < E) {
        const float* row = a.Wg + (int64_t)n * d + k_warp + q * 16 + kq;
        u[q] = *reinterpret_cast<const float2*>(row);
        v[q] = *reinterpret_cast<const float2*>(row + 8);
      }
    }
  }
  // the producer requests the first tiles once the W_g loads are out
  if (warp < kMmaWarps) named_bar_arrive(2, 32 * (kMmaWarps + 1));
  else if (warp == kMmaProducer) named_bar_sync(2, 32 * (kMmaWarps + 1));
  int64_t issued = 0;  // producer lane 0: tiles whose loads were issued
  if (warp == kMmaProducer && lane == 0) {
    tma_prefetch_desc(&xmap);
    for (int i = 0; i < kMmaSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kMmaWarps);
    }
    for (int i = 0; i < kMmaRecv; ++i) {
      mbar_init(&recv_full[i], 1);
      mbar_init(&recv_empty[i], kMmaCtas);
      if (i < my_tiles) mbar_arrive_expect_tx(&recv_full[i], kMmaRecvBytes);
    }
    fence_barrier_init();
    for (; issued < my_tiles && issued < kMmaSlots; ++issued) issue(issued);
  }
  if (warp < kMmaWarps) {
#pragma unroll
    for (int q = 0; q < kMmaMaxSteps; ++q) {
      const float w[4] = {u[q].x, u[q].y, v[q].x, v[q].y};
      uint32_t h[4], m[4], lo[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) split3(w[c], h[c], m[c], lo[c]);
      bh[q][0] = h[0] | (h[1] << 16);
      bh[q][1] = h[2] | (h[3] << 16);
      bm[q][0] = m[0] | (m[1] << 16);
      bm[q][1] = m[2] | (m[3] << 16);
      bl[q][0] = lo[0] | (lo[1] << 16);
      bl[q][1] = lo[2] | (lo[3] << 16);
    }
  }
  __syncthreads();  // this CTA's barrier inits and zeroed counts are visible to its threads
  // every CTA's mbarriers are initialised (and the init fenced) before any
  // peer stores or arrives on them; nothing else needs ordering here
  cluster_arrive_relaxed();
  cluster_wait();

  bool ok = true;
  if (warp < kMmaWarps) {
    // ldmatrix rows: thread l addresses row l % 8 of matrix l / 8; matrices
    // 0..3 are (tokens 0-7, inputs 0-7), (tokens 8-15, inputs 0-7), (tokens
    // 0-7, inputs 8-15), (tokens 8-15, inputs 8-15): the A fragment's order.
    // Token row r of chunk c is the 128-byte row 16 c + r of the slot, whose
    // 16-byte pieces are permuted by r % 8 (the swizzle).
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8, lpiece = lane >> 4;
    // this lane's partials: tokens n and n + 8 (finished by CTAs n / 4 and
    // n / 4 + 2, as their token n % 4), experts kq and kq + 1
    const uint32_t dst_off =
        (uint32_t)(((crank * kMmaWarps + warp) * kMmaPerCta + (n % kMmaPerCta)) * 8 + kq) * 4;
    const uint32_t dst_rank0 = (uint32_t)(n / kMmaPerCta), dst_rank1 = dst_rank0 + 2;
    for (int64_t j = 0; j < my_tiles; ++j) {
      const int slot = (int)(j % kMmaSlots);
      if (ok) ok = mbar_wait(&full[slot], (uint32_t)((j / kMmaSlots) & 1), nullptr);
      // six independent accumulators (one per weight term and step parity)
      // keep the MMAs of consecutive steps from waiting on each other
      float acc[6][4];
#pragma unroll
      for (int q = 0; q < 6; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
      if (ok) {
        const uint32_t base = smem_u32(smem + (size_t)slot * slot_bytes);
#pragma unroll
        for (int ks = 0; ks < kMmaMaxSteps; ++ks) {
          if (ks < steps) {
            const int k0 = warp * steps * 16 + ks * 16;  // first input of the step in this CTA's quarter
            const uint32_t row = (uint32_t)((k0 >> 6) * kMmaTile + lrow);
            const uint32_t piece = (uint32_t)(((k0 & 63) >> 3) + lpiece);
            uint32_t af[4];
            ldmatrix_x4(base + row * 128 + ((piece ^ (row & 7)) << 4), af);
            float (&ch)[4] = acc[(ks & 1) * 3], (&cm)[4] = acc[(ks & 1) * 3 + 1], (&cq)[4] = acc[(ks & 1) * 3 + 2];
            mma_bf16_16816(ch, af, bh[ks][0], bh[ks][1]);
            mma_bf16_16816(cm, af, bm[ks][0], bm[ks][1]);
            mma_bf16_16816(cq, af, bl[ks][0], bl[ks][1]);
          }
        }
      }
      __syncwarp();  // the warp's reads of the slot are done
      if (lane == 0) mbar_arrive(&empty[slot]);
      float c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[q] = ((acc[0][q] + acc[3][q]) + (acc[1][q] + acc[4][q])) + (acc[2][q] + acc[5][q]);
      // into the finishing CTAs' ring entry, once every CTA has read tile j - ring from it
      const int b = (int)(j % kMmaRecv);
      if (j >= kMmaRecv && !mbar_wait(&recv_empty[b], (uint32_t)(((j / kMmaRecv) + 1) & 1), nullptr)) ok = false;
      const uint32_t dst = smem_u32(s_recv + (size_t)b * kMmaRecvFloats) + dst_off;
      const uint32_t bar = smem_u32(&recv_full[b]);
      st_async_f32x2(map_to_rank(dst, dst_rank0), c[0], c[1], map_to_rank(bar, dst_rank0));
      st_async_f32x2(map_to_rank(dst, dst_rank1), c[2], c[3], map_to_rank(bar, dst_rank1));
    }
    if (!ok && lane == 0) record_status(a.status, kStatusTimeout);
  } else if (warp == kMmaProducer) {
    if (lane == 0) {
      // refill each slot once all MMA warps have read it
      for (; issued < my_tiles; ++issued) {
        const int64_t prev = issued - kMmaSlots;
        if (!mbar_wait(&empty[prev % kMmaSlots], (uint32_t)((prev / kMmaSlots) & 1), nullptr)) {
          record_status(a.status, kStatusTimeout);
          break;
        }
        issue(issued);
      }
      // a CTA leaves only with no load in flight (the MMA warps wait for
      // every load, but may have given up on one)
      for (int64_t q = issued - kMmaSlots > 0 ? issued - kMmaSlots : 0; q < issued; ++q)
        mbar_wait(&full[q % kMmaSlots], (uint32_t)((q / kMmaSlots) & 1), nullptr, kWaitLimitNs / 8);
    }
  } else {
    // finishing warp f: tiles f, f + 4, ...; segment s (lanes 8s .. 8s+7)
    // finishes token 4 crank + s of the tile, lane e of the segment the logit
    // of expert e: the partials of the four CTAs' eight warps, CTA order,
    // warp order within a CTA
    const int f = warp - kMmaFinisher0, seg = lane >> 3, e = lane & 7;
    for (int64_t jj = f; jj < my_tiles; jj += kMmaFinishers) {
      const int b = (int)(jj % kMmaRecv);
      const int64_t t = (cl + jj * nclusters) * kMmaTile + crank * kMmaPerCta + seg;
      const bool okf = mbar_wait(&recv_full[b], (uint32_t)((jj / kMmaRecv) & 1), nullptr);
      // the entry's next use (tile jj + ring, this warp's too) expects its
      // bytes again; they come only after this warp reports the entry read
      if (lane == 0 && okf && jj + kMmaRecv < my_tiles) mbar_arrive_expect_tx(&recv_full[b], kMmaRecvBytes);
      float v = 0.f;
      if (okf) {
        const float* r = s_recv + (size_t)b * kMmaRecvFloats + seg * 8 + e;
#pragma unroll
        for (int c = 0; c < kMmaCtas; ++c) {
          float sc = 0.f;
#pragma unroll
          for (int w = 0; w < kMmaWarps; ++w) sc += r[(c * kMmaWarps + w) * kMmaPerCta * 8];
          v += sc;
        }
      }
      __syncwarp();  // v holds the sums: the senders may reuse the entry
      // (only entries that are used again are reported, so that every arrive
      // on a peer is awaited by that peer before it exits)
      if (lane < kMmaCtas && jj + kMmaRecv < my_tiles)
        mbar_arrive_remote_relaxed(map_to_rank(smem_u32(&recv_empty[b]), (uint32_t)lane));
      if (!okf && lane == 0) record_status(a.status, kStatusTimeout);
      finish_token<8, 8>(a, t, v, e, s_count, okf && t < a.T);
    }
  }
  // A CTA may leave now: every store a peer makes into it (a ring entry) and
  // every arrive on it (an entry read, reported only for entries in use
  // again) is awaited before this point.
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

// clusters of 4 router CTAs that can be resident at once on this device
static int router_mma_clusters(const cudaLaunchConfig_t& cfg) {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  if (dev >= 0 && cached[dev] > 0) return cached[dev];
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, router_mma_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    clusters = 0;
  }
  if (dev >= 0 && clusters > 0) cached[dev] = clusters;
  return clusters;
}

// x as (64 inputs, T rows, d / 64 chunks): strides 2 bytes, d * 2 bytes, 128
// bytes; a box is a CTA's quarter of 16 rows, stored chunk-major with the
// 128-byte swizzle.  False if the driver refuses the map.
static bool encode_router_map(CUtensorMap* m, const uint16_t* x, int64_t T, int d) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)(d / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)kMmaTile, (cuuint32_t)(d / kMmaCtas / 64)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// false: the tensor-core router cannot take this launch (the caller uses another)
static bool launch_router_mma(const RouterArgs& a, int num_sms, cudaStream_t s, cudaError_t* err) {
  CUtensorMap xmap;
  if (!encode_router_map(&xmap, a.x, a.T, a.d)) return false;
  const size_t smem = mma_smem_bytes(a.d);
  *err = cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (*err != cudaSuccess) return true;
  const int64_t ntiles = (a.T + kMmaTile - 1) / kMmaTile;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kMmaCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kMmaThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many clusters as fit at once (each walks several tiles), at most one per tile
  int64_t nclusters = num_sms / kMmaCtas;
  cfg.gridDim = dim3((unsigned)(nclusters * kMmaCtas), 1, 1);
  const int fit = router_mma_clusters(cfg);
  if (fit > 0 && fit < nclusters) nclusters = fit;
  if (ntiles < nclusters) nclusters = ntiles;
  if (nclusters < 1) nclusters = 1;
  cfg.gridDim = dim3((unsigned)(nclusters * kMmaCtas), 1, 1);
  *err = cudaLaunchKernelEx(&cfg, router_mma_kernel, xmap, a, ntiles, nclusters);
  return true;
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
  // From 192 tokens: tensor cores (fewer instructions per token, a quarter
  // of W_g per CTA; measured faster from 192 tokens, 12.3 -> 10.2 us at 256
  // and 16.4 -> 12.3 us at 1023); fewer tokens: the register kernel (the two
  // time the same there).
  if (a.T >= kMmaMinTokens && a.E <= 8 && a.d % (16 * kMmaWarps * kMmaCtas) == 0 &&
      a.d <= 16 * kMmaWarps * kMmaCtas * kMmaMaxSteps && (reinterpret_cast<uintptr_t>(a.x) & 15) == 0) {
    cudaError_t err = cudaSuccess;
    if (launch_router_mma(a, num_sms, s, &err)) return err;
  }
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
