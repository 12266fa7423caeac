// Router and top-k gate.
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (G(x) = Softmax(TopK(x . W_g)), logits outside the top-k at -inf), and
// "Mixtral", section "MoE Layer" (bias-free nn.Linear router, topk of the
// logits, softmax over the k kept logits).
//
// Logits are fp32 dot products of a token's bf16 row with the E rows of W_g,
// read as 16-byte vectors.  A block takes a group of tokens (one token when
// there are few, so that many SMs share the work) and splits d over its warps;
// every W_g vector a warp reads serves all tokens of the group.  The top-k
// (ties to the smaller expert index), the k-way softmax and the full-softmax
// probability of each chosen expert are computed redundantly per lane and
// lanes 0..k-1 write one slot each.  The per-expert histogram is aggregated in
// shared memory and added to global memory once per block.
#include <cfloat>
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

constexpr int kMaxK = 8;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// All lanes hold all E logits of token t.  Top-k by repeated arg-max over
// the experts not yet chosen (strict '>' keeps the smaller index on equal
// logits); softmax over the k kept logits; full softmax over all E at the
// chosen experts.  Lane j < k writes slot j and counts it in *hist.
template <int EMAX>
__device__ __forceinline__ void finish_token(const RouterArgs& a, int64_t t, const float (&acc)[EMAX], int lane,
                                             int* hist) {
  const int E = a.E, k = a.k;
  int sel[kMaxK];
  float sl[kMaxK];
  uint32_t chosen = 0;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    sel[j] = 0;
    sl[j] = 0.f;
    if (j < k) {
      int best = -1;
      float bl = -FLT_MAX;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E && !((chosen >> e) & 1u) && (best < 0 || acc[e] > bl)) {
          best = e;
          bl = acc[e];
        }
      }
      sel[j] = best;
      sl[j] = bl;
      chosen |= 1u << best;
    }
  }
  const float m = sl[0];
  float zk = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j)
    if (j < k) zk += expf(sl[j] - m);
  float zE = 0.f;
#pragma unroll
  for (int e = 0; e < EMAX; ++e)
    if (e < E) zE += expf(acc[e] - m);
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k && lane == j) {
      const float ej = expf(sl[j] - m);
      a.topk_idx[t * k + j] = sel[j];
      a.topk_w[t * k + j] = ej / zk;
      a.topk_p[t * k + j] = ej / zE;
      atomicAdd(&hist[sel[j]], 1);
    }
  }
  if (a.logits) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E && lane == e) a.logits[t * E + e] = acc[e];
  }
  if (a.next_idx) {
    // ranks k .. 2k-1 (capacity fallback): continue the same arg-max order
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        int best = -1;
        float bl = -FLT_MAX;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < E && !((chosen >> e) & 1u) && (best < 0 || acc[e] > bl)) {
            best = e;
            bl = acc[e];
          }
        }
        if (best >= 0) chosen |= 1u << best;
        if (lane == j) {
          a.next_idx[t * k + j] = best;
          a.next_p[t * k + j] = best >= 0 ? expf(bl - m) / zE : 0.f;
        }
      }
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
    float lg[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGroupWarps; ++w) v += s_part[w][warp][e];
      lg[e] = v;
    }
    finish_token<EMAX>(a, t0 + warp, lg, lane, s_count);
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
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
  (void)num_sms;
  if (a.E <= 8) return launch_router_e<8>(a, s);
  if (a.E <= 16) return launch_router_e<16>(a, s);
  return launch_router_e<32>(a, s);
}

}  // namespace moe
