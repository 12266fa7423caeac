// Router and top-k gate.
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (G(x) = Softmax(TopK(x . W_g)), logits outside the top-k at -inf), and
// "Mixtral", section "MoE Layer" (bias-free nn.Linear router, topk of the
// logits, softmax over the k kept logits).
//
// Logits are fp32 dot products of a token's bf16 row with the E rows of W_g,
// read as 16-byte vectors.  Many tokens: one warp per group of tokens, W_g
// staged once per block in shared memory (E * d * 4 bytes) when it fits, each
// W_g vector serving the whole group; a butterfly shuffle leaves every logit
// in every lane.  Few tokens: one block per token with d split over the
// block's threads.  The top-k (ties to the smaller expert index), the k-way
// softmax and the full-softmax probability of each chosen expert are computed
// redundantly per lane and lanes 0..k-1 write one slot each.  The per-expert
// histogram is aggregated in shared memory and added to global memory once
// per block (or added directly by the per-token blocks).
#include <cfloat>
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

constexpr int kRouterThreads = 512;
constexpr int kMaxK = 8;
constexpr size_t kRouterMaxStage = 160 * 1024;

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

// Many tokens: one warp per TPW tokens; each W_g vector read from shared
// memory (when staged) serves the TPW tokens.
template <int EMAX, int TPW, bool STAGED>
__global__ void __launch_bounds__(kRouterThreads) router_tokens_kernel(RouterArgs a) {
  extern __shared__ __align__(16) float s_wg[];
  __shared__ int s_count[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int E = a.E, d = a.d;
  if (tid < 32) s_count[tid] = 0;
  const float* wg = a.Wg;
  if (STAGED) {
    const int64_t n4 = (int64_t)E * d / 4;
    const float4* src = reinterpret_cast<const float4*>(a.Wg);
    float4* dst = reinterpret_cast<float4*>(s_wg);
    for (int64_t i = tid; i < n4; i += blockDim.x) dst[i] = __ldg(src + i);
    wg = s_wg;
  }
  __syncthreads();

  const int nvec = d >> 3;
  const int64_t groups = (a.T + TPW - 1) / TPW;
  for (int64_t g = (int64_t)blockIdx.x * nwarps + warp; g < groups; g += (int64_t)gridDim.x * nwarps) {
    const int64_t t0 = g * TPW;
    float acc[TPW][EMAX];
#pragma unroll
    for (int i = 0; i < TPW; ++i)
#pragma unroll
      for (int e = 0; e < EMAX; ++e) acc[i][e] = 0.f;
    for (int v = lane; v < nvec; v += 32) {
      float xf[TPW][8];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        if (t0 + i < a.T) {
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + (t0 + i) * d) + v), xf[i]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) xf[i][q] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          const float4* w = reinterpret_cast<const float4*>(wg + (int64_t)e * d + (int64_t)v * 8);
          const float4 w0 = w[0], w1 = w[1];
#pragma unroll
          for (int i = 0; i < TPW; ++i) acc[i][e] = dot8(xf[i], w0, w1, acc[i][e]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], off);
      }
      if (t0 + i < a.T) finish_token<EMAX>(a, t0 + i, acc[i], lane, s_count);
    }
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

// Few tokens: one block per token, the d dimension split over all threads,
// W_g read straight from L2.
constexpr int kSplitThreads = 256;

template <int EMAX>
__global__ void __launch_bounds__(kSplitThreads) router_split_kernel(RouterArgs a) {
  __shared__ float s_part[kSplitThreads / 32][EMAX];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, d = a.d;
  const int64_t t = blockIdx.x;
  const int nvec = d >> 3;
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
  for (int v = tid; v < nvec; v += kSplitThreads) {
    float xf[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + t * d) + v), xf);
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        const float4* w = reinterpret_cast<const float4*>(a.Wg + (int64_t)e * d + (int64_t)v * 8);
        acc[e] = dot8(xf, __ldg(w), __ldg(w + 1), acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e) s_part[warp][e] = acc[e];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kSplitThreads / 32; ++w) v += s_part[w][e];
      acc[e] = v;
    }
    finish_token<EMAX>(a, t, acc, lane, a.counts);
  }
}

constexpr int64_t kSplitMaxT = 512;

template <int EMAX>
static cudaError_t launch_router_e(const RouterArgs& a, int num_sms, cudaStream_t s) {
  if (a.T <= kSplitMaxT) {
    router_split_kernel<EMAX><<<(unsigned)a.T, kSplitThreads, 0, s>>>(a);
    return cudaGetLastError();
  }
  constexpr int TPW = EMAX <= 8 ? 4 : 1;
  const int warps = kRouterThreads / 32;
  int64_t blocks = (a.T + warps * TPW - 1) / (warps * TPW);
  if (blocks > num_sms) blocks = num_sms;
  const size_t stage = (size_t)a.E * a.d * sizeof(float);
  if (stage <= kRouterMaxStage) {
    cudaError_t err = cudaFuncSetAttribute(router_tokens_kernel<EMAX, TPW, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRouterMaxStage);
    if (err != cudaSuccess) return err;
    router_tokens_kernel<EMAX, TPW, true><<<(unsigned)blocks, kRouterThreads, stage, s>>>(a);
  } else {
    router_tokens_kernel<EMAX, TPW, false><<<(unsigned)blocks, kRouterThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a, int num_sms, cudaStream_t s, bool counts_zeroed) {
  if (!counts_zeroed) {
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
    if (err != cudaSuccess) return err;
  }
  if (a.E <= 8) return launch_router_e<8>(a, num_sms, s);
  if (a.E <= 16) return launch_router_e<16>(a, num_sms, s);
  return launch_router_e<32>(a, num_sms, s);
}

}  // namespace moe
