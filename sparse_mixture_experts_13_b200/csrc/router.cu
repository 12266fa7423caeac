// Router and top-k gate.
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (G(x) = Softmax(TopK(x . W_g)), logits outside the top-k at -inf), and
// "Mixtral", section "MoE Layer" (bias-free nn.Linear router, topk of the
// logits, softmax over the k kept logits).
//
// One warp per token.  Lane l reads 16-byte vectors l, l+32, ... of the
// token's bf16 row and accumulates E fp32 dot products against W_g, which the
// block stages once in shared memory (E * d * 4 bytes) when it fits.  A
// butterfly shuffle leaves every logit in every lane; the top-k (ties to the
// smaller expert index), the k-way softmax and the full-softmax probability
// of each chosen expert are computed redundantly per lane and lanes 0..k-1
// write one slot each.  The per-expert histogram is aggregated in shared
// memory and added to global memory once per block.
#include <cfloat>
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

constexpr int kRouterThreads = 512;
constexpr size_t kRouterMaxStage = 160 * 1024;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int EMAX, bool STAGED>
__global__ void __launch_bounds__(kRouterThreads) router_topk_kernel(RouterArgs a) {
  extern __shared__ __align__(16) float s_wg[];
  __shared__ int s_count[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int E = a.E, k = a.k, d = a.d;
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
  for (int64_t t = (int64_t)blockIdx.x * nwarps + warp; t < a.T; t += (int64_t)gridDim.x * nwarps) {
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + t * d);
#pragma unroll 2
    for (int v = lane; v < nvec; v += 32) {
      float xf[8];
      bf16x8_to_f32(__ldg(xr + v), xf);
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          const float4* w = reinterpret_cast<const float4*>(wg + (int64_t)e * d + (int64_t)v * 8);
          const float4 w0 = w[0], w1 = w[1];
          float s = acc[e];
          s = fmaf(xf[0], w0.x, s);
          s = fmaf(xf[1], w0.y, s);
          s = fmaf(xf[2], w0.z, s);
          s = fmaf(xf[3], w0.w, s);
          s = fmaf(xf[4], w1.x, s);
          s = fmaf(xf[5], w1.y, s);
          s = fmaf(xf[6], w1.z, s);
          s = fmaf(xf[7], w1.w, s);
          acc[e] = s;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }

    // top-k: repeated arg-max over the experts not yet chosen; strict '>'
    // keeps the smaller index on equal logits.
    int sel[4] = {0, 0, 0, 0};
    float sl[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t chosen = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
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
    // softmax over the k kept logits (largest first), and the full softmax
    // over all E logits evaluated at the chosen experts.
    const float m = sl[0];
    float zk = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j < k) zk += expf(sl[j] - m);
    float zE = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) zE += expf(acc[e] - m);

#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < k && lane == j) {
        const float ej = expf(sl[j] - m);
        a.topk_idx[t * k + j] = sel[j];
        a.topk_w[t * k + j] = ej / zk;
        a.topk_p[t * k + j] = ej / zE;
        atomicAdd(&s_count[sel[j]], 1);
      }
    }
    if (a.logits) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E && lane == e) a.logits[t * E + e] = acc[e];
    }
  }
  __syncthreads();
  if (tid < E && s_count[tid] != 0) atomicAdd(&a.counts[tid], s_count[tid]);
}

template <int EMAX>
static cudaError_t launch_router_e(const RouterArgs& a, int num_sms, cudaStream_t s) {
  const int warps = kRouterThreads / 32;
  int64_t blocks = (a.T + warps - 1) / warps;
  if (blocks > num_sms) blocks = num_sms;
  const size_t stage = (size_t)a.E * a.d * sizeof(float);
  if (stage <= kRouterMaxStage) {
    cudaError_t err = cudaFuncSetAttribute(router_topk_kernel<EMAX, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kRouterMaxStage);
    if (err != cudaSuccess) return err;
    router_topk_kernel<EMAX, true><<<(unsigned)blocks, kRouterThreads, stage, s>>>(a);
  } else {
    router_topk_kernel<EMAX, false><<<(unsigned)blocks, kRouterThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a, int num_sms, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
  if (err != cudaSuccess) return err;
  if (a.E <= 8) return launch_router_e<8>(a, num_sms, s);
  if (a.E <= 16) return launch_router_e<16>(a, num_sms, s);
  return launch_router_e<32>(a, num_sms, s);
}

}  // namespace moe
