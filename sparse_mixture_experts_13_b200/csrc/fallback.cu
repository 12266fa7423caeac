// Next-best-expert fallback for slots that overflow an expert's capacity.
//
// Source: "How Mixtral 8x7B uses mixture of experts", section "Routing
// without auxiliary loss": slots beyond a full expert's capacity go to a
// fallback, usually the token's next-best expert.  Reading taken: after the
// capacity pass, the dropped slots of token t, in slot order, move to t's
// experts at router ranks k, k+1, ... (logit descending, index ascending; the
// router writes those ranks and their full-softmax probabilities).  At each
// expert the moved slots compete, under the same policy, for the capacity the
// first pass left; a moved slot keeps its gate weight; one that does not fit
// is dropped.
//
// Both passes select with the same radix select over 64-bit keys that are
// unique per expert:
//   by probability: (bits of p as float) << 32 | (0xFFFFFFFF - t)
//   by token order:                              0xFFFFFFFF - t
// so "keep the r largest keys" is the policy in either case.  The result is
// an expert per slot (-1 = dropped) and its histogram, which the ordinary
// grouping kernel then lays out in slot order.
#include <cstdint>

#include "moe_internal.h"
#include "select.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kFbThreads = 256;

__device__ __forceinline__ uint64_t fb_key(bool by_prob, float p, int64_t t) {
  const uint64_t order = (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
  return by_prob ? (((uint64_t)__float_as_uint(p) << 32) | order) : order;
}

// keys1[s]: the first pass's key of slot s at its top-k expert.
__global__ void __launch_bounds__(kFbThreads) fb_keys_kernel(const float* __restrict__ p, uint64_t* __restrict__ keys,
                                                             int64_t S, int32_t k, int32_t by_prob) {
  for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < S; s += (int64_t)gridDim.x * blockDim.x)
    keys[s] = fb_key(by_prob != 0, by_prob ? p[s] : 0.f, s / k);
}

// One block per expert: thresh[e] = the r-th largest key among the slots with
// expert[s] == e, r = cap - (used ? used[e] : 0).  0 when every such slot
// fits, ~0 when none does.
__global__ void __launch_bounds__(kSelectThreads) fb_select_kernel(const int32_t* __restrict__ expert,
                                                                   const uint64_t* __restrict__ keys,
                                                                   const int32_t* __restrict__ counts,
                                                                   const int32_t* __restrict__ used, int64_t cap,
                                                                   uint64_t* __restrict__ thresh, int64_t S) {
  const int e = blockIdx.x;
  const int64_t cnt = counts[e];
  const int64_t room = cap - (used ? (int64_t)used[e] : 0);
  if (cnt <= room) {
    if (threadIdx.x == 0) thresh[e] = 0;
    return;
  }
  if (room <= 0) {
    if (threadIdx.x == 0) thresh[e] = ~0ull;
    return;
  }
  const uint64_t t = block_radix_select(
      [&](int64_t s, uint64_t& key) {
        if (expert[s] != e) return false;
        key = keys[s];
        return true;
      },
      S, cnt, room);
  if (threadIdx.x == 0) thresh[e] = t;
}

// One thread per token: keep or move each slot.  A kept slot keeps its
// expert (eff = idx); the m-th dropped slot of the token becomes a candidate
// for the expert at router rank k + m with its key there (eff = -2, pending),
// or is dropped (eff = -1) when the token has no such rank.
__global__ void __launch_bounds__(kFbThreads) fb_classify_kernel(
    const int32_t* __restrict__ idx, const uint64_t* __restrict__ keys1, const uint64_t* __restrict__ thresh1,
    const int32_t* __restrict__ next_idx, const float* __restrict__ next_p, int32_t* __restrict__ eff,
    int32_t* __restrict__ cand, uint64_t* __restrict__ keys2, int32_t* kept1_count, int32_t* cand_count, int64_t T,
    int32_t k, int32_t E, int32_t by_prob) {
  __shared__ int32_t h_kept[32], h_cand[32];
  if (threadIdx.x < 32) {
    h_kept[threadIdx.x] = 0;
    h_cand[threadIdx.x] = 0;
  }
  __syncthreads();
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
    int m = 0;
    for (int j = 0; j < k; ++j) {
      const int64_t s = t * k + j;
      const int32_t e = idx[s];
      if (keys1[s] >= thresh1[e]) {
        eff[s] = e;
        cand[s] = -1;
        atomicAdd(&h_kept[e], 1);
        continue;
      }
      const int32_t e2 = next_idx[t * k + m];
      const float p2 = next_p[t * k + m];
      ++m;
      if (e2 >= 0 && e2 < E) {
        eff[s] = -2;
        cand[s] = e2;
        keys2[s] = fb_key(by_prob != 0, by_prob ? p2 : 0.f, t);
        atomicAdd(&h_cand[e2], 1);
      } else {
        eff[s] = -1;
        cand[s] = -1;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < E) {
    if (h_kept[threadIdx.x]) atomicAdd(&kept1_count[threadIdx.x], h_kept[threadIdx.x]);
    if (h_cand[threadIdx.x]) atomicAdd(&cand_count[threadIdx.x], h_cand[threadIdx.x]);
  }
}

// One thread per slot: settle the pending candidates and count the experts
// that process a slot.
__global__ void __launch_bounds__(kFbThreads) fb_finalize_kernel(const int32_t* __restrict__ cand,
                                                                 const uint64_t* __restrict__ keys2,
                                                                 const uint64_t* __restrict__ thresh2,
                                                                 int32_t* __restrict__ eff, int32_t* counts_eff,
                                                                 int64_t S, int32_t E) {
  __shared__ int32_t h[32];
  if (threadIdx.x < 32) h[threadIdx.x] = 0;
  __syncthreads();
  for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < S; s += (int64_t)gridDim.x * blockDim.x) {
    int32_t e = eff[s];
    if (e == -2) {
      const int32_t e2 = cand[s];
      e = keys2[s] >= thresh2[e2] ? e2 : -1;
      eff[s] = e;
    }
    if (e >= 0) atomicAdd(&h[e], 1);
  }
  __syncthreads();
  if (threadIdx.x < E && h[threadIdx.x]) atomicAdd(&counts_eff[threadIdx.x], h[threadIdx.x]);
}

unsigned grid_for(int64_t n, int num_sms) {
  int64_t b = (n + kFbThreads - 1) / kFbThreads;
  if (b > 4 * num_sms) b = 4 * num_sms;
  return (unsigned)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_fallback(const FallbackArgs& a, int num_sms, cudaStream_t s) {
  const int64_t S = a.T * a.k;
  const int32_t by_prob = a.policy == 0 ? 1 : 0;
  fb_keys_kernel<<<grid_for(S, num_sms), kFbThreads, 0, s>>>(a.topk_p, a.keys1, S, a.k, by_prob);
  cudaError_t err = cudaFuncSetAttribute(fb_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (err != cudaSuccess) return err;
  fb_select_kernel<<<a.E, kSelectThreads, kSelectSmem, s>>>(a.topk_idx, a.keys1, a.counts, nullptr, a.cap,
                                                            a.thresh1, S);
  fb_classify_kernel<<<grid_for(a.T, num_sms), kFbThreads, 0, s>>>(a.topk_idx, a.keys1, a.thresh1, a.next_idx,
                                                                    a.next_p, a.eff, a.cand, a.keys2, a.kept1_count,
                                                                    a.cand_count, a.T, a.k, a.E, by_prob);
  fb_select_kernel<<<a.E, kSelectThreads, kSelectSmem, s>>>(a.cand, a.keys2, a.cand_count, a.kept1_count, a.cap,
                                                            a.thresh2, S);
  fb_finalize_kernel<<<grid_for(S, num_sms), kFbThreads, 0, s>>>(a.cand, a.keys2, a.thresh2, a.eff, a.counts_eff, S,
                                                                  a.E);
  return cudaGetLastError();
}

}  // namespace moe
