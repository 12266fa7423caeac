// Router statistics: per-slot expert histograms and first-two-choice pair
// counts of the top-k indices.
//
// Sources: "How Mixtral 8x7B uses mixture of experts", "Expert
// specialization" (per layer, the bincount of the top-2 expert indices over
// the tokens: an expert-activation heatmap) and "Mixtral 8x7B — MoE Complete
// Guide", "Inspecting Expert Routing" (the most common expert in each top-k
// position).
//   slot_counts[j][e] = #{t : topk_idx[t][j] == e}          [k, E]
//   pair_counts[a][b] = #{t : topk_idx[t][0..1] == (a, b)}  [E, E], k >= 2
// Each block builds its histograms in shared memory (atomics) from a
// contiguous range of tokens and adds them to the outputs with one global
// atomic per non-zero bin.
#include <cstdint>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kStatsThreads = 256;

__global__ void __launch_bounds__(kStatsThreads) router_stats_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                                     int32_t E, int32_t k, int32_t* slot_counts,
                                                                     int32_t* pair_counts) {
  __shared__ int32_t h_slot[8 * 32];
  __shared__ int32_t h_pair[32 * 32];
  const int n_slot = k * E, n_pair = pair_counts ? E * E : 0;
  for (int i = threadIdx.x; i < n_slot; i += blockDim.x) h_slot[i] = 0;
  for (int i = threadIdx.x; i < n_pair; i += blockDim.x) h_pair[i] = 0;
  __syncthreads();
  const int64_t per_block = (T + gridDim.x - 1) / gridDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * per_block;
  const int64_t t1 = t0 + per_block < T ? t0 + per_block : T;
  for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int32_t* row = idx + t * k;
    int32_t first = 0;
    for (int j = 0; j < k; ++j) {
      const int32_t e = row[j];
      if (j == 0) first = e;
      if (e >= 0 && e < E) {
        atomicAdd(&h_slot[j * E + e], 1);
        if (j == 1 && n_pair && first >= 0 && first < E) atomicAdd(&h_pair[first * E + e], 1);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_slot; i += blockDim.x)
    if (h_slot[i]) atomicAdd(&slot_counts[i], h_slot[i]);
  for (int i = threadIdx.x; i < n_pair; i += blockDim.x)
    if (h_pair[i]) atomicAdd(&pair_counts[i], h_pair[i]);
}

}  // namespace

cudaError_t launch_router_stats(const int32_t* idx, int64_t T, int32_t E, int32_t k, int32_t* slot_counts,
                                int32_t* pair_counts, bool accumulate, int num_sms, cudaStream_t s) {
  if (!accumulate) {
    cudaError_t err = cudaMemsetAsync(slot_counts, 0, sizeof(int32_t) * k * E, s);
    if (err == cudaSuccess && pair_counts) err = cudaMemsetAsync(pair_counts, 0, sizeof(int32_t) * E * E, s);
    if (err != cudaSuccess) return err;
  }
  if (T == 0) return cudaSuccess;
  // enough tokens per block that the per-block flush stays small against the counting
  int64_t blocks = (T + 4 * kStatsThreads - 1) / (4 * kStatsThreads);
  if (blocks > 2 * num_sms) blocks = 2 * num_sms;
  if (blocks < 1) blocks = 1;
  router_stats_kernel<<<(unsigned)blocks, kStatsThreads, 0, s>>>(idx, T, E, k, slot_counts,
                                                                  k >= 2 ? pair_counts : nullptr);
  return cudaGetLastError();
}

}  // namespace moe
