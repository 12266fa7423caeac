// Expert parallelism: the experts of the layer are split over `world` ranks
// (one process per GPU), rank o owning experts o*epr .. o*epr + epr - 1.
//
// Source: "How Mixtral 8x7B uses mixture of experts", sections "Tensor
// parallelism vs expert parallelism" (the experts are divided among the GPUs;
// an all-to-all at the MoE layer sends the tokens to the ranks that own
// their experts, a second one sends the results back; expert_parallel_forward:
// router, dispatch, local experts, combine) and "Capacity factor tuning"
// (with expert parallelism, uneven routing loads some GPUs more than others).
//
// The two all-to-all steps are fused into the kernels on either side of
// them, over peer memory:
//   ep_plan_kernel      from the all-gathered routed counts C[r][e] of every
//                       rank: where this rank's slots of expert e start in
//                       the owner's receive buffer, and the row ranges of
//                       this rank's own experts;
//   ep_dispatch_kernel  the grouping step with a remote destination: each
//                       slot's token row is stored straight into the owner's
//                       receive buffer (16-byte stores through the owner's
//                       buffer pointer), and the row is kept for the return;
//   ep_combine_kernel   the gate-weighted combine reading each slot's result
//                       row from its owner's output buffer.
// An owner's receive buffer holds its experts' rows expert by expert, and
// within an expert the source ranks in rank order, each in token order, so
// the owner runs the ordinary grouped GEMMs on it.
//
// With a capacity ("Routing without auxiliary loss": each expert keeps at
// most cf x (tokens x k / E) slots), the ranks' tokens are one batch, their
// concatenation in rank order, so the capacity counts every rank's slots of
// an expert and only the owner sees them all:
//   ep_dispatch_kernel  also stores each slot's 64-bit priority key beside
//                       its row (full-softmax probability, then the smaller
//                       index in the concatenated batch);
//   ep_select_kernel    on the owner, one block per local expert: keeps the
//                       cap rows of largest key (by probability) or the
//                       first cap rows, which are the first in token order
//                       (by order), and writes row_map (kept row or -1) and
//                       the kept offsets;
//   ep_compact_kernel   gathers the kept rows for the owner's GEMMs;
//   ep_combine_kernel   follows the owner's row_map; a dropped slot adds 0.  Between dispatch, expert
// GEMMs and combine the ranks must synchronise (the caller's barrier); the
// kernels themselves never wait on another rank.  No TMA is used on peer
// memory.
#include <cstdint>

#include "moe_internal.h"
#include "select.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

// One block: recv_off[e] = start row of this rank's slots of expert e in the
// buffer of e's owner; owner_off[l] = start row of local expert l (l = 0 ..
// epr) in this rank's receive buffer.
__global__ void ep_plan_kernel(const int32_t* __restrict__ counts_all, int32_t E, int32_t rank, int32_t world,
                               int32_t* __restrict__ recv_off, int32_t* __restrict__ owner_off) {
  const int epr = E / world;
  if (threadIdx.x == 0) {
    // rows of each owner's buffer, expert by expert, source ranks in order
    for (int o = 0; o < world; ++o) {
      int32_t row = 0;
      for (int l = 0; l < epr; ++l) {
        const int e = o * epr + l;
        if (o == rank) owner_off[l] = row;
        for (int r = 0; r < world; ++r) {
          if (r == rank) recv_off[e] = row;
          row += counts_all[r * E + e];
        }
      }
      if (o == rank) owner_off[epr] = row;
    }
  }
}

// One warp per slot of this rank: copy the token's row to its owner.
// Priority key of a slot: probability bits, then the smaller token index
// (the same order as the single-device capacity selection).
__device__ __forceinline__ uint64_t ep_slot_key(float p, int64_t t) {
  return ((uint64_t)__float_as_uint(p) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
}

// Tokens of the ranks below `rank` (each token has k slots in the counts).
__device__ __forceinline__ int64_t ep_tokens_before(const int32_t* counts_all, int32_t E, int32_t k, int32_t rank) {
  int64_t n = 0;
  for (int r = 0; r < rank; ++r)
    for (int e = 0; e < E; ++e) n += counts_all[r * E + e];
  return n / k;
}

// One warp per slot of this rank: copy the token's row to its owner (and,
// with peer_keys, the slot's priority key to the same row of the owner's
// key buffer).
__global__ void __launch_bounds__(256) ep_dispatch_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ topk_idx,
                                                          const int32_t* __restrict__ offsets,
                                                          const int32_t* __restrict__ slot_pos,
                                                          const int32_t* __restrict__ recv_off,
                                                          uint16_t* const* __restrict__ peer_x, int32_t* ret_row,
                                                          int64_t S, int32_t k, int32_t d, int32_t epr,
                                                          const float* __restrict__ topk_p,
                                                          const int32_t* __restrict__ counts_all, int32_t E,
                                                          int32_t rank, uint64_t* const* __restrict__ peer_keys) {
  __shared__ int64_t s_tbase;
  if (threadIdx.x == 0) s_tbase = peer_keys ? ep_tokens_before(counts_all, E, k, rank) : 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nvec = d >> 3;
  for (int64_t s = w0; s < S; s += nw) {
    const int32_t e = topk_idx[s];
    const int32_t row = recv_off[e] + (slot_pos[s] - offsets[e]);
    if (lane == 0) {
      ret_row[s] = row;
      if (peer_keys) peer_keys[e / epr][row] = ep_slot_key(topk_p[s], s_tbase + s / k);
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (s / k) * (int64_t)d);
    uint4* dst = reinterpret_cast<uint4*>(peer_x[e / epr] + (int64_t)row * d);
    for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
  }
  // the rows may live on another GPU: make them visible system-wide before
  // the kernel ends (the caller's barrier then orders the owner's reads)
  __threadfence_system();
}

// One warp per (token, 256 columns): y[t] = sum_j w[t, j] * out_o[row(t, j)],
// fp32 in slot order, one bf16 rounding.
__global__ void __launch_bounds__(256) ep_combine_kernel(const int32_t* __restrict__ topk_idx,
                                                         const float* __restrict__ topk_w,
                                                         const int32_t* __restrict__ ret_row,
                                                         const uint16_t* const* __restrict__ peer_y,
                                                         uint16_t* __restrict__ y, int64_t T, int32_t k, int32_t d,
                                                         int32_t epr, const int32_t* const* __restrict__ peer_map) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int chunks = (d + 255) / 256;
  for (int64_t it = w0; it < T * chunks; it += nw) {
    const int64_t t = it / chunks;
    const int col = (int)(it % chunks) * 256 + lane * 8;
    if (col >= d) continue;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t s = t * k + j;
      const int32_t e = topk_idx[s];
      const float w = topk_w[s];
      int32_t row = ret_row[s];
      if (peer_map) row = peer_map[e / epr][row];  // kept row on the owner, or -1: dropped
      if (row < 0) continue;
      const uint4 v = *reinterpret_cast<const uint4*>(peer_y[e / epr] + (int64_t)row * d + col);
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(q[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(q[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + t * (int64_t)d + col) = o;
  }
}

// Owner side, one block per local expert l (rows lo .. hi-1 of the receive
// buffer): cap = floor(cf * T_all * k / E) over all ranks' tokens T_all;
// kept rows are numbered in row order after the kept rows of the lower
// local experts.
__global__ void __launch_bounds__(kSelectThreads) ep_select_kernel(const int32_t* __restrict__ counts_all,
                                                                   int32_t world, int32_t E, int32_t k, float cf,
                                                                   int32_t policy, const int32_t* __restrict__ owner_off,
                                                                   const uint64_t* __restrict__ keys, int32_t epr,
                                                                   int32_t* __restrict__ kept_off,
                                                                   int32_t* __restrict__ row_map) {
  __shared__ int64_t s_cap;
  __shared__ int32_t s_base;
  __shared__ int32_t s_warp[kSelectThreads / 32];
  __shared__ int32_t s_run;
  const int l = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t lo = owner_off[l], hi = owner_off[l + 1];
  const int64_t M = hi - lo;
  if (tid == 0) {
    const int64_t slots = ep_tokens_before(counts_all, E, 1, world);  // every rank's slots
    const int64_t T_all = slots / k;
    const int64_t cap = (int64_t)floor((double)cf * (double)T_all * (double)k / (double)E);
    int32_t base = 0;
    for (int j = 0; j < l; ++j) base += (int32_t)min((int64_t)(owner_off[j + 1] - owner_off[j]), cap);
    s_cap = cap;
    s_base = base;
    s_run = 0;
    kept_off[l] = base;
    if (l == epr - 1) kept_off[epr] = base + (int32_t)min(M, cap);
  }
  __syncthreads();
  const int64_t cap = s_cap;
  uint64_t thr = 0;  // by probability: keep keys >= thr
  if (policy == 0 && M > cap)
    thr = cap == 0 ? ~0ull
                   : block_radix_select(
                         [&](int64_t i, uint64_t& key) {
                           key = keys[lo + i];
                           return true;
                         },
                         M, M, cap);
  // number the kept rows in row order: a block-wide scan per chunk
  for (int64_t c0 = 0; c0 < M; c0 += blockDim.x) {
    const int64_t i = c0 + tid;
    bool kept = false;
    if (i < M) kept = policy == 0 ? (M <= cap || keys[lo + i] >= thr) : i < cap;
    const uint32_t ballot = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) s_warp[warp] = __popc(ballot);
    __syncthreads();
    int32_t before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    const int32_t rank = s_run + before + __popc(ballot & ((1u << lane) - 1u));
    if (i < M) row_map[lo + i] = kept ? s_base + rank : -1;
    __syncthreads();
    if (tid == 0) {
      int32_t n = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) n += s_warp[w];
      s_run += n;
    }
    __syncthreads();
  }
}

// One warp per received row: the kept rows into the compacted buffer.
__global__ void __launch_bounds__(256) ep_compact_kernel(const uint16_t* __restrict__ x_recv,
                                                         const int32_t* __restrict__ row_map,
                                                         const int32_t* __restrict__ owner_off, int32_t epr,
                                                         uint16_t* __restrict__ x_kept, int32_t d) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t rows = owner_off[epr];
  const int nvec = d >> 3;
  for (int64_t r = w0; r < rows; r += nw) {
    const int32_t to = row_map[r];
    if (to < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x_recv + r * (int64_t)d);
    uint4* dst = reinterpret_cast<uint4*>(x_kept + (int64_t)to * d);
    for (int v = lane; v < nvec; v += 32) dst[v] = src[v];
  }
}

unsigned warps_grid(int64_t items, int num_sms) {
  int64_t b = (items + 7) / 8;  // 8 warps per block
  if (b > 8 * num_sms) b = 8 * num_sms;
  return (unsigned)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_ep_plan(const int32_t* counts_all, int32_t E, int32_t rank, int32_t world, int32_t* recv_off,
                           int32_t* owner_off, cudaStream_t s) {
  ep_plan_kernel<<<1, 32, 0, s>>>(counts_all, E, rank, world, recv_off, owner_off);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const int32_t* offsets,
                               const int32_t* slot_pos, const int32_t* recv_off, uint16_t* const* peer_x,
                               int32_t* ret_row, int64_t S, int32_t k, int32_t d, int32_t epr, int num_sms,
                               cudaStream_t s, const EpKeys* keys) {
  ep_dispatch_kernel<<<warps_grid(S, num_sms), 256, 0, s>>>(
      x, topk_idx, offsets, slot_pos, recv_off, peer_x, ret_row, S, k, d, epr, keys ? keys->topk_p : nullptr,
      keys ? keys->counts_all : nullptr, keys ? keys->E : 0, keys ? keys->rank : 0, keys ? keys->peer_keys : nullptr);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const int32_t* topk_idx, const float* topk_w, const int32_t* ret_row,
                              const uint16_t* const* peer_y, uint16_t* y, int64_t T, int32_t k, int32_t d, int32_t epr,
                              int num_sms, cudaStream_t s, const int32_t* const* peer_map) {
  ep_combine_kernel<<<warps_grid(T * ((d + 255) / 256), num_sms), 256, 0, s>>>(topk_idx, topk_w, ret_row, peer_y, y, T,
                                                                                k, d, epr, peer_map);
  return cudaGetLastError();
}

cudaError_t launch_ep_select(const int32_t* counts_all, int32_t world, int32_t E, int32_t k, float cf, int32_t policy,
                             const int32_t* owner_off, const uint64_t* keys, int32_t epr, int32_t* kept_off,
                             int32_t* row_map, const uint16_t* x_recv, uint16_t* x_kept, int32_t d, int num_sms,
                             cudaStream_t s) {
  cudaError_t err = cudaFuncSetAttribute(ep_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (err != cudaSuccess) return err;
  ep_select_kernel<<<epr, kSelectThreads, kSelectSmem, s>>>(counts_all, world, E, k, cf, policy, owner_off, keys, epr,
                                                            kept_off, row_map);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  ep_compact_kernel<<<8 * num_sms, 256, 0, s>>>(x_recv, row_map, owner_off, epr, x_kept, d);
  return cudaGetLastError();
}

}  // namespace moe
