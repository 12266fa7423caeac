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
// the owner runs the ordinary grouped GEMMs on it.  Between dispatch, expert
// GEMMs and combine the ranks must synchronise (the caller's barrier); the
// kernels themselves never wait on another rank.  No TMA is used on peer
// memory.
#include <cstdint>

#include "moe_internal.h"
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
__global__ void __launch_bounds__(256) ep_dispatch_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ topk_idx,
                                                          const int32_t* __restrict__ offsets,
                                                          const int32_t* __restrict__ slot_pos,
                                                          const int32_t* __restrict__ recv_off,
                                                          uint16_t* const* __restrict__ peer_x, int32_t* ret_row,
                                                          int64_t S, int32_t k, int32_t d, int32_t epr) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nvec = d >> 3;
  for (int64_t s = w0; s < S; s += nw) {
    const int32_t e = topk_idx[s];
    const int32_t row = recv_off[e] + (slot_pos[s] - offsets[e]);
    if (lane == 0) ret_row[s] = row;
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
                                                         int32_t epr) {
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
      const uint4 v = *reinterpret_cast<const uint4*>(peer_y[e / epr] + (int64_t)ret_row[s] * d + col);
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
                               cudaStream_t s) {
  ep_dispatch_kernel<<<warps_grid(S, num_sms), 256, 0, s>>>(x, topk_idx, offsets, slot_pos, recv_off, peer_x, ret_row,
                                                             S, k, d, epr);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const int32_t* topk_idx, const float* topk_w, const int32_t* ret_row,
                              const uint16_t* const* peer_y, uint16_t* y, int64_t T, int32_t k, int32_t d, int32_t epr,
                              int num_sms, cudaStream_t s) {
  ep_combine_kernel<<<warps_grid(T * ((d + 255) / 256), num_sms), 256, 0, s>>>(topk_idx, topk_w, ret_row, peer_y, y, T,
                                                                                k, d, epr);
  return cudaGetLastError();
}

}  // namespace moe
