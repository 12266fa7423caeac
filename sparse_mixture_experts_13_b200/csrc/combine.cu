// Gate-weighted combine (un-permute).
//
// Source: "Mixtral and Mixture-of-Experts, Explained", section "How it works"
// (y = sum_i G(x)_i . Expert_i(x)), and "How Mixtral 8x7B uses mixture of
// experts", section "The architecture in one diagram" (out += weight *
// expert_out, scattered back to the tokens).
//
//   y[t] = sum over kept slots j of t (slot_pos >= 0) of w[t, j] * o_j
//
// where o_j is the expert output row slot_pos[t*k+j] of y_perm (bf16), or the
// sum in split order of the fp32 split-K partials of that row.  fp32
// accumulation in slot order, one bf16 rounding at the end; no atomics, so
// the result is bit-reproducible.
#include <cstdint>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8_unpack(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per (token, chunk of 32 * CPL columns); lane l owns CPL
// consecutive columns.  The launch picks CPL = 16 for bf16 rows of y_perm and
// CPL = 4 for fp32 split-K partials.  From bf16 rows every row load of a lane is
// issued before the sums; from partials (narrow chunks, so that more warps
// share a token) up to 8 splits of every slot are in flight at once.
template <int CPL, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  constexpr int kCols = 32 * CPL;
  constexpr int NV = CPL / 8;  // 16-byte bf16 vectors per lane
  pdl_wait();  // the expert GEMMs' outputs (and, through them, the router's)
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int chunks = (a.d + kCols - 1) / kCols;
  const int64_t items = a.T * chunks;
  for (int64_t it = warp_global; it < items; it += nwarps) {
    const int64_t t = it / chunks;
    const int col = (int)(it % chunks) * kCols + lane * CPL;
    if (col >= a.d) continue;
    int32_t pos[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      pos[j] = -1;
      w[j] = 0.f;
      if (j < a.k) {
        pos[j] = a.slot_pos[t * a.k + j];
        w[j] = a.topk_w[t * a.k + j];
        if (pos[j] >= 0 && !MOE_DCHECK(a.status, pos[j] < a.T * a.k)) pos[j] = -1;
      }
    }
    float acc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
    if constexpr (CPL >= 8) {  // bf16 rows of y_perm
      uint4 raw[KMAX][NV];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (pos[j] >= 0) {
          const uint4* src = reinterpret_cast<const uint4*>(a.y_perm + (int64_t)pos[j] * a.d + col);
#pragma unroll
          for (int h = 0; h < NV; ++h) raw[j][h] = src[h];
        }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (pos[j] < 0) continue;
        float o[8];
#pragma unroll
        for (int h = 0; h < NV; ++h) {
          bf16x8_unpack(raw[j][h], o);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[8 * h + i] = fmaf(w[j], o[i], acc[8 * h + i]);
        }
      }
    } else {
      // Every slot's splits are loaded before any is added (SPR splits per
      // round), so the loads of a token overlap; each slot's splits are still
      // summed in split order.
      constexpr int SPR = KMAX <= 2 ? 8 : 2;
      constexpr int NQ = CPL / 4;
      float o[KMAX][CPL];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[j][i] = 0.f;
      for (int sp0 = 0; sp0 < a.splits; sp0 += SPR) {
        float4 qv[KMAX][SPR][NQ];
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
#pragma unroll
          for (int u = 0; u < SPR; ++u)
#pragma unroll
            for (int c = 0; c < NQ; ++c) {
              qv[j][u][c] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (pos[j] >= 0 && sp0 + u < a.splits)
                qv[j][u][c] = reinterpret_cast<const float4*>(a.partials + (int64_t)(sp0 + u) * a.part_stride +
                                                              (int64_t)pos[j] * a.d + col)[c];
            }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
#pragma unroll
          for (int u = 0; u < SPR; ++u)
            if (sp0 + u < a.splits) {
#pragma unroll
              for (int c = 0; c < NQ; ++c) {
                o[j][4 * c] += qv[j][u][c].x;
                o[j][4 * c + 1] += qv[j][u][c].y;
                o[j][4 * c + 2] += qv[j][u][c].z;
                o[j][4 * c + 3] += qv[j][u][c].w;
              }
            }
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (pos[j] >= 0) {
#pragma unroll
          for (int i = 0; i < CPL; ++i) acc[i] = fmaf(w[j], o[j][i], acc[i]);
        }
    }
    if constexpr (CPL >= 8) {
      uint4* dst = reinterpret_cast<uint4*>(a.y + t * a.d + col);
#pragma unroll
      for (int h = 0; h < NV; ++h)
        dst[h] = make_uint4(pack_bf16x2(acc[8 * h], acc[8 * h + 1]), pack_bf16x2(acc[8 * h + 2], acc[8 * h + 3]),
                            pack_bf16x2(acc[8 * h + 4], acc[8 * h + 5]), pack_bf16x2(acc[8 * h + 6], acc[8 * h + 7]));
    } else {
      *reinterpret_cast<uint2*>(a.y + t * a.d + col) =
          make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
    }
  }
}

cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s) {
  const int cpl = a.y_perm ? 16 : 4;
  const int64_t warps_needed = a.T * ((a.d + 32 * cpl - 1) / (32 * cpl));
  int64_t blocks = (warps_needed + 7) / 8;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const dim3 g((unsigned)blocks), b(256);
  if (a.k <= 2) {
    if (cpl == 16) return launch_k(combine_kernel<16, 2>, g, b, 0, s, a.pdl, a);
    return launch_k(combine_kernel<4, 2>, g, b, 0, s, a.pdl, a);
  }
  if (cpl == 16) return launch_k(combine_kernel<16, 8>, g, b, 0, s, a.pdl, a);
  return launch_k(combine_kernel<4, 8>, g, b, 0, s, a.pdl, a);
}

// y_perm[r] = bf16(sum over splits of partials[sp][r]) for rows r < offsets[E].
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partials, int32_t splits,
                                                            int64_t part_stride, const int32_t* __restrict__ offsets,
                                                            int32_t E, uint16_t* __restrict__ y_perm, int32_t d,
                                                            int64_t S, uint32_t* status) {
  int64_t rows = offsets[E];
  if (!MOE_DCHECK(status, rows >= 0 && rows <= S)) rows = 0;
  const int nvec = d >> 3;
  const int64_t total = rows * nvec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nvec;
    const int v = (int)(i % nvec);
    float o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = 0.f;
    for (int sp = 0; sp < splits; ++sp) {
      const float4* src = reinterpret_cast<const float4*>(partials + sp * part_stride + r * d) + 2 * v;
      const float4 p0 = __ldg(src), p1 = __ldg(src + 1);
      o[0] += p0.x; o[1] += p0.y; o[2] += p0.z; o[3] += p0.w;
      o[4] += p1.x; o[5] += p1.y; o[6] += p1.z; o[7] += p1.w;
    }
    reinterpret_cast<uint4*>(y_perm + r * d)[v] =
        make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
  }
}

cudaError_t launch_splitk_reduce(const float* partials, int32_t splits, int64_t part_stride, const int32_t* offsets,
                                 int32_t E, uint16_t* y_perm, int64_t S, int32_t d, int num_sms, cudaStream_t s,
                                 uint32_t* status) {
  int64_t blocks = (S * (d / 8) + 255) / 256;
  const int64_t cap = (int64_t)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  splitk_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(partials, splits, part_stride, offsets, E, y_perm, d, S,
                                                         status);
  return cudaGetLastError();
}

}  // namespace moe
