// Capacity selection and grouping of slots by expert.
//
// Source: "How Mixtral 8x7B uses mixture of experts", sections "The
// architecture in one diagram" (group the tokens by expert, run each expert
// on its group, return the results to the tokens) and "Routing without
// auxiliary loss" (capacity factor; the excess slots of an expert are
// dropped; each expert's slots are ordered by router probability).
//
// capacity_select_kernel (capacity mode, drop by probability): one block per
//   expert finds, by an 8-pass MSB-first radix select (select.cuh) over 64-bit keys
//   key = (bits of p as float) << 32 | (0xFFFFFFFF - t),
//   the cap-th largest key of the expert's slots.  Keys are unique (a token
//   routes to an expert at most once), so exactly cap slots satisfy
//   key >= threshold.  Experts with at most cap slots get threshold 0.
//   A slot whose expert is negative was dropped before grouping (the
//   next-best-expert fallback marks slots so) and is skipped.
//
// permute_kernel: a single-pass scan with decoupled look-back.  Each block
//   takes a tile of kPermuteTile consecutive slots in ticket order, ranks its
//   eligible slots per expert (warp match + popc, then across warps), publishes
//   the tile's per-expert aggregate, and one thread per expert walks back over
//   the predecessors' published words (flag in the top 2 bits: 1 = aggregate,
//   2 = inclusive prefix) until it meets an inclusive prefix.  The row of a
//   kept slot is offsets[e] + (eligible slots of e before it).  All of the
//   block's warps then copy the kept tokens' rows of x into x_perm with
//   16-byte vector loads and stores -- except when launch_permute runs the
//   row copy as gather_rows_kernel (a warp per row over every SM), which it
//   does for the look-back path: same rows, 3-13 us per step less at T =
//   4096-8192.
#include <cstdint>

#include "moe_internal.h"
#include "select.cuh"
#include "sm100.cuh"

namespace moe {

constexpr int kPermuteThreads = 512;
constexpr int kPermuteWarpsSlots = kPermuteTile / 32;  // warps that rank slots
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagIncl = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;

int64_t permute_tiles(int64_t S) { return (S + kPermuteTile - 1) / kPermuteTile; }

__device__ __forceinline__ uint64_t slot_key(float p, int64_t t) {
  return ((uint64_t)__float_as_uint(p) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
}

__global__ void __launch_bounds__(kSelectThreads) capacity_select_kernel(const int32_t* __restrict__ idx,
                                                                         const float* __restrict__ p,
                                                                         const int32_t* __restrict__ counts,
                                                                         uint64_t* __restrict__ thresh,
                                                                         int64_t S, int32_t k, int64_t cap) {
  pdl_trigger();
  pdl_wait();  // the router's outputs
  const int e = blockIdx.x;
  const int64_t cnt = counts[e];
  if (cnt <= cap) {
    if (threadIdx.x == 0) thresh[e] = 0;  // every slot qualifies
    return;
  }
  if (cap == 0) {
    if (threadIdx.x == 0) thresh[e] = ~0ull;  // no key reaches it (keys < 2^63)
    return;
  }
  const uint64_t t = block_radix_select(
      [&](int64_t s, uint64_t& key) {
        if (idx[s] != e) return false;
        key = slot_key(p[s], s / k);
        return true;
      },
      S, cnt, cap);
  if (threadIdx.x == 0) thresh[e] = t;
}

__global__ void __launch_bounds__(kPermuteThreads) permute_kernel(PermuteArgs a) {
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_wcnt[kPermuteWarpsSlots][32];
  __shared__ int32_t s_wpre[kPermuteWarpsSlots][32];
  __shared__ int32_t s_excl[32];
  __shared__ int32_t s_tile;
  __shared__ int32_t s_nkept;
  __shared__ int32_t s_row[kPermuteTile];
  __shared__ int32_t s_tok[kPermuteTile];

  // The expert GEMM that follows may launch at once: before its own wait it
  // only prefetches weights.
  pdl_trigger();
  pdl_wait();  // the router's (or capacity selection's) outputs
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, k = a.k;
  const int64_t S = a.T * k;
  if (tid == 0) {
    s_tile = (int32_t)atomicAdd(a.ticket, 1u);
    s_nkept = 0;
    int32_t acc = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = acc;
      int32_t c = a.counts[e];
      if (a.cap >= 0 && c > a.cap) c = (int32_t)a.cap;
      acc += c;
    }
    s_off[E] = acc;
  }
  if (tid < kPermuteWarpsSlots * 32) s_wcnt[tid >> 5][tid & 31] = 0;
  __syncthreads();
  const int64_t tile = s_tile;
  if (tile == 0 && tid <= E) a.offsets[tid] = s_off[tid];

  // ---- rank eligible slots of this tile per expert
  const bool ranker = tid < kPermuteTile;
  const int64_t s = tile * kPermuteTile + tid;
  int e = -1;
  bool elig = false;
  if (ranker && s < S) {
    e = a.topk_idx[s];
    elig = e >= 0 && MOE_DCHECK(a.status, e < E);  // a negative expert marks a slot dropped before grouping
    if (elig && a.cap >= 0 && a.policy == 0) elig = slot_key(a.topk_p[s], s / k) >= a.thresh[e];
  }
  int rank_w = 0;
  if (ranker) {
    const uint32_t peers = __match_any_sync(0xffffffffu, elig ? e : -1);
    rank_w = __popc(peers & ((1u << lane) - 1u));
    if (elig && rank_w == 0) s_wcnt[warp][e] = __popc(peers);
  }
  __syncthreads();
  if (tid < E) {
    int32_t run = 0;
    for (int w = 0; w < kPermuteWarpsSlots; ++w) {
      s_wpre[w][tid] = run;
      run += s_wcnt[w][tid];
    }
    // ---- decoupled look-back for expert `tid`
    const uint32_t agg = (uint32_t)run;
    uint32_t* words = a.tile_state;
    int32_t excl = 0;
    if (tile == 0) {
      st_release_u32(&words[tid], kFlagIncl | agg);
    } else {
      st_release_u32(&words[tile * E + tid], kFlagAgg | agg);
      int64_t pred = tile - 1;
      bool timed_out = false;
      while (pred >= 0) {
        uint32_t v;
        if (!wait_published(&words[pred * E + tid], ~kValueMask, &v)) {
          timed_out = true;
          break;
        }
        excl += (int32_t)(v & kValueMask);
        if ((v & ~kValueMask) == kFlagIncl) break;
        --pred;
      }
      if (timed_out) record_status(a.status, kStatusTimeout);
      st_release_u32(&words[tile * E + tid], kFlagIncl | ((uint32_t)excl + agg));
    }
    s_excl[tid] = excl;
  }
  __syncthreads();

  // ---- rows of the tile's slots
  if (ranker && s < S) {
    int32_t row = -1;
    if (elig) {
      const int32_t rank = s_excl[e] + s_wpre[warp][e] + rank_w;
      const bool kept = !(a.cap >= 0 && a.policy == 1 && rank >= a.cap);
      if (kept && MOE_DCHECK(a.status, s_off[e] + rank < s_off[e + 1] && s_off[e] + rank < S)) {
        row = s_off[e] + rank;
        a.perm_slot[row] = (int32_t)s;
        const int q = atomicAdd(&s_nkept, 1);
        s_row[q] = row;
        s_tok[q] = (int32_t)(s / k);
      }
    }
    a.slot_pos[s] = row;
  }
  __syncthreads();

  // ---- gather the kept tokens' rows (16-byte vectors, all warps); skipped
  // when only the grouping is wanted (x_perm == nullptr)
  const int nkept = a.x_perm ? s_nkept : 0;
  const int nvec = a.d >> 3;
  const int nwarps = blockDim.x >> 5;
  for (int i = warp; i < nkept; i += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (int64_t)s_tok[i] * a.d);
    uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (int64_t)s_row[i] * a.d);
    int v = lane;
    for (; v + 224 < nvec; v += 256) {
      uint4 r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) r[u] = __ldg(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[v + 32 * u] = r[u];
    }
    for (; v < nvec; v += 32) dst[v] = __ldg(src + v);
  }
}

// Few slots (S <= kSmallSlots): every block ranks all slots itself in shared
// memory -- warp 0 walks them in order, 32 at a time, keeping a running count
// per expert -- so no look-back is needed, and the blocks then share the row
// gather.  Block 0 writes offsets, slot_pos and perm_slot.
constexpr int kSmallSlots = 1024;
constexpr int kSmallBlocks = 64;

__global__ void __launch_bounds__(256) permute_small_kernel(PermuteArgs a) {
  __shared__ int32_t s_off[33];
  __shared__ int32_t s_run[32];
  __shared__ int32_t s_row[kSmallSlots];   // row of slot s, or -1
  __shared__ int32_t s_list[kSmallSlots];  // kept slots in row order
  pdl_trigger();
  pdl_wait();  // the router's (or capacity selection's) outputs
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, k = a.k;
  const int S = (int)(a.T * k);
  if (tid == 0) {
    int32_t acc = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = acc;
      int32_t c = a.counts[e];
      if (a.cap >= 0 && c > a.cap) c = (int32_t)a.cap;
      acc += c;
    }
    s_off[E] = acc;
  }
  if (tid < 32) s_run[tid] = 0;
  __syncthreads();
  if (warp == 0) {
    for (int base = 0; base < S; base += 32) {
      const int s = base + lane;
      int e = -1;
      bool elig = false;
      if (s < S) {
        e = a.topk_idx[s];
        elig = e >= 0 && MOE_DCHECK(a.status, e < E);  // a negative expert marks a slot dropped before grouping
        if (elig && a.cap >= 0 && a.policy == 0) elig = slot_key(a.topk_p[s], s / k) >= a.thresh[e];
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, elig ? e : -1);
      const int before = __popc(peers & ((1u << lane) - 1u));
      int32_t row = -1;
      if (elig) {
        const int32_t rank = s_run[e] + before;
        if (!(a.cap >= 0 && a.policy == 1 && rank >= a.cap) &&
            MOE_DCHECK(a.status, s_off[e] + rank < s_off[e + 1] && s_off[e] + rank < S))
          row = s_off[e] + rank;
      }
      __syncwarp();
      if (elig && before == 0) s_run[e] += __popc(peers);
      if (s < S) {
        s_row[s] = row;
        if (row >= 0) s_list[row] = s;
      }
      __syncwarp();
    }
  }
  __syncthreads();
  const int N = s_off[E];
  if (blockIdx.x == 0) {
    if (tid <= E) a.offsets[tid] = s_off[tid];
    for (int s = tid; s < S; s += blockDim.x) a.slot_pos[s] = s_row[s];
    for (int r = tid; r < N; r += blockDim.x) a.perm_slot[r] = s_list[r];
  }
  const int nvec = a.d >> 3;
  const int nwarps = blockDim.x >> 5;
  const int n_gather = a.x_perm ? N : 0;  // grouping only when x_perm == nullptr
  for (int r = blockIdx.x + gridDim.x * warp; r < n_gather; r += gridDim.x * nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (int64_t)(s_list[r] / k) * a.d);
    uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (int64_t)r * a.d);
    int v = lane;
    for (; v + 224 < nvec; v += 256) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = __ldg(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[v + 32 * u] = q[u];
    }
    for (; v < nvec; v += 32) dst[v] = __ldg(src + v);
  }
}

// Row copy of the grouping with many slots: x_perm[r] = x[perm_slot[r] / k]
// for the grouped rows r < offsets[E], apart from the ranking so that every
// SM copies (the ranking kernel has one block per 64 slots).  A warp copies
// a row with up to 8 KB of loads in flight (16-byte vectors).
constexpr int kGatherThreads = 256;
__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                                     const int32_t* __restrict__ perm_slot,
                                                                     const int32_t* __restrict__ offsets, int32_t E,
                                                                     int32_t k, int32_t d, int64_t T, int64_t S,
                                                                     uint16_t* __restrict__ x_perm, uint32_t* status) {
  pdl_wait();     // the grouping's rows
  pdl_trigger();  // the expert GEMM may start its weight prefetch
  int64_t rows = offsets[E];
  if (!MOE_DCHECK(status, rows >= 0 && rows <= S)) rows = 0;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nvec = d >> 3;
  for (int64_t r = warp; r < rows; r += nwarps) {
    const int64_t tok = perm_slot[r] / k;
    if (!MOE_DCHECK(status, tok >= 0 && tok < T)) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + tok * d);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + r * d);
    for (int v0 = 0; v0 < nvec; v0 += 512) {
      uint4 q[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < nvec) q[u] = __ldg(src + v);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < nvec) dst[v] = q[u];
      }
    }
  }
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s, bool state_zeroed) {
  const int64_t S = a.T * a.k;
  const int64_t tiles = permute_tiles(S);
  cudaError_t err = cudaSuccess;
  if (!state_zeroed && S > kSmallSlots) {
    err = cudaMemsetAsync(a.tile_state, 0, sizeof(uint32_t) * tiles * a.E, s);
    if (err != cudaSuccess) return err;
    err = cudaMemsetAsync(a.ticket, 0, sizeof(uint32_t), s);
    if (err != cudaSuccess) return err;
  }
  if (a.cap >= 0 && a.policy == 0) {
    err = cudaFuncSetAttribute(capacity_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
    if (err != cudaSuccess) return err;
    err = launch_k(capacity_select_kernel, dim3(a.E), dim3(kSelectThreads), kSelectSmem, s, a.pdl, a.topk_idx,
                   a.topk_p, a.counts, a.thresh, S, a.k, a.cap);
    if (err != cudaSuccess) return err;
  }
  if (S <= kSmallSlots) {
    const int blocks = (int)(S < kSmallBlocks ? S : kSmallBlocks);
    return launch_k(permute_small_kernel, dim3(blocks), dim3(256), 0, s, a.pdl, a);
  }
  // ranking and rows; the row copy follows as its own kernel
  PermuteArgs rank_only = a;
  rank_only.x_perm = nullptr;
  err = launch_k(permute_kernel, dim3((unsigned)tiles), dim3(kPermuteThreads), 0, s, a.pdl, rank_only);
  if (err != cudaSuccess || !a.x_perm) return err;
  // a warp per row, up to 1024 blocks (grid-stride beyond)
  int64_t blocks = (S + (kGatherThreads / 32) - 1) / (kGatherThreads / 32);
  if (blocks > 1024) blocks = 1024;
  return launch_k(gather_rows_kernel, dim3((unsigned)blocks), dim3(kGatherThreads), 0, s, a.pdl, a.x, a.perm_slot,
                  a.offsets, a.E, a.k, a.d, a.T, S, a.x_perm, a.status);
}

// ---------------------------------------------------------------------------
// Fixed scratch for moe_permute_noalloc (callers that cannot allocate device
// memory).  Layout: [0, 256) status word and tile ticket; [256, 512) capacity
// thresholds of up to 32 experts; then the look-back words of up to
// kNoAllocMaxSlots / kPermuteTile tiles x 32 experts.  In host code the
// symbol is only a stand-in, never a device address: the address is looked up
// once per device with cudaGetSymbolAddress and passed to the kernels.
constexpr int64_t kNoAllocMaxSlots = 65536;
constexpr size_t kNoAllocHeader = 512;
constexpr size_t kNoAllocBytes = kNoAllocHeader + sizeof(uint32_t) * (kNoAllocMaxSlots / kPermuteTile) * 32;
static __device__ __align__(256) unsigned char g_permute_scratch[kNoAllocBytes];

namespace {
void* g_scratch_addr[kMaxDevices];  // device address per device, once looked up
}  // namespace

}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_shape* sh, const moe_bf16* x, const int32_t* topk_idx,
                                          const float* topk_p, const int32_t* counts, int32_t* offsets,
                                          int32_t* slot_pos, int32_t* perm_slot, moe_bf16* x_perm,
                                          moe_stream_t stream) {
  using namespace moe;
  moe_status st = api_check_shape(sh);
  if (st != MOE_OK) return st;
  if (sh->T == 0) return MOE_OK;
  const int64_t S = sh->T * sh->k;
  if (S > kNoAllocMaxSlots) return MOE_ERR_UNSUPPORTED;
  auto al = [](const void* p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!al(x, 16) || !al(x_perm, 16) || !al(topk_idx, 4) || !al(counts, 4) || !al(offsets, 4) || !al(slot_pos, 4) ||
      !al(perm_slot, 4))
    return MOE_ERR_INVALID_ARG;
  const int64_t cap = api_capacity(sh);
  if (cap >= 0 && sh->drop_policy == MOE_DROP_BY_PROB && !al(topk_p, 4)) return MOE_ERR_INVALID_ARG;
  if (cap >= 0 && sh->drop_policy >= MOE_DROP_BY_PROB_NEXT_BEST) return MOE_ERR_UNSUPPORTED;
  int sms = 0;
  st = api_check_device(&sms);
  if (st != MOE_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;  // as api_check_device
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_permute_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  unsigned char* base = static_cast<unsigned char*>(g_scratch_addr[dev]);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t words = (size_t)permute_tiles(S) * sh->E;
  // status word, ticket and the look-back words this call uses start at zero
  if (cudaMemsetAsync(base, 0, 8, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(base + kNoAllocHeader, 0, sizeof(uint32_t) * words, s) != cudaSuccess) return MOE_ERR_CUDA;
  PermuteArgs a{};
  a.x = x;
  a.topk_idx = topk_idx;
  a.topk_p = topk_p;
  a.counts = counts;
  a.offsets = offsets;
  a.slot_pos = slot_pos;
  a.perm_slot = perm_slot;
  a.x_perm = x_perm;
  a.status = reinterpret_cast<uint32_t*>(base);
  a.ticket = reinterpret_cast<uint32_t*>(base + 4);
  a.thresh = reinterpret_cast<uint64_t*>(base + 256);
  a.tile_state = reinterpret_cast<uint32_t*>(base + kNoAllocHeader);
  a.T = sh->T;
  a.d = sh->d_model;
  a.E = sh->E;
  a.k = sh->k;
  a.cap = cap;
  a.policy = sh->drop_policy;
  return launch_permute(a, s, true) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_permute_noalloc_status(moe_stream_t stream) {
  using namespace moe;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (!g_scratch_addr[dev]) return MOE_OK;  // no call on this device yet
  uint32_t v = 0;
  if (cudaMemcpy(&v, g_scratch_addr[dev], sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  return v == 0 ? MOE_OK : (moe_status)v;
}
