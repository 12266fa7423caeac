// Block-wide selection of the r-th largest 64-bit key, shared by the capacity
// pass (drop by probability) and the next-best-expert fallback.
#pragma once
#include <cstdint>

namespace moe {

constexpr int kSelectThreads = 1024;
// Keys of one expert cached in dynamic shared memory (16384 x 8 bytes); an
// expert with more slots is scanned in global memory on every pass.
constexpr int kSelectCache = 16384;
constexpr int kSelectSmem = kSelectCache * 8;

// MSB-first radix select over 8 passes of 8 bits: returns the `need`-th
// largest key among the slots s in [0, S) for which key_of(s, key) is true
// (need >= 1, and at least `need` such slots; `count` is their number).
// Keys must be distinct, so exactly `need` keys are >= the result.  Every
// thread of the block must call it, with kSelectSmem bytes of dynamic shared
// memory.  The keys are first compacted into shared memory when they fit, so
// the passes read no global memory.  Histogram updates are aggregated per
// warp (one shared-memory atomic per distinct bin and warp), since the keys
// of one expert share their leading bytes and would otherwise pile onto a
// single bin.
template <class KeyOf>
__device__ __forceinline__ uint64_t block_radix_select(KeyOf key_of, int64_t S, int64_t count, int64_t need) {
  extern __shared__ uint64_t s_keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint64_t s_prefix;
  __shared__ int64_t s_need;
  __shared__ uint32_t s_n;
  const int lane = threadIdx.x & 31;
  const bool cached = count <= kSelectCache;
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_need = need;
    s_n = 0;
  }
  __syncthreads();
  if (cached) {
    for (int64_t base = threadIdx.x - lane; base < S; base += blockDim.x) {
      const int64_t s = base + lane;
      uint64_t key = 0;
      const bool mine = s < S && key_of(s, key);
      const uint32_t ballot = __ballot_sync(0xffffffffu, mine);
      uint32_t pos = 0;
      if (lane == 0 && ballot) pos = atomicAdd(&s_n, (uint32_t)__popc(ballot));
      pos = __shfl_sync(0xffffffffu, pos, 0);
      if (mine) {
        const uint32_t at = pos + __popc(ballot & ((1u << lane) - 1u));
        if (at < (uint32_t)kSelectCache) s_keys[at] = key;
      }
    }
    __syncthreads();
  }
  const int64_t n = cached ? (int64_t)min(s_n, (uint32_t)kSelectCache) : S;
  uint64_t mask = 0;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint64_t prefix = s_prefix;
    // warp-uniform trip count: every lane of a warp runs the same iterations
    for (int64_t base = threadIdx.x - lane; base < n; base += blockDim.x) {
      const int64_t s = base + lane;
      uint64_t key = 0;
      bool mine = false;
      if (s < n) {
        if (cached) {
          key = s_keys[s];
          mine = true;
        } else {
          mine = key_of(s, key);
        }
      }
      mine = mine && (key & mask) == prefix;
      const uint32_t bin = mine ? (uint32_t)((key >> shift) & 0xFF) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (mine && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // the largest bin b whose suffix sum (bins b..255) reaches s_need, or 0:
      // lane l holds bins 8l..8l+7; a suffix scan over the lanes finds the
      // lane, then that lane walks its 8 bins downwards
      uint32_t c[8], loc = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[8 * lane + i];
        loc += c[i];
      }
      uint32_t suf = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += v;
      }
      const int64_t left = s_need;
      const uint32_t ok = __ballot_sync(0xffffffffu, (int64_t)suf >= left);
      const int hi = ok ? 31 - __clz(ok) : 0;
      if (lane == hi) {
        int64_t cum = (int64_t)(suf - loc);  // bins above this lane's eight
        int b = 8 * lane;
        bool found = false;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (!found) {
            if (cum + c[i] >= left || i == 0) {
              found = true;
              b = 8 * lane + i;
            } else {
              cum += c[i];
            }
          }
        }
        s_need = left - cum;
        s_prefix = prefix | ((uint64_t)b << shift);
      }
    }
    mask |= 0xFFull << shift;
    __syncthreads();
  }
  return s_prefix;
}

}  // namespace moe
