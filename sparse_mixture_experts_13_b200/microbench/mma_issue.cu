// Issue cost of tcgen05.mma at the small N of the decode GEMMs.
//
// One CTA of 16 warps on one SM.  Thread 0 (warp 0, scheduler 0) issues
// `iters` MMAs back to back into one accumulator (M = 128 rows, N token
// columns), with a tcgen05.commit after every `commit_every` of them (to one
// mbarrier, or to a ring of four), and reads clock64 before and after issuing
// and once the last commit has arrived.  Optional busy warps run a fused
// multiply-add loop meanwhile: `busy` of them on each scheduler whose bit is
// set in `smsp_mask` (warp w runs on scheduler w % 4).
//
// Kinds: 0 = kind::f16 with bf16 A and B (K = 16 per instruction),
//        1 = kind::i8 with signed 8-bit A and B (K = 32 per instruction).
// A from shared memory (128-byte swizzle, K-major) or from tensor memory.
// The operands are zero; the accumulator is int32 or fp32.
//
//   mma_issue [iters]   prints one JSON line per configuration
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <cuda_runtime.h>

#include "sm100.cuh"

using namespace moe;

namespace {

__host__ __device__ constexpr uint32_t idesc_s8(int M, int N) {
  return (2u << 4)                       // D format: s32
         | (1u << 7)                     // A: signed 8-bit
         | (1u << 10)                    // B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_i8_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_i8_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_st_zero8(uint32_t taddr) {
  const uint32_t z = 0;
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(z)
               : "memory");
}

constexpr int kThreads = 512;
constexpr int kSmemA = 128 * 128;  // 128 rows x 128 bytes
constexpr int kSmemB = 256 * 128;  // up to 256 rows x 128 bytes
constexpr uint32_t kACol = 256;    // A operand columns in tensor memory (8 used)
constexpr long long kBusyMax = 1ll << 22;

struct Result {
  long long issue, total;
  unsigned status, busy_iters;
};

template <int KIND, bool A_TMEM>
__global__ void __launch_bounds__(kThreads, 1) issue_kernel(int n, int iters, int commit_every, int busy,
                                                             int smsp_mask, int ring, Result* out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t bars[4];
  __shared__ uint64_t fin;  // warm-up and final drain only: exactly two phases
  __shared__ uint32_t tbase_s;
  __shared__ volatile int done;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint8_t* sa = smem;
  uint8_t* sb = smem + kSmemA;
  for (int i = tid; i < (kSmemA + kSmemB) / 16; i += kThreads) reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&bars[b], 1);
    mbar_init(&fin, 1);
    fence_barrier_init();
    done = 0;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(&tbase_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tbase_s;
  if (A_TMEM && warp < 4) {
    tmem_st_zero8(tbase + ((uint32_t)(warp * 32) << 16) + kACol);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    const uint32_t idesc = KIND == 0 ? make_idesc_bf16(128, n) : idesc_s8(128, n);
    const uint64_t ad = make_sdesc_sw128(smem_u32(sa)), bd = make_sdesc_sw128(smem_u32(sb));
    uint32_t commits = 0;
    auto one = [&](int i) {
      const uint64_t koff = (uint64_t)((i & 3) * 2);  // 32-byte K step inside the 128-byte row
      const uint32_t acc = i > 0;
      if (KIND == 0) {
        if (A_TMEM) mma_f16_ts(tbase, tbase + kACol, bd + koff, idesc, acc);
        else umma_bf16(tbase, ad + koff, bd + koff, idesc, acc);
      } else {
        if (A_TMEM) mma_i8_ts(tbase, tbase + kACol, bd + koff, idesc, acc);
        else mma_i8_ss(tbase, ad + koff, bd + koff, idesc, acc);
      }
    };
    uint32_t uses[4] = {0, 0, 0, 0};
    auto commit = [&](int b) {
      umma_commit(&bars[b]);
      ++uses[b];
      ++commits;
    };
    for (int i = 0; i < 64; ++i) one(i);  // warm-up
    umma_commit(&fin);
    bool ok = mbar_wait(&fin, 0, nullptr);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      one(i + 1);
      if (commit_every > 0 && (i + 1) % commit_every == 0) commit(ring ? (int)(commits % 4) : 0);
    }
    const long long t1 = clock64();
    // commits complete in order, so this one arriving means every MMA is done
    // (the loop's barriers may be several phases behind and are not waited on)
    umma_commit(&fin);
    ok = mbar_wait(&fin, 1, nullptr) && ok;
    const long long t2 = clock64();
    out->issue = t1 - t0;
    out->total = t2 - t0;
    out->status = ok ? 0u : kStatusTimeout;
    done = 1;
  } else if (warp >= 4 && ((smsp_mask >> (warp & 3)) & 1) && (warp - 4) / 4 < busy) {
    // fused multiply-adds until the issuing thread is done (bounded)
    float a0 = tid, a1 = tid + 1, a2 = tid + 2, a3 = tid + 3;
    long long it = 0;
    while (!done && it < kBusyMax) {
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        a0 = fmaf(a0, 1.0001f, 0.5f);
        a1 = fmaf(a1, 1.0001f, 0.5f);
        a2 = fmaf(a2, 1.0001f, 0.5f);
        a3 = fmaf(a3, 1.0001f, 0.5f);
      }
      ++it;
    }
    if ((a0 + a1 + a2 + a3) == 12345.f) out->busy_iters = (unsigned)it;  // keeps the loop
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

template <int KIND, bool A_TMEM>
int run(int n, int iters, int commit_every, int busy, Result* dres, int smsp_mask = 0xF, int ring = 0) {
  const int smem = kSmemA + kSmemB + 1024;
  if (cudaFuncSetAttribute(issue_kernel<KIND, A_TMEM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  cudaMemset(dres, 0, sizeof(Result));
  issue_kernel<KIND, A_TMEM><<<1, kThreads, smem>>>(n, iters, commit_every, busy, smsp_mask, ring, dres);
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  Result r;
  cudaMemcpy(&r, dres, sizeof(r), cudaMemcpyDeviceToHost);
  const int K = KIND == 0 ? 16 : 32;
  printf("{\"kind\": \"%s\", \"a\": \"%s\", \"M\": 128, \"N\": %d, \"K\": %d, \"iters\": %d, \"commit_every\": %d, "
         "\"commit_ring\": %d, \"busy_per_scheduler\": %d, \"busy_scheduler_mask\": %d, "
         "\"issue_cycles_per_mma\": %.2f, \"cycles_per_mma\": %.2f, \"weights_per_kcycle\": %.1f, \"status\": %u}\n",
         KIND == 0 ? "f16(bf16)" : "i8(s8)", A_TMEM ? "tmem" : "smem", n, K, iters, commit_every, ring, busy, smsp_mask,
         (double)r.issue / iters, (double)r.total / iters, 128.0 * K * 1000.0 / ((double)r.total / iters), r.status);
  return r.status != 0 ? 3 : 0;
}

}  // namespace

int main(int argc, char** argv) {
  const int iters = argc > 1 ? atoi(argv[1]) : 4096;
  Result* d = nullptr;
  if (cudaMalloc(&d, sizeof(Result)) != cudaSuccess) return 1;
  int rc = 0;
  const int ns[] = {16, 32, 64, 128};
  for (int n : ns) {
    rc |= run<0, false>(n, iters, 0, 0, d);
    rc |= run<0, true>(n, iters, 0, 0, d);
    rc |= run<1, false>(n, iters, 0, 0, d);
    rc |= run<1, true>(n, iters, 0, 0, d);
  }
  // commits: one barrier, or a ring of four barriers
  for (int ce : {1, 4, 16, 64}) {
    rc |= run<1, true>(32, iters, ce, 0, d, 0xF, 0);
    rc |= run<1, true>(32, iters, ce, 0, d, 0xF, 1);
  }
  // busy warps: on every scheduler, or only on the three the issuer does not use
  for (int busy : {1, 3}) {
    for (int mask : {0xF, 0xE}) {
      rc |= run<1, true>(32, iters, 0, busy, d, mask, 0);
      rc |= run<1, true>(32, iters, 4, busy, d, mask, 1);
      rc |= run<0, true>(16, iters, 8, busy, d, mask, 1);
    }
  }
  cudaFree(d);
  return rc;
}
