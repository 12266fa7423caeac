// Internal host-side declarations shared by the kernels' launchers and the
// C ABI (moe_api.cu).  Not part of the public interface.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

// Launch `kernel` on `s`; with pdl, as a programmatic dependent of the kernel
// queued before it (it may start while that kernel runs and must call
// griddepcontrol.wait before reading that kernel's output).  Only used when
// the previous operation in the stream is one of this library's kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
  if (!pdl) {
    kernel<<<grid, block, smem, s>>>(static_cast<KArgs>(args)...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Devices with a per-device cache entry (device checks, scratch addresses).
constexpr int kMaxDevices = 64;

// Argument checks shared by the C entry points (defined in moe_api.cu).
moe_status api_check_shape(const moe_shape* sh);
moe_status api_check_device(int* num_sms);
int64_t api_capacity(const moe_shape* sh);  // -1: dropless

struct RouterArgs {
  const uint16_t* x;   // [T, d] bf16
  const float* Wg;     // [E, d]
  float* logits;       // [T, E] or nullptr
  int32_t* topk_idx;   // [T, k]
  float* topk_w;       // [T, k]
  float* topk_p;       // [T, k]
  int32_t* counts;     // [E], zeroed by the launcher unless the caller did
  int32_t* next_idx;   // [T, k] router ranks k .. 2k-1 (-1 past E - 1), or nullptr
  float* next_p;       // [T, k] their full-softmax probabilities
  int64_t T;
  int32_t d, E, k;
  uint32_t* status;    // device status word (a wait that gives up), or nullptr
};
cudaError_t launch_router(const RouterArgs& a, int num_sms, cudaStream_t s, bool counts_zeroed);

struct PermuteArgs {
  const uint16_t* x;         // [T, d]
  const int32_t* topk_idx;   // [S]
  const float* topk_p;       // [S] (capacity by probability only)
  const int32_t* counts;     // [E]
  int32_t* offsets;          // [E + 1]
  int32_t* slot_pos;         // [S]
  int32_t* perm_slot;        // [S]
  uint16_t* x_perm;          // [S, d]
  uint32_t* tile_state;      // [n_tiles * E] lookback words, zeroed by the launcher
  uint32_t* ticket;          // tile ticket, zeroed by the launcher
  uint64_t* thresh;          // [E] capacity thresholds
  uint32_t* status;          // device status word
  int64_t T;
  int32_t d, E, k;
  int64_t cap;               // < 0: dropless
  int32_t policy;            // 0 by probability, 1 by token order
  bool pdl;                  // launched as dependents of the router's kernel
};
constexpr int kPermuteTile = 64;  // slots per permutation tile
int64_t permute_tiles(int64_t S);
// state_zeroed: tile_state and ticket were cleared by the caller.
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s, bool state_zeroed);

// Expert GEMMs.  The tensor maps are encoded on the host per call.
struct ExpertGemmArgs {
  const int32_t* offsets;   // [E + 1]
  const uint16_t* x_perm;   // [S, d]
  const uint16_t* W1;       // [E, f, d]
  const uint16_t* W3;       // [E, f, d]
  const uint16_t* W2;       // [E, d, f]
  uint16_t* h;              // [S, f]
  uint16_t* y_perm;         // [S, d] (nullptr: leave split-K partials only)
  float* partials;          // [splits, S, d] for the streaming variant
  uint32_t* status;
  int64_t S;
  int32_t d, f, E;
  int32_t variant;          // 1 tiled, 2 streaming
  int32_t stream_bn;        // streaming variant: token tile (16..128)
  int32_t splits;           // streaming variant: split-K count of the down projection
  int32_t splits1;          // streaming variant: split-K count of the gate/up projection (1: none)
  float* partials1;         // [splits1, S, 2 f] gate/up partials when splits1 > 1
  int num_sms;
  cudaEvent_t between;      // recorded after the first GEMM if not null
  bool pair;                // tiled variant: CTA-pair (cta_group::2) kernels
  uint32_t* tile_counters;  // [2] tile counters of the pair kernels, zeroed by the caller
  bool pdl;                 // launched as dependents of the grouping kernel (no event in between)
  uint64_t* clock_probe;    // profiled calls: [8] clock records of the two GEMMs, else nullptr
};
// Streaming-variant parameters chosen from host-known sizes.
void stream_params(int64_t T, int32_t k, int32_t d, int32_t f, int32_t E, int num_sms, int32_t* bn,
                   int32_t* splits, int32_t* splits1);
cudaError_t launch_expert_gemms(const ExpertGemmArgs& a, cudaStream_t s);

// Expert GEMMs with 4-bit weights (codes [E, R, K/2], scales [E, K/64, R]
// bf16; w = (code - 8) * scale).  One schedule: the streaming one, with the
// down projection's K split into fp32 partials summed by the combine.
struct ExpertGemmQ4Args {
  const int32_t* offsets;   // [E + 1]
  const uint16_t* x_perm;   // [S, d]
  const uint8_t* W1c;       // [E, f, d/2]
  const uint16_t* W1s;      // [E, d/64, f]
  const uint8_t* W3c;
  const uint16_t* W3s;
  const uint8_t* W2c;       // [E, d, f/2]
  const uint16_t* W2s;      // [E, f/64, d]
  uint16_t* h;              // [S, f]
  float* partials;          // [splits, S, d]
  uint32_t* status;
  int64_t S;
  int32_t d, f, E;
  int32_t bn;               // token tile (16..128)
  int32_t splits;           // requested split-K count of the down projection
  int num_sms;
  cudaEvent_t between;      // recorded after the first GEMM if not null
  bool pdl;                 // launched as dependents of the grouping kernel (no event in between)
  uint64_t* clock_probe;    // profiled calls: [8] clock records of the two GEMMs, else nullptr
  uint8_t* act_q;           // token tiles <= 32: the quantised activations as the tiled token operand
  float* act_scale;         // (q4i8_act_bytes) and their per-row scales [S]; nullptr: the bf16-dequantising kernels
};
// The integer-MMA 4-bit GEMMs (token tiles of 16 and 32).
cudaError_t launch_expert_gemms_q4i8(const ExpertGemmQ4Args& a, cudaStream_t s);
// inputs per pipeline stage of those kernels for a token tile, and the bytes
// of their tiled token operand
int32_t q4i8_stage_inputs(int32_t bn);
size_t q4i8_act_bytes(int64_t S, int32_t E, int32_t d, int32_t f, int32_t bn);
// Tensor maps of the 4-bit format (expert_gemm_q4.cu).
bool encode_codes(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows);
bool encode_scales(CUtensorMap* m, const void* base, int64_t E, int64_t R, int64_t K, int box_rows);
void q4_params(int64_t T, int32_t k, int32_t d, int32_t f, int32_t E, int num_sms, int32_t* bn, int32_t* splits);
// number of K splits the down projection really uses for a requested count
// (token tile bn decides the kernel and its K granularity)
int32_t q4_effective_splits(int32_t f, int32_t splits, int32_t bn);
cudaError_t launch_expert_gemms_q4(const ExpertGemmQ4Args& a, cudaStream_t s);
// W [E, R, K] bf16 -> codes and scales (K a multiple of 64, R a multiple of 8)
cudaError_t launch_quantize_q4(const uint16_t* W, int32_t E, int32_t R, int32_t K, uint8_t* codes,
                               uint16_t* scales, cudaStream_t s);

// Per-slot expert histograms [k, E] and first-two-choice pair counts [E, E]
// (nullable; k >= 2) of topk_idx [T, k]; zeroed first unless `accumulate`.
cudaError_t launch_router_stats(const int32_t* idx, int64_t T, int32_t E, int32_t k, int32_t* slot_counts,
                                int32_t* pair_counts, bool accumulate, int num_sms, cudaStream_t s);

// Next-best-expert fallback (capacity mode): decides the expert of every
// slot (eff, -1 = dropped) and its histogram counts_eff; kept1_count,
// cand_count and counts_eff must be zero before the launch.
struct FallbackArgs {
  const int32_t* topk_idx;   // [S]
  const float* topk_p;       // [S]
  const int32_t* counts;     // [E] router histogram
  const int32_t* next_idx;   // [T, k] router ranks k ..
  const float* next_p;       // [T, k]
  uint64_t* keys1;           // [S]
  uint64_t* keys2;           // [S]
  int32_t* cand;             // [S]
  int32_t* eff;              // [S] out
  uint64_t* thresh1;         // [E]
  uint64_t* thresh2;         // [E]
  int32_t* kept1_count;      // [E]
  int32_t* cand_count;       // [E]
  int32_t* counts_eff;       // [E] out
  int64_t T;
  int32_t E, k;
  int64_t cap;
  int32_t policy;            // 0 by probability, 1 by token order
};
cudaError_t launch_fallback(const FallbackArgs& a, int num_sms, cudaStream_t s);

// Expert parallelism (csrc/ep.cu).
cudaError_t launch_ep_plan(const int32_t* counts_all, int32_t E, int32_t rank, int32_t world, int32_t* recv_off,
                           int32_t* owner_off, cudaStream_t s);
// Capacity with expert parallelism: what the dispatch needs to store each
// slot's priority key in its owner's key buffer.
struct EpKeys {
  const float* topk_p;        // [S] full-softmax probabilities of this rank's slots
  const int32_t* counts_all;  // [world, E] routed counts of every rank
  int32_t E, rank;
  uint64_t* const* peer_keys; // [world] device pointers to the owners' key buffers
};
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const int32_t* offsets,
                               const int32_t* slot_pos, const int32_t* recv_off, uint16_t* const* peer_x,
                               int32_t* ret_row, int64_t S, int32_t k, int32_t d, int32_t epr, int num_sms,
                               cudaStream_t s, const EpKeys* keys = nullptr);
cudaError_t launch_ep_combine(const int32_t* topk_idx, const float* topk_w, const int32_t* ret_row,
                              const uint16_t* const* peer_y, uint16_t* y, int64_t T, int32_t k, int32_t d, int32_t epr,
                              int num_sms, cudaStream_t s, const int32_t* const* peer_map = nullptr);
cudaError_t launch_ep_select(const int32_t* counts_all, int32_t world, int32_t E, int32_t k, float cf, int32_t policy,
                             const int32_t* owner_off, const uint64_t* keys, int32_t epr, int32_t* kept_off,
                             int32_t* row_map, const uint16_t* x_recv, uint16_t* x_kept, int32_t d, int num_sms,
                             cudaStream_t s);

struct CombineArgs {
  const uint16_t* y_perm;   // [S, d] bf16, or nullptr when reading partials
  const float* partials;    // [splits, S, d] fp32 (if y_perm == nullptr)
  int32_t splits;
  int64_t part_stride;      // elements between splits
  const int32_t* slot_pos;  // [S]
  const float* topk_w;      // [S]
  uint16_t* y;              // [T, d]
  int64_t T;
  int32_t d, k;
  bool pdl;                 // launched as a dependent of the down-projection GEMM
  uint32_t* status;         // device status word (debug bounds checks), or nullptr
};
cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s);

// y_perm[r] = bf16(sum_s partials[s][r]) for r < offsets[E].
cudaError_t launch_splitk_reduce(const float* partials, int32_t splits, int64_t part_stride,
                                 const int32_t* offsets, int32_t E, uint16_t* y_perm, int64_t S,
                                 int32_t d, int num_sms, cudaStream_t s, uint32_t* status);

// Driver entry point for tensor-map encoding (resolved once through the runtime).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace moe
