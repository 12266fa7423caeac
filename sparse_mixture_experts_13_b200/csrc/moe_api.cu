// C ABI of the sparse mixture-of-experts layer (declared in include/moe.h):
// argument checks, workspace layout, choice of the expert-GEMM schedule and
// the launch sequence.  No entry point allocates memory or synchronises
// (except moe_read_device_status).
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe.h"
#include "moe_internal.h"

using namespace moe;

namespace {

// Split-K and workspace sizes are derived with this SM count so that the
// workspace size is a function of the shape alone; grids use the real count.
constexpr int kPlanSms = 148;
constexpr size_t kAlign = 256;
#ifdef MOE_DEBUG
constexpr bool kDebugBuild = true;
#else
constexpr bool kDebugBuild = false;
#endif
// Profiled calls: the two expert GEMMs each write {clock64, globaltimer} of
// CTA 0 at entry and exit here (bytes 64 .. 127 of the control header, which
// the layer clears at the start of every call).
constexpr size_t kClockProbeOffset = 64;
constexpr size_t kGuard = 256;        // debug build: guard bytes after each region past the control region
constexpr int kMaxGuards = 32;
#ifdef MOE_DEBUG
constexpr unsigned char kGuardByte = 0xA5;
#endif

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_shape(const moe_shape* sh) {
  if (!sh) return MOE_ERR_INVALID_ARG;
  if (sh->T < 0) return MOE_ERR_INVALID_ARG;
  if (sh->E < 1 || sh->E > 32) return MOE_ERR_INVALID_ARG;
  if (sh->k < 1 || sh->k > 8 || sh->k > sh->E) return MOE_ERR_INVALID_ARG;
  if (sh->d_model < 64 || sh->d_model > 65536 || sh->d_model % 64) return MOE_ERR_INVALID_ARG;
  if (sh->d_ff < 64 || sh->d_ff > 65536 || sh->d_ff % 64) return MOE_ERR_INVALID_ARG;
  if (sh->T * (int64_t)sh->k >= ((int64_t)1 << 30)) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(sh->capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (sh->drop_policy < MOE_DROP_BY_PROB || sh->drop_policy > MOE_DROP_BY_ORDER_NEXT_BEST) return MOE_ERR_INVALID_ARG;
  if (sh->gemm_variant < MOE_VARIANT_AUTO || sh->gemm_variant > MOE_VARIANT_TILED_SINGLE) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int64_t capacity_of(const moe_shape* sh) {
  if (sh->capacity_factor <= 0.f) return -1;
  return (int64_t)std::floor((double)sh->capacity_factor * (double)sh->T * (double)sh->k / (double)sh->E);
}

// Capacity mode with the next-best-expert fallback.
bool fallback_of(const moe_shape* sh) {
  return sh->capacity_factor > 0.f && sh->drop_policy >= MOE_DROP_BY_PROB_NEXT_BEST;
}

// AUTO: the weight-streaming schedule up to 128 tokens; single-CTA tiles
// while an expert's mean slot count fits one 128-token tile (T k / E <= 112);
// CTA pairs above.  Measured on one B200 at d_model 4096, d_ff 14336, E 8,
// top-2: single-CTA tiles 3-6 % faster than pairs from 160 to 448 tokens,
// pairs 11 % faster at 512.
int variant_of(const moe_shape* sh) {
  if (sh->gemm_variant != MOE_VARIANT_AUTO) return sh->gemm_variant;
  if (sh->T <= 128) return MOE_VARIANT_STREAM;
  if (sh->T * sh->k <= 112 * (int64_t)sh->E) return MOE_VARIANT_TILED_SINGLE;
  return MOE_VARIANT_TILED;
}

struct Layout {
  // control region, cleared at the start of moe_layer_forward: status word,
  // tile ticket, two GEMM tile counters, counts, look-back words
  size_t status, ticket, counts, tile_state, ctrl_end;
  size_t thresh, partials, topk_idx, topk_w, topk_p, offsets, slot_pos, perm_slot, x_perm, h, y_perm,
      x_stage, y_stage, total;
  // next-best-expert fallback only (0 otherwise); fb_counts sits in the
  // control region: kept1_count, cand_count, counts_eff [3 E]
  size_t fb_counts, next_idx, next_p, keys1, keys2, cand, eff, thresh2;
  bool fallback;
  int variant;
  bool q4;                 // 4-bit expert weights (always the streaming schedule)
  int32_t bn, splits;      // streaming schedule: token tile, requested split-K count
  int32_t splits1;         // streaming schedule: gate/up split-K count (1: none)
  size_t partials1;        // gate/up partials [splits1, S, 2 f] when splits1 > 1
  int32_t eff_splits;      // split-K partial buffers the down projection writes
  size_t act_q, act_scale; // 4-bit, token tiles <= 32: tiled quantised activations and their scales [S]
  size_t guards[kMaxGuards];  // debug build: offsets of the guards
  int nguards;
};

// End of a region that ends at `end`: the next 256-byte boundary, followed
// in debug builds by a guard.
size_t next_region(Layout& L, size_t end) {
  size_t o = align_up(end);
  if (kDebugBuild && L.nguards < kMaxGuards) {
    L.guards[L.nguards++] = o;
    o += kGuard;
  }
  return o;
}

// q4: layout of the 4-bit entry points (split-K partials always present).
Layout layout_of(const moe_shape* sh, bool q4 = false) {
  Layout L{};
  const int64_t T = sh->T, S = T * sh->k;
  const int64_t d = sh->d_model, f = sh->d_ff, E = sh->E;
  L.variant = q4 ? MOE_VARIANT_STREAM : variant_of(sh);
  L.q4 = q4;
  L.bn = 128;
  L.splits = 1;
  L.splits1 = 1;
  L.eff_splits = 1;
  if (q4) {
    q4_params(T, sh->k, sh->d_model, sh->d_ff, sh->E, kPlanSms, &L.bn, &L.splits);
    L.eff_splits = q4_effective_splits(sh->d_ff, L.splits, L.bn);
  } else if (L.variant == MOE_VARIANT_STREAM) {
    stream_params(T, sh->k, sh->d_model, sh->d_ff, sh->E, kPlanSms, &L.bn, &L.splits, &L.splits1);
    const int32_t num_kb = sh->d_ff / 64;
    const int32_t kbps = (num_kb + L.splits - 1) / L.splits;
    L.eff_splits = (num_kb + kbps - 1) / kbps;
  }
  size_t o = 0;
  L.status = o;
  L.ticket = o + 4;
  o = align_up(o + 16);
  L.counts = o;
  o = align_up(o + 4 * E);
  L.fallback = fallback_of(sh);
  if (L.fallback) {
    L.fb_counts = o;
    o = align_up(o + 3 * 4 * E);
  }
  L.tile_state = o;
  o = align_up(o + 4 * (size_t)permute_tiles(S) * E);
  L.ctrl_end = o;
  L.thresh = o;
  o = next_region(L, o + 8 * E);
  L.partials = o;
  if (L.variant == MOE_VARIANT_STREAM) o = next_region(L, o + 4 * (size_t)L.eff_splits * S * d);
  L.partials1 = o;
  if (L.splits1 > 1) o = next_region(L, o + 4 * (size_t)L.splits1 * S * 2 * f);
  L.topk_idx = o;
  o = next_region(L, o + 4 * S);
  L.topk_w = o;
  o = next_region(L, o + 4 * S);
  L.topk_p = o;
  o = next_region(L, o + 4 * S);
  L.offsets = o;
  o = next_region(L, o + 4 * (E + 1));
  L.slot_pos = o;
  o = next_region(L, o + 4 * S);
  L.perm_slot = o;
  o = next_region(L, o + 4 * S);
  L.x_perm = o;
  o = next_region(L, o + 2 * (size_t)S * d);
  L.h = o;
  o = next_region(L, o + 2 * (size_t)S * f);
  L.y_perm = o;
  o = next_region(L, o + 2 * (size_t)S * d);
  L.x_stage = o;
  o = next_region(L, o + 2 * (size_t)T * d);
  L.y_stage = o;
  o = next_region(L, o + 2 * (size_t)T * d);
  if (L.fallback) {
    L.next_idx = o;
    o = next_region(L, o + 4 * S);
    L.next_p = o;
    o = next_region(L, o + 4 * S);
    L.keys1 = o;
    o = next_region(L, o + 8 * S);
    L.keys2 = o;
    o = next_region(L, o + 8 * S);
    L.cand = o;
    o = next_region(L, o + 4 * S);
    L.eff = o;
    o = next_region(L, o + 4 * S);
    L.thresh2 = o;
    o = next_region(L, o + 8 * E);
  }
  if (L.q4 && L.bn <= 32) {
    L.act_q = o;
    o = next_region(L, o + q4i8_act_bytes(S, E, d, f, L.bn));
    L.act_scale = o;
    o = next_region(L, o + 4 * (size_t)S);
  }
  L.total = o;
  return L;
}

moe_status check_ws(const moe_shape* sh, const void* ws, size_t ws_bytes, bool q4 = false) {
  if (!ws || !aligned(ws, kAlign)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < layout_of(sh, q4).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Device checks, cached per device: sm_100 family and SM count.
int g_dev_state[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
int g_dev_sms[kMaxDevices];

moe_status check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  if (g_dev_state[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_dev_sms[dev] = sms;
    g_dev_state[dev] = (major == 10) ? 1 : 2;
  }
  if (g_dev_state[dev] != 1) return MOE_ERR_UNSUPPORTED;
  *num_sms = g_dev_sms[dev];
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

#define MOE_TRY(expr)                  \
  do {                                 \
    moe_status _st = (expr);           \
    if (_st != MOE_OK) return _st;     \
  } while (0)

moe_status check_bf16(const void* p) { return (p && aligned(p, 16)) ? MOE_OK : MOE_ERR_INVALID_ARG; }
moe_status check_i32(const void* p) { return (p && aligned(p, 4)) ? MOE_OK : MOE_ERR_INVALID_ARG; }

moe_status run_router(const moe_shape* sh, const moe_bf16* x, const float* Wg, float* logits, int32_t* idx, float* w,
                      float* p, int32_t* counts, int num_sms, cudaStream_t s, bool counts_zeroed,
                      int32_t* next_idx = nullptr, float* next_p = nullptr, uint32_t* status = nullptr) {
  RouterArgs a{x, Wg, logits, idx, w, p, counts, next_idx, next_p, sh->T, sh->d_model, sh->E, sh->k, status};
  return cuda_status(launch_router(a, num_sms, s, counts_zeroed));
}

moe_status run_permute(const moe_shape* sh, const Layout& L, const moe_bf16* x, const int32_t* idx, const float* p,
                       const int32_t* counts, int32_t* offsets, int32_t* slot_pos, int32_t* perm_slot,
                       moe_bf16* x_perm, void* ws, cudaStream_t s, bool state_zeroed, bool pdl = false) {
  PermuteArgs a{};
  a.pdl = pdl;
  a.x = x;
  a.topk_idx = idx;
  a.topk_p = p;
  a.counts = counts;
  a.offsets = offsets;
  a.slot_pos = slot_pos;
  a.perm_slot = perm_slot;
  a.x_perm = x_perm;
  a.tile_state = at<uint32_t>(ws, L.tile_state);
  a.ticket = at<uint32_t>(ws, L.ticket);
  a.thresh = at<uint64_t>(ws, L.thresh);
  a.status = at<uint32_t>(ws, L.status);
  a.T = sh->T;
  a.d = sh->d_model;
  a.E = sh->E;
  a.k = sh->k;
  a.cap = capacity_of(sh);
  a.policy = sh->drop_policy;
  return cuda_status(launch_permute(a, s, state_zeroed));
}

moe_status run_gemms(const moe_shape* sh, const Layout& L, const moe_bf16* x_perm, const int32_t* offsets,
                     const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2, moe_bf16* h, moe_bf16* y_perm,
                     void* ws, int num_sms, cudaStream_t s, cudaEvent_t between = nullptr, bool pdl = false) {
  ExpertGemmArgs a{};
  a.pdl = pdl;
  // profiled calls (events between the kernels): clock records in the
  // control header's spare bytes 64 .. 127
  a.clock_probe = between ? at<uint64_t>(ws, L.status + kClockProbeOffset) : nullptr;
  a.offsets = offsets;
  a.x_perm = x_perm;
  a.W1 = W1;
  a.W3 = W3;
  a.W2 = W2;
  a.h = h;
  a.y_perm = y_perm;
  a.partials = at<float>(ws, L.partials);
  a.status = at<uint32_t>(ws, L.status);
  a.S = sh->T * sh->k;
  a.d = sh->d_model;
  a.f = sh->d_ff;
  a.E = sh->E;
  a.variant = L.variant == MOE_VARIANT_STREAM ? 2 : 1;
  a.pair = L.variant == MOE_VARIANT_TILED;
  a.stream_bn = L.bn;
  a.splits = L.splits;
  a.splits1 = L.splits1;
  a.partials1 = L.splits1 > 1 ? at<float>(ws, L.partials1) : nullptr;
  a.num_sms = num_sms;
  a.between = between;
  a.tile_counters = at<uint32_t>(ws, L.status) + 2;  // words 2 and 3 of the control header
  return cuda_status(launch_expert_gemms(a, s));
}

// Expert weights of one call: bf16 matrices, or 4-bit codes and scales.
struct ExpertWeights {
  const moe_bf16 *W1, *W3, *W2;
  const uint8_t *W1c, *W3c, *W2c;
  const moe_bf16 *W1s, *W3s, *W2s;
};

moe_status run_gemms_q4(const moe_shape* sh, const Layout& L, const moe_bf16* x_perm, const int32_t* offsets,
                        const ExpertWeights& W, moe_bf16* h, void* ws, int num_sms, cudaStream_t s,
                        cudaEvent_t between = nullptr, bool pdl = false) {
  ExpertGemmQ4Args a{};
  a.pdl = pdl;
  a.clock_probe = between ? at<uint64_t>(ws, L.status + kClockProbeOffset) : nullptr;
  a.offsets = offsets;
  a.x_perm = x_perm;
  a.W1c = W.W1c;
  a.W1s = W.W1s;
  a.W3c = W.W3c;
  a.W3s = W.W3s;
  a.W2c = W.W2c;
  a.W2s = W.W2s;
  a.h = h;
  a.partials = at<float>(ws, L.partials);
  a.status = at<uint32_t>(ws, L.status);
  a.S = sh->T * sh->k;
  a.d = sh->d_model;
  a.f = sh->d_ff;
  a.E = sh->E;
  a.bn = L.bn;
  a.splits = L.splits;
  a.num_sms = num_sms;
  a.between = between;
  if (L.act_q) {
    a.act_q = at<uint8_t>(ws, L.act_q);
    a.act_scale = at<float>(ws, L.act_scale);
  }
  return cuda_status(launch_expert_gemms_q4(a, s));
}

moe_status check_q4_weights(const ExpertWeights& W) {
  const void* ps[6] = {W.W1c, W.W3c, W.W2c, W.W1s, W.W3s, W.W2s};
  for (const void* p : ps)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

namespace moe {
moe_status api_check_shape(const moe_shape* sh) { return check_shape(sh); }
moe_status api_check_device(int* num_sms) { return check_device(num_sms); }
int64_t api_capacity(const moe_shape* sh) { return capacity_of(sh); }
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return layout_of(shape).total;
}

moe_status moe_router_topk(const moe_shape* sh, const moe_bf16* x, const float* Wg, float* logits,
                           int32_t* topk_idx, float* topk_w, float* topk_p, int32_t* counts, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(topk_w));
  MOE_TRY(check_i32(topk_p));
  MOE_TRY(check_i32(counts));
  if (logits && !aligned(logits, 4)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return run_router(sh, x, Wg, logits, topk_idx, topk_w, topk_p, counts, sms, (cudaStream_t)stream, false);
}

moe_status moe_permute(const moe_shape* sh, const moe_bf16* x, const int32_t* topk_idx, const float* topk_p,
                       const int32_t* counts, int32_t* offsets, int32_t* slot_pos, int32_t* perm_slot,
                       moe_bf16* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(counts));
  MOE_TRY(check_i32(offsets));
  MOE_TRY(check_i32(slot_pos));
  MOE_TRY(check_i32(perm_slot));
  MOE_TRY(check_bf16(x_perm));
  if (sh->capacity_factor > 0.f && sh->drop_policy == MOE_DROP_BY_PROB) MOE_TRY(check_i32(topk_p));
  // the fallback needs the router's ranks past the top k, which only the
  // whole-layer entry points compute
  if (fallback_of(sh)) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, 8, s)));  // status word and tile ticket
  return run_permute(sh, L, x, topk_idx, topk_p, counts, offsets, slot_pos, perm_slot, x_perm, ws, s, false);
}

moe_status moe_grouped_swiglu(const moe_shape* sh, const moe_bf16* x_perm, const int32_t* offsets,
                              const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2, moe_bf16* h,
                              moe_bf16* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(x_perm));
  MOE_TRY(check_i32(offsets));
  MOE_TRY(check_bf16(W1));
  MOE_TRY(check_bf16(W3));
  MOE_TRY(check_bf16(W2));
  MOE_TRY(check_bf16(h));
  MOE_TRY(check_bf16(y_perm));
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, 16, s)));  // status, ticket, GEMM tile counters
  MOE_TRY(run_gemms(sh, L, x_perm, offsets, W1, W3, W2, h, y_perm, ws, sms, s));
  if (L.variant == MOE_VARIANT_STREAM) {
    const int64_t S = sh->T * sh->k;
    MOE_TRY(cuda_status(launch_splitk_reduce(at<float>(ws, L.partials), L.eff_splits, S * (int64_t)sh->d_model,
                                             offsets, sh->E, y_perm, S, sh->d_model, sms, s,
                                             at<uint32_t>(ws, L.status))));
  }
  return MOE_OK;
}

moe_status moe_combine(const moe_shape* sh, const moe_bf16* y_perm, const int32_t* slot_pos, const float* topk_w,
                       moe_bf16* y, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(y_perm));
  MOE_TRY(check_i32(slot_pos));
  MOE_TRY(check_i32(topk_w));
  MOE_TRY(check_bf16(y));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  CombineArgs a{};
  a.y_perm = y_perm;
  a.slot_pos = slot_pos;
  a.topk_w = topk_w;
  a.y = y;
  a.T = sh->T;
  a.d = sh->d_model;
  a.k = sh->k;
  return cuda_status(launch_combine(a, sms, (cudaStream_t)stream));
}

// Debug build: MOE_DEBUG_FAIL_STAGE=n makes the layer entry points fail with
// MOE_ERR_CUDA just before queuing stage n (1 router, 2 capacity / grouping,
// 3 expert GEMMs, 4 combine, 5 output copies).
static int debug_fail_stage() {
  if (!kDebugBuild) return 0;
  const char* v = std::getenv("MOE_DEBUG_FAIL_STAGE");
  return v ? std::atoi(v) : 0;
}
#define MOE_STAGE(n)                                     \
  do {                                                   \
    if (fail_at == (n)) return MOE_ERR_CUDA;             \
  } while (0)

// keep_status: leave the status word (bytes 0 .. 3 of ws) as an earlier call
// on the same stream left it (a later chunk of one host-buffer call)
static moe_status layer_forward_impl(const moe_shape* sh, const moe_bf16* x, const float* Wg, const ExpertWeights& W,
                                     bool q4, moe_bf16* y, int32_t* topk_idx_out, int32_t* counts_out, void* ws,
                                     int sms, cudaStream_t s, cudaEvent_t const* ev = nullptr,
                                     bool keep_status = false) {
  const Layout L = layout_of(sh, q4);
  const int64_t S = sh->T * sh->k;
  int32_t* idx = at<int32_t>(ws, L.topk_idx);
  float* w = at<float>(ws, L.topk_w);
  float* p = at<float>(ws, L.topk_p);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot_pos = at<int32_t>(ws, L.slot_pos);
  int32_t* perm_slot = at<int32_t>(ws, L.perm_slot);
  moe_bf16* x_perm = at<moe_bf16>(ws, L.x_perm);
  moe_bf16* h = at<moe_bf16>(ws, L.h);
  moe_bf16* y_perm = at<moe_bf16>(ws, L.y_perm);
  auto mark = [&](int i) { return ev ? cuda_status(cudaEventRecord(ev[i], s)) : MOE_OK; };
  // Without events between them, each kernel after the router is launched
  // as a programmatic dependent of the one before (its set-up overlaps that
  // kernel; it waits for it before reading its output).
  const bool pdl = ev == nullptr;
  const int fail_at = debug_fail_stage();
  MOE_TRY(mark(0));
  {
    // one clear of the control region (status, ticket, counts, look-back words)
    const size_t from = keep_status ? L.ticket : 0;
    MOE_TRY(cuda_status(cudaMemsetAsync(static_cast<uint8_t*>(ws) + from, 0, L.ctrl_end - from, s)));
  }
  MOE_STAGE(1);
  if (L.fallback) {
    MOE_TRY(run_router(sh, x, Wg, nullptr, idx, w, p, counts, sms, s, true, at<int32_t>(ws, L.next_idx),
                       at<float>(ws, L.next_p), at<uint32_t>(ws, L.status)));
    MOE_TRY(mark(1));
    MOE_STAGE(2);
    FallbackArgs fa{};
    fa.topk_idx = idx;
    fa.topk_p = p;
    fa.counts = counts;
    fa.next_idx = at<int32_t>(ws, L.next_idx);
    fa.next_p = at<float>(ws, L.next_p);
    fa.keys1 = at<uint64_t>(ws, L.keys1);
    fa.keys2 = at<uint64_t>(ws, L.keys2);
    fa.cand = at<int32_t>(ws, L.cand);
    fa.eff = at<int32_t>(ws, L.eff);
    fa.thresh1 = at<uint64_t>(ws, L.thresh);
    fa.thresh2 = at<uint64_t>(ws, L.thresh2);
    fa.kept1_count = at<int32_t>(ws, L.fb_counts);
    fa.cand_count = fa.kept1_count + sh->E;
    fa.counts_eff = fa.kept1_count + 2 * sh->E;
    fa.T = sh->T;
    fa.E = sh->E;
    fa.k = sh->k;
    fa.cap = capacity_of(sh);
    fa.policy = sh->drop_policy - MOE_DROP_BY_PROB_NEXT_BEST;
    MOE_TRY(cuda_status(launch_fallback(fa, sms, s)));
    // group by the expert each slot landed on; dropped slots carry -1
    moe_shape dropless = *sh;
    dropless.capacity_factor = 0.f;
    dropless.drop_policy = MOE_DROP_BY_PROB;
    MOE_TRY(run_permute(&dropless, L, x, fa.eff, p, fa.counts_eff, offsets, slot_pos, perm_slot, x_perm, ws, s,
                        true, pdl));
  } else {
    MOE_TRY(run_router(sh, x, Wg, nullptr, idx, w, p, counts, sms, s, true, nullptr, nullptr,
                       at<uint32_t>(ws, L.status)));
    MOE_TRY(mark(1));
    MOE_STAGE(2);
    MOE_TRY(run_permute(sh, L, x, idx, p, counts, offsets, slot_pos, perm_slot, x_perm, ws, s, true, pdl));
  }
  MOE_TRY(mark(2));
  MOE_STAGE(3);
  if (q4)
    MOE_TRY(run_gemms_q4(sh, L, x_perm, offsets, W, h, ws, sms, s, ev ? ev[3] : nullptr, pdl));
  else
    MOE_TRY(run_gemms(sh, L, x_perm, offsets, W.W1, W.W3, W.W2, h, y_perm, ws, sms, s, ev ? ev[3] : nullptr, pdl));
  MOE_TRY(mark(4));
  MOE_STAGE(4);
  CombineArgs c{};
  c.pdl = pdl;
  c.status = at<uint32_t>(ws, L.status);
  c.slot_pos = slot_pos;
  c.topk_w = w;
  c.y = y;
  c.T = sh->T;
  c.d = sh->d_model;
  c.k = sh->k;
  if (L.variant == MOE_VARIANT_STREAM) {
    c.y_perm = nullptr;
    c.partials = at<float>(ws, L.partials);
    c.splits = L.eff_splits;
    c.part_stride = S * (int64_t)sh->d_model;
  } else {
    c.y_perm = y_perm;
  }
  MOE_TRY(cuda_status(launch_combine(c, sms, s)));
  MOE_TRY(mark(5));
  MOE_STAGE(5);
  if (topk_idx_out)
    MOE_TRY(cuda_status(cudaMemcpyAsync(topk_idx_out, idx, sizeof(int32_t) * S, cudaMemcpyDeviceToDevice, s)));
  if (counts_out)
    MOE_TRY(cuda_status(cudaMemcpyAsync(counts_out, counts, sizeof(int32_t) * sh->E, cudaMemcpyDeviceToDevice, s)));
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_shape* sh, const moe_bf16* x, const float* Wg, const moe_bf16* W1,
                             const moe_bf16* W3, const moe_bf16* W2, moe_bf16* y, int32_t* topk_idx_out,
                             int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_bf16(W1));
  MOE_TRY(check_bf16(W3));
  MOE_TRY(check_bf16(W2));
  MOE_TRY(check_bf16(y));
  if (topk_idx_out && !aligned(topk_idx_out, 4)) return MOE_ERR_INVALID_ARG;
  if (counts_out && !aligned(counts_out, 4)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const ExpertWeights Wt{W1, W3, W2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  return layer_forward_impl(sh, x, Wg, Wt, false, y, topk_idx_out, counts_out, ws, sms, (cudaStream_t)stream);
}

moe_status moe_layer_forward_profiled(const moe_shape* sh, const moe_bf16* x, const float* Wg, const moe_bf16* W1,
                                      const moe_bf16* W3, const moe_bf16* W2, moe_bf16* y, void* const* events,
                                      void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_bf16(W1));
  MOE_TRY(check_bf16(W3));
  MOE_TRY(check_bf16(W2));
  MOE_TRY(check_bf16(y));
  if (!events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const ExpertWeights Wt{W1, W3, W2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  return layer_forward_impl(sh, x, Wg, Wt, false, y, nullptr, nullptr, ws, sms, (cudaStream_t)stream,
                            reinterpret_cast<cudaEvent_t const*>(events));
}

// Chunks of a host-buffer call.  In dropless mode every token is routed,
// grouped, computed and combined on its own: the router's sum for a token,
// a CTA-pair GEMM's output row and the combine of a token do not depend on
// which other tokens share the call.  So for T >= 4096 the layer runs on
// 2 to 8 consecutive groups of about 4096 tokens and at least 2048 (the
// same router and GEMM kernels as the whole call, same results bit for
// bit), and each group's copies overlap the other groups' kernels.
// Measured at d_model 4096, d_ff 14336: groups of 2048 at T = 4096 (3.40 ->
// 3.07 ms per call), of 4096 at T = 8192 (6.5 -> 5.5 ms); groups of 1024
// were no faster than one call.  1: one call.
static int64_t host_chunks(const moe_shape* sh) {
  if (kDebugBuild || sh->capacity_factor > 0.f || variant_of(sh) != MOE_VARIANT_TILED || sh->T < 4096) return 1;
  int64_t C = sh->T / 4096;
  if (C < 2) C = 2;
  if (C > 8) C = 8;
  moe_shape part = *sh;
  part.T = sh->T / C;  // the smallest group
  return variant_of(&part) == MOE_VARIANT_TILED ? C : 1;
}

// The two copy streams (host to device, device to host) of chunked
// host-buffer calls made on `user` (a stream of the current device): one
// pair per user stream, so that calls on different streams do not queue
// behind each other's copies; created on first use and kept for the
// process (invalid after the device is reset).  Past kCopyPairs user
// streams on a device, the pairs are shared (still correct, less overlap).
constexpr int kCopyPairs = 8;
static moe_status copy_streams(cudaStream_t user, cudaStream_t* in, cudaStream_t* out) {
  struct Pair {
    cudaStream_t user, in, out;
    bool used;
  };
  static Pair pairs[kMaxDevices][kCopyPairs];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  Pair* row = pairs[dev];
  int slot = -1;
  for (int i = 0; i < kCopyPairs && slot < 0; ++i)
    if (row[i].used && row[i].user == user) slot = i;
  for (int i = 0; i < kCopyPairs && slot < 0; ++i)
    if (!row[i].used) {
      if (cudaStreamCreateWithFlags(&row[i].in, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaStreamCreateWithFlags(&row[i].out, cudaStreamNonBlocking) != cudaSuccess) {
        cudaStreamDestroy(row[i].in);
        return MOE_ERR_CUDA;
      }
      row[i].user = user;
      row[i].used = true;
      slot = i;
    }
  if (slot < 0) slot = (int)((reinterpret_cast<uintptr_t>(user) >> 4) % kCopyPairs);
  *in = row[slot].in;
  *out = row[slot].out;
  return MOE_OK;
}

// Chunked host-buffer layer: group c's x goes in on the input copy stream,
// its kernels run on `s` once it has arrived, and its y goes out on the
// output copy stream once they are done; the call's work ends on `s`.
static moe_status layer_forward_host_chunked(const moe_shape* sh, int64_t C, const moe_bf16* x_host, const float* Wg,
                                             const ExpertWeights& Wt, moe_bf16* y_host, moe_bf16* xd, moe_bf16* yd,
                                             void* ws, int sms, cudaStream_t s) {
  cudaStream_t cin = nullptr, cout = nullptr;
  MOE_TRY(copy_streams(s, &cin, &cout));
  constexpr int kMaxEvents = 2 * 8 + 2;
  cudaEvent_t ev[kMaxEvents] = {};
  const int nev = (int)(2 * C + 2);
  moe_status st = MOE_OK;
  for (int i = 0; i < nev && st == MOE_OK; ++i)
    st = cuda_status(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming));
  const int64_t d = sh->d_model;
  auto rows = [&](int64_t c) { return sh->T * c / C; };
  // the copies into the staged x wait for the work already queued on s
  if (st == MOE_OK) st = cuda_status(cudaEventRecord(ev[0], s));
  if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(cin, ev[0], 0));
  for (int64_t c = 0; c < C && st == MOE_OK; ++c) {
    const int64_t r0 = rows(c), n = rows(c + 1) - r0;
    st = cuda_status(cudaMemcpyAsync(xd + r0 * d, x_host + r0 * d, 2 * (size_t)n * d, cudaMemcpyHostToDevice, cin));
    if (st == MOE_OK) st = cuda_status(cudaEventRecord(ev[1 + c], cin));
  }
  for (int64_t c = 0; c < C && st == MOE_OK; ++c) {
    const int64_t r0 = rows(c), n = rows(c + 1) - r0;
    st = cuda_status(cudaStreamWaitEvent(s, ev[1 + c], 0));
    moe_shape part = *sh;
    part.T = n;
    if (st == MOE_OK)
      st = layer_forward_impl(&part, xd + r0 * d, Wg, Wt, false, yd + r0 * d, nullptr, nullptr, ws, sms, s, nullptr,
                              c > 0);
    if (st == MOE_OK) st = cuda_status(cudaEventRecord(ev[1 + C + c], s));
    if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(cout, ev[1 + C + c], 0));
    if (st == MOE_OK)
      st = cuda_status(cudaMemcpyAsync(y_host + r0 * d, yd + r0 * d, 2 * (size_t)n * d, cudaMemcpyDeviceToHost, cout));
  }
  // the call's last copy is ordered before whatever follows on s, also when
  // a step above failed (copies already queued still finish before it)
  if (ev[nev - 1]) {
    const moe_status j = cuda_status(cudaEventRecord(ev[nev - 1], cout));
    const moe_status w = j == MOE_OK ? cuda_status(cudaStreamWaitEvent(s, ev[nev - 1], 0)) : j;
    if (st == MOE_OK) st = w;
  }
  for (int i = 0; i < nev; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  return st;
}

moe_status moe_layer_forward_host(const moe_shape* sh, const moe_bf16* x_host, const float* Wg, const moe_bf16* W1,
                                  const moe_bf16* W3, const moe_bf16* W2, moe_bf16* y_host, void* ws,
                                  size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_bf16(W1));
  MOE_TRY(check_bf16(W3));
  MOE_TRY(check_bf16(W2));
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = 2 * (size_t)sh->T * sh->d_model;
  moe_bf16* xd = at<moe_bf16>(ws, L.x_stage);
  moe_bf16* yd = at<moe_bf16>(ws, L.y_stage);
  const ExpertWeights Wt{W1, W3, W2, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  const int64_t C = host_chunks(sh);
  if (C > 1) return layer_forward_host_chunked(sh, C, x_host, Wg, Wt, y_host, xd, yd, ws, sms, s);
  MOE_TRY(cuda_status(cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s)));
  MOE_TRY(layer_forward_impl(sh, xd, Wg, Wt, false, yd, nullptr, nullptr, ws, sms, s));
  return cuda_status(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, s));
}

moe_status moe_ep_plan(const int32_t* counts_all, int32_t E, int32_t rank, int32_t world, int32_t* recv_off,
                       int32_t* owner_off, moe_stream_t stream) {
  if (E < 1 || E > 32 || world < 1 || world > 32 || E % world || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_i32(counts_all));
  MOE_TRY(check_i32(recv_off));
  MOE_TRY(check_i32(owner_off));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_ep_plan(counts_all, E, rank, world, recv_off, owner_off, (cudaStream_t)stream));
}

moe_status moe_ep_dispatch(const moe_shape* sh, int32_t world, const moe_bf16* x, const int32_t* topk_idx,
                           const int32_t* counts, const int32_t* recv_off, moe_bf16* const* peer_x, int32_t* ret_row,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (world < 1 || world > 32 || sh->E % world) return MOE_ERR_INVALID_ARG;
  if (sh->T == 0) return MOE_OK;
  if (sh->capacity_factor > 0.f) return MOE_ERR_UNSUPPORTED;  // the expert-parallel layer is dropless
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(counts));
  MOE_TRY(check_i32(recv_off));
  MOE_TRY(check_bf16(peer_x));
  MOE_TRY(check_i32(ret_row));
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, 8, s)));  // status word and tile ticket
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot_pos = at<int32_t>(ws, L.slot_pos);
  // this rank's slots ranked per expert in token order (no local copy of x)
  MOE_TRY(run_permute(sh, L, x, topk_idx, nullptr, counts, offsets, slot_pos, at<int32_t>(ws, L.perm_slot), nullptr,
                      ws, s, false));
  return cuda_status(launch_ep_dispatch(x, topk_idx, offsets, slot_pos, recv_off,
                                        reinterpret_cast<uint16_t* const*>(peer_x), ret_row, sh->T * sh->k, sh->k,
                                        sh->d_model, sh->E / world, sms, s));
}

moe_status moe_ep_combine(const moe_shape* sh, int32_t world, const int32_t* topk_idx, const float* topk_w,
                          const int32_t* ret_row, const moe_bf16* const* peer_y, moe_bf16* y, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (world < 1 || world > 32 || sh->E % world) return MOE_ERR_INVALID_ARG;
  if (sh->T == 0) return MOE_OK;
  if (sh->capacity_factor > 0.f) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(topk_w));
  MOE_TRY(check_i32(ret_row));
  MOE_TRY(check_bf16(peer_y));
  MOE_TRY(check_bf16(y));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_ep_combine(topk_idx, topk_w, ret_row, reinterpret_cast<const uint16_t* const*>(peer_y),
                                       y, sh->T, sh->k, sh->d_model, sh->E / world, sms, (cudaStream_t)stream));
}

moe_status moe_ep_dispatch_cap(const moe_shape* sh, int32_t world, int32_t rank, const int32_t* counts_all,
                               const moe_bf16* x, const int32_t* topk_idx, const float* topk_p, const int32_t* counts,
                               const int32_t* recv_off, moe_bf16* const* peer_x, uint64_t* const* peer_keys,
                               int32_t* ret_row, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (world < 1 || world > 32 || sh->E % world || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  if (!(sh->capacity_factor > 0.f)) return MOE_ERR_INVALID_ARG;              // the dropless path is moe_ep_dispatch
  if (sh->drop_policy > MOE_DROP_BY_ORDER) return MOE_ERR_UNSUPPORTED;       // no next-best fallback here
  if (sh->T == 0) return MOE_OK;
  const bool by_prob = sh->drop_policy == MOE_DROP_BY_PROB;
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(counts));
  MOE_TRY(check_i32(counts_all));
  MOE_TRY(check_i32(recv_off));
  MOE_TRY(check_bf16(peer_x));
  MOE_TRY(check_i32(ret_row));
  if (by_prob) {
    MOE_TRY(check_i32(topk_p));
    MOE_TRY(check_bf16(peer_keys));
  }
  MOE_TRY(check_ws(sh, ws, ws_bytes));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  moe_shape dropless = *sh;  // every slot is sent; the owners select
  dropless.capacity_factor = 0.f;
  const Layout L = layout_of(&dropless);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, 8, s)));
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot_pos = at<int32_t>(ws, L.slot_pos);
  MOE_TRY(run_permute(&dropless, L, x, topk_idx, nullptr, counts, offsets, slot_pos, at<int32_t>(ws, L.perm_slot),
                      nullptr, ws, s, false));
  const EpKeys keys{topk_p, counts_all, sh->E, rank, peer_keys};
  return cuda_status(launch_ep_dispatch(x, topk_idx, offsets, slot_pos, recv_off,
                                        reinterpret_cast<uint16_t* const*>(peer_x), ret_row, sh->T * sh->k, sh->k,
                                        sh->d_model, sh->E / world, sms, s, by_prob ? &keys : nullptr));
}

moe_status moe_ep_select(const moe_shape* sh, int32_t world, const int32_t* counts_all, const int32_t* owner_off,
                         const uint64_t* keys, const moe_bf16* x_recv, moe_bf16* x_kept, int32_t* kept_off,
                         int32_t* row_map, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (world < 1 || world > 32 || sh->E % world) return MOE_ERR_INVALID_ARG;
  if (!(sh->capacity_factor > 0.f)) return MOE_ERR_INVALID_ARG;
  if (sh->drop_policy > MOE_DROP_BY_ORDER) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_i32(counts_all));
  MOE_TRY(check_i32(owner_off));
  MOE_TRY(check_bf16(x_recv));
  MOE_TRY(check_bf16(x_kept));
  MOE_TRY(check_i32(kept_off));
  MOE_TRY(check_i32(row_map));
  if (sh->drop_policy == MOE_DROP_BY_PROB) MOE_TRY(check_bf16(keys));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_ep_select(counts_all, world, sh->E, sh->k, sh->capacity_factor, sh->drop_policy, owner_off,
                                      keys, sh->E / world, kept_off, row_map, x_recv, x_kept, sh->d_model, sms,
                                      (cudaStream_t)stream));
}

moe_status moe_ep_combine_cap(const moe_shape* sh, int32_t world, const int32_t* topk_idx, const float* topk_w,
                              const int32_t* ret_row, const int32_t* const* peer_map, const moe_bf16* const* peer_y,
                              moe_bf16* y, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (world < 1 || world > 32 || sh->E % world) return MOE_ERR_INVALID_ARG;
  if (sh->T == 0) return MOE_OK;
  MOE_TRY(check_i32(topk_idx));
  MOE_TRY(check_i32(topk_w));
  MOE_TRY(check_i32(ret_row));
  MOE_TRY(check_bf16(peer_map));
  MOE_TRY(check_bf16(peer_y));
  MOE_TRY(check_bf16(y));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_ep_combine(topk_idx, topk_w, ret_row, reinterpret_cast<const uint16_t* const*>(peer_y),
                                       y, sh->T, sh->k, sh->d_model, sh->E / world, sms, (cudaStream_t)stream,
                                       peer_map));
}

moe_status moe_router_stats(const moe_shape* sh, const int32_t* topk_idx, int32_t* slot_counts, int32_t* pair_counts,
                            int32_t accumulate, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  MOE_TRY(check_i32(slot_counts));
  if (pair_counts && (sh->k < 2 || !aligned(pair_counts, 4))) return MOE_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return MOE_ERR_INVALID_ARG;
  if (sh->T > 0) MOE_TRY(check_i32(topk_idx));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_router_stats(topk_idx, sh->T, sh->E, sh->k, slot_counts, pair_counts, accumulate != 0,
                                         sms, (cudaStream_t)stream));
}

moe_status moe_quantize_q4(const moe_bf16* W, int32_t E, int32_t R, int32_t K, uint8_t* codes, moe_bf16* scales,
                           moe_stream_t stream) {
  if (E < 1 || E > 32 || R < 8 || R > 65536 || R % 8 || K < 64 || K > 65536 || K % 64) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_bf16(W));
  MOE_TRY(check_bf16(codes));
  MOE_TRY(check_bf16(scales));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  return cuda_status(launch_quantize_q4(W, E, R, K, codes, scales, (cudaStream_t)stream));
}

size_t moe_workspace_size_q4(const moe_shape* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return layout_of(shape, true).total;
}

moe_status moe_grouped_swiglu_q4(const moe_shape* sh, const moe_bf16* x_perm, const int32_t* offsets,
                                 const uint8_t* W1c, const moe_bf16* W1s, const uint8_t* W3c, const moe_bf16* W3s,
                                 const uint8_t* W2c, const moe_bf16* W2s, moe_bf16* h, moe_bf16* y_perm, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  const ExpertWeights Wt{nullptr, nullptr, nullptr, W1c, W3c, W2c, W1s, W3s, W2s};
  MOE_TRY(check_bf16(x_perm));
  MOE_TRY(check_i32(offsets));
  MOE_TRY(check_q4_weights(Wt));
  MOE_TRY(check_bf16(h));
  MOE_TRY(check_bf16(y_perm));
  MOE_TRY(check_ws(sh, ws, ws_bytes, true));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh, true);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, 16, s)));
  MOE_TRY(run_gemms_q4(sh, L, x_perm, offsets, Wt, h, ws, sms, s));
  const int64_t S = sh->T * sh->k;
  return cuda_status(launch_splitk_reduce(at<float>(ws, L.partials), L.eff_splits, S * (int64_t)sh->d_model, offsets,
                                          sh->E, y_perm, S, sh->d_model, sms, s, at<uint32_t>(ws, L.status)));
}

static moe_status check_layer_q4(const moe_shape* sh, const moe_bf16* x, const float* Wg, const ExpertWeights& W,
                                 const moe_bf16* y, const void* ws, size_t ws_bytes, int* sms) {
  MOE_TRY(check_bf16(x));
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_q4_weights(W));
  MOE_TRY(check_bf16(y));
  MOE_TRY(check_ws(sh, ws, ws_bytes, true));
  return check_device(sms);
}

moe_status moe_layer_forward_q4(const moe_shape* sh, const moe_bf16* x, const float* Wg, const uint8_t* W1c,
                                const moe_bf16* W1s, const uint8_t* W3c, const moe_bf16* W3s, const uint8_t* W2c,
                                const moe_bf16* W2s, moe_bf16* y, int32_t* topk_idx_out, int32_t* counts_out,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  const ExpertWeights Wt{nullptr, nullptr, nullptr, W1c, W3c, W2c, W1s, W3s, W2s};
  if (topk_idx_out && !aligned(topk_idx_out, 4)) return MOE_ERR_INVALID_ARG;
  if (counts_out && !aligned(counts_out, 4)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  MOE_TRY(check_layer_q4(sh, x, Wg, Wt, y, ws, ws_bytes, &sms));
  return layer_forward_impl(sh, x, Wg, Wt, true, y, topk_idx_out, counts_out, ws, sms, (cudaStream_t)stream);
}

moe_status moe_layer_forward_q4_host(const moe_shape* sh, const moe_bf16* x_host, const float* Wg, const uint8_t* W1c,
                                     const moe_bf16* W1s, const uint8_t* W3c, const moe_bf16* W3s, const uint8_t* W2c,
                                     const moe_bf16* W2s, moe_bf16* y_host, void* ws, size_t ws_bytes,
                                     moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  const ExpertWeights Wt{nullptr, nullptr, nullptr, W1c, W3c, W2c, W1s, W3s, W2s};
  MOE_TRY(check_bf16(Wg));
  MOE_TRY(check_q4_weights(Wt));
  MOE_TRY(check_ws(sh, ws, ws_bytes, true));
  int sms = 0;
  MOE_TRY(check_device(&sms));
  const Layout L = layout_of(sh, true);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = 2 * (size_t)sh->T * sh->d_model;
  moe_bf16* xd = at<moe_bf16>(ws, L.x_stage);
  moe_bf16* yd = at<moe_bf16>(ws, L.y_stage);
  MOE_TRY(cuda_status(cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s)));
  MOE_TRY(layer_forward_impl(sh, xd, Wg, Wt, true, yd, nullptr, nullptr, ws, sms, s));
  return cuda_status(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, s));
}

moe_status moe_layer_forward_q4_profiled(const moe_shape* sh, const moe_bf16* x, const float* Wg, const uint8_t* W1c,
                                         const moe_bf16* W1s, const uint8_t* W3c, const moe_bf16* W3s,
                                         const uint8_t* W2c, const moe_bf16* W2s, moe_bf16* y, void* const* events,
                                         void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_shape(sh));
  if (sh->T == 0) return MOE_OK;
  const ExpertWeights Wt{nullptr, nullptr, nullptr, W1c, W3c, W2c, W1s, W3s, W2s};
  if (!events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  MOE_TRY(check_layer_q4(sh, x, Wg, Wt, y, ws, ws_bytes, &sms));
  return layer_forward_impl(sh, x, Wg, Wt, true, y, nullptr, nullptr, ws, sms, (cudaStream_t)stream,
                            reinterpret_cast<cudaEvent_t const*>(events));
}

moe_status moe_read_device_status(const void* ws, moe_stream_t stream) {
  if (!ws || !aligned(ws, kAlign)) return MOE_ERR_WORKSPACE;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  return v == 0 ? MOE_OK : (moe_status)v;
}

int32_t moe_debug_build(void) { return kDebugBuild ? 1 : 0; }

moe_status moe_debug_workspace_arm(const moe_shape* sh, void* ws, size_t ws_bytes, int32_t q4, moe_stream_t stream) {
#ifndef MOE_DEBUG
  (void)sh, (void)ws, (void)ws_bytes, (void)q4, (void)stream;
  return MOE_ERR_UNSUPPORTED;
#else
  MOE_TRY(check_shape(sh));
  MOE_TRY(check_ws(sh, ws, ws_bytes, q4 != 0));
  const Layout L = layout_of(sh, q4 != 0);
  for (int i = 0; i < L.nguards; ++i)
    MOE_TRY(cuda_status(cudaMemsetAsync(at<uint8_t>(ws, L.guards[i]), kGuardByte, kGuard, (cudaStream_t)stream)));
  return MOE_OK;
#endif
}

moe_status moe_debug_workspace_check(const moe_shape* sh, const void* ws, size_t ws_bytes, int32_t q4,
                                     moe_stream_t stream) {
#ifndef MOE_DEBUG
  (void)sh, (void)ws, (void)ws_bytes, (void)q4, (void)stream;
  return MOE_ERR_UNSUPPORTED;
#else
  MOE_TRY(check_shape(sh));
  MOE_TRY(check_ws(sh, ws, ws_bytes, q4 != 0));
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  const Layout L = layout_of(sh, q4 != 0);
  unsigned char buf[kGuard];
  for (int i = 0; i < L.nguards; ++i) {
    if (cudaMemcpy(buf, static_cast<const uint8_t*>(ws) + L.guards[i], kGuard, cudaMemcpyDeviceToHost) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (size_t j = 0; j < kGuard; ++j)
      if (buf[j] != kGuardByte) return MOE_ERR_WORKSPACE;
  }
  return MOE_OK;
#endif
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported device or request";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_BOUNDS: return "device-side bounds check failed (debug build)";
  }
  return "unknown status";
}

}  // extern "C"
