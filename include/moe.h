/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse mixture-of-experts layer.
 *
 * The layer (Mixtral style): for each token x_t (a row of x),
 *   logits_t = x_t . Wg^T                     (fp32 router, E experts)
 *   idx_t    = the k experts of largest logit (k = 2 for Mixtral)
 *   w_t      = softmax over those k logits    (gate weights, sum to 1)
 *   y_t      = sum_j w_tj * Expert_{idx_tj}(x_t),
 *   Expert_e(v) = W2_e (SiLU(W1_e v) * (W3_e v)),  SiLU(a) = a * sigmoid(a)
 * with an optional per-expert capacity: at most floor(cf * T * k / E) slots
 * per expert, an overflowed slot contributing zero (the token passes through
 * on the residual path outside this layer).
 *
 * Sources (web pages, by title and section):
 *   "Mixtral and Mixture-of-Experts, Explained", "How it works" -- the gate
 *       G(x) = Softmax(TopK(x . W_g)) and y = sum_i G(x)_i Expert_i(x).
 *   "How Mixtral 8x7B uses mixture of experts", "The architecture in one
 *       diagram" (top-2 of the router softmax, renormalised; batch tokens by
 *       expert, run experts, scatter back) and "Routing without auxiliary
 *       loss" (capacity factor; excess tokens dropped; sorted by router
 *       probability per expert).
 *   "Mixtral" (vanos001), "MoE Layer" (MixtralMoE / MixtralExpert: bias-free
 *       nn.Linear router [E, d]; expert w2(silu(w1 x) * w3 x)) and "SwiGLU
 *       Experts".
 *
 * Conventions for every entry point
 *   - Layouts are row-major.  x [T, d]; Wg [E, d] (fp32); W1, W3 [E, f, d];
 *     W2 [E, d, f]; slot s = t * k + j, j = 0 the larger logit.
 *   - Matrices of bf16 are passed as raw 16-bit patterns (moe_bf16).
 *   - All pointers are DEVICE pointers unless the name ends in _host.  The
 *     caller allocates every buffer, including the workspace; the library
 *     allocates no memory and keeps no state between calls apart from cached
 *     device attributes, driver entry points and the copy streams of
 *     moe_layer_forward_host's chunked calls.
 *   - Calls are asynchronous on `stream`; none synchronises except
 *     moe_read_device_status.  A workspace may serve one call in flight at a
 *     time.
 *   - Host threads: the first call on each device fills a small per-device
 *     cache (compute capability and SM count; for moe_permute_noalloc also
 *     its scratch address; moe_layer_forward_host's copy streams are created
 *     under a lock).  Make one call on each device from a single thread
 *     before calling from several threads at once; afterwards calls
 *     from different threads are independent if their buffers, workspaces
 *     and streams are (not moe_permute_noalloc: all its calls share one
 *     scratch array).
 *   - Arguments are checked before any work is queued; on failure the call
 *     returns the status and queues nothing.  T == 0 is a no-op (MOE_OK).
 *     Requirements: 1 <= E <= 32, 1 <= k <= min(E, 8), d_model and d_ff
 *     multiples of 64 in [64, 65536], T * k < 2^30, finite capacity_factor,
 *     bf16 / fp32 matrices 16-byte aligned, int32 arrays 4-byte aligned,
 *     workspace 256-byte aligned and at least moe_workspace_size() bytes.
 *   - A queued kernel that fails to launch gives MOE_ERR_CUDA.  Device-side
 *     waits are bounded; one that gives up writes MOE_ERR_TIMEOUT into the
 *     workspace's status word (read it with moe_read_device_status) and the
 *     kernel returns without trapping.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same handle as cudaStream_t */
typedef uint16_t moe_bf16;                /* raw bfloat16 bits */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or enum */
  MOE_ERR_UNSUPPORTED = 2, /* valid request the library does not handle (e.g. not sm_100) */
  MOE_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  MOE_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  MOE_ERR_BOUNDS = 6       /* a device-side bounds check failed (debug build only) */
} moe_status;

/* Which slots an overfull expert drops (capacity mode only). */
typedef enum {
  MOE_DROP_BY_PROB = 0, /* keep the cap slots of highest router probability
                           (full softmax over E), ties to the smaller token */
  MOE_DROP_BY_ORDER = 1, /* keep the first cap slots in token order */
  /* The same two policies with a next-best-expert fallback ("How Mixtral 8x7B
   * uses mixture of experts", "Routing without auxiliary loss": slots beyond
   * a full expert's capacity go to a fallback, usually the token's next-best
   * expert).  After the capacity pass,
   * the dropped slots of a token, in slot order, move to its experts at
   * router ranks k, k+1, ... (logit descending, index ascending); at each
   * expert they compete under the same policy (probability of that expert,
   * or token order) for the capacity the first pass left; a moved slot keeps
   * its gate weight; one that does not fit is dropped.  Whole-layer entry
   * points only (moe_permute returns MOE_ERR_UNSUPPORTED). */
  MOE_DROP_BY_PROB_NEXT_BEST = 2,
  MOE_DROP_BY_ORDER_NEXT_BEST = 3
} moe_drop_policy;

/* Expert-GEMM schedule.  Both compute the same function. */
typedef enum {
  MOE_VARIANT_AUTO = 0,         /* STREAM when T <= 128, TILED_SINGLE while T*k/E <= 112, TILED above */
  MOE_VARIANT_TILED = 1,        /* 256-token x 256-column tiles on CTA pairs
                                   (one MMA over two SMs): compute-bound sizes */
  MOE_VARIANT_STREAM = 2,       /* weights as the 128-row MMA operand, tokens as N,
                                   split-K on the down projection: weight-streaming sizes */
  MOE_VARIANT_TILED_SINGLE = 3  /* 128-token x 256-column tiles on single CTAs */
} moe_gemm_variant;

typedef struct {
  int64_t T;               /* tokens (rows of x) */
  int32_t d_model;         /* d: hidden size */
  int32_t d_ff;            /* f: expert inner size */
  int32_t E;               /* experts */
  int32_t k;               /* experts per token */
  float capacity_factor;   /* <= 0: dropless (default); else cap = floor(cf*T*k/E) */
  int32_t drop_policy;     /* moe_drop_policy */
  int32_t gemm_variant;    /* moe_gemm_variant */
} moe_shape;

/* Bytes of workspace every entry point below accepts for this shape
 * (moe_layer_forward needs all of it; the stage entry points use parts).
 * Returns 0 if the shape is invalid. */
MOE_API size_t moe_workspace_size(const moe_shape *shape);

/* Router and gate.  Source: "Mixtral and Mixture-of-Experts, Explained",
 * "How it works" (G(x) = Softmax(TopK(x . W_g))); "Mixtral", "MoE Layer"
 * (topk of the logits, softmax over the k kept ones).
 *   x [T, d] bf16, Wg [E, d] fp32                                   (in)
 *   logits [T, E] fp32, may be NULL                                  (out)
 *   topk_idx [T, k] int32: experts by descending logit, equal logits
 *            ordered by the smaller index                            (out)
 *   topk_w [T, k] fp32: softmax over the k kept logits               (out)
 *   topk_p [T, k] fp32: softmax over all E logits at the kept experts
 *            (the capacity priority)                                 (out)
 *   counts [E] int32: slots routed to each expert (histogram)        (out)
 * Logits are accumulated in fp32. */
MOE_API moe_status moe_router_topk(const moe_shape *shape, const moe_bf16 *x, const float *Wg,
                           float *logits, int32_t *topk_idx, float *topk_w, float *topk_p,
                           int32_t *counts, moe_stream_t stream);

/* Capacity and grouping of slots by expert.  Source: "How Mixtral 8x7B uses
 * mixture of experts", "The architecture in one diagram" (batch tokens by
 * expert) and "Routing without auxiliary loss" (capacity, drop).
 *   x [T, d], topk_idx [T, k], counts [E] (from moe_router_topk)    (in)
 *   topk_p [T, k]: read only in capacity mode with MOE_DROP_BY_PROB,
 *            may be NULL otherwise                                   (in)
 *   offsets [E + 1]: rows of expert e are offsets[e] .. offsets[e+1]-1;
 *            offsets[E] = kept slots N                               (out)
 *   slot_pos [T * k]: row of slot s, or -1 if dropped                (out)
 *   perm_slot [T * k]: slot of row r for r < N (rest untouched)      (out)
 *   x_perm [T * k, d]: x_perm[r] = x[perm_slot[r] / k] for r < N     (out)
 * Rows of one expert are in ascending token order. */
MOE_API moe_status moe_permute(const moe_shape *shape, const moe_bf16 *x, const int32_t *topk_idx,
                       const float *topk_p, const int32_t *counts, int32_t *offsets,
                       int32_t *slot_pos, int32_t *perm_slot, moe_bf16 *x_perm, void *ws,
                       size_t ws_bytes, moe_stream_t stream);

/* moe_permute without a workspace argument, for callers that cannot
 * allocate device memory: for example an inference-engine plug-in whose
 * enqueue step is handed only input/output pointers and a stream, or a
 * latency-critical loop that must never enter the CUDA allocator (cudaMalloc
 * can synchronise the device and take unbounded time).  The pages have no
 * counterpart of this entry point; it exists for such callers.
 *
 * Same arguments (minus ws / ws_bytes), results and ordering as moe_permute.
 * Its scratch (look-back words, tile ticket, capacity thresholds) is a fixed
 * array of about 129 KB in the library's device memory, present on every GPU
 * that loads the library until the process exits.  Limits: T * k <= 65536
 * slots (E <= 32 as everywhere); larger shapes return MOE_ERR_UNSUPPORTED and
 * queue nothing.  The first call on each device looks up the array's device
 * address (a host-side runtime query, no allocation); make that first call
 * before any stream capture.  All calls share the one array and it keeps the
 * last call's contents: each call clears what must start at zero, and calls
 * whose work overlaps on the GPU (other streams, other host threads) race on
 * it, so serialise them.  A device-side look-back wait that gives up is
 * recorded in that shared array; moe_permute_noalloc_status reads it.  The
 * looked-up address belongs to the device's context as it was at that first
 * call: after cudaDeviceReset (or any other teardown of the device's primary
 * context) in the same process, the address is stale and this entry point
 * must not be called on that device again. */
MOE_API moe_status moe_permute_noalloc(const moe_shape *shape, const moe_bf16 *x,
                                       const int32_t *topk_idx, const float *topk_p,
                                       const int32_t *counts, int32_t *offsets, int32_t *slot_pos,
                                       int32_t *perm_slot, moe_bf16 *x_perm, moe_stream_t stream);

/* Device status of the last moe_permute_noalloc call on the current device
 * (the pages have no counterpart): synchronises `stream`, then reads the
 * status word of the shared scratch array.  MOE_OK, or MOE_ERR_TIMEOUT if a
 * look-back wait of that call gave up (its outputs are then invalid), or
 * MOE_ERR_CUDA if the stream reports an error.  Each moe_permute_noalloc
 * call clears the word first, so only the most recent call is reported;
 * before any call on the device it returns MOE_OK.  Allocates nothing. */
MOE_API moe_status moe_permute_noalloc_status(moe_stream_t stream);

/* Grouped SwiGLU experts on tensor cores.  Source: "Mixtral", "MoE Layer"
 * (MixtralExpert.forward) and "SwiGLU Experts".  For each expert e and row r
 * in offsets[e] .. offsets[e+1]-1:
 *   h[r]      = SiLU(x_perm[r] . W1[e]^T) * (x_perm[r] . W3[e]^T)   [f] bf16
 *   y_perm[r] = h[r] . W2[e]^T                                        [d] bf16
 * bf16 operands, fp32 accumulation, results rounded to bf16 (nearest even).
 * Rows r >= offsets[E] of h and y_perm are left untouched.
 * Precondition (not checked: offsets live on the device): offsets[0] = 0,
 * offsets non-decreasing and offsets[E] <= T * k, as moe_permute writes
 * them.  Other offsets make the kernels read and write outside the buffers. */
MOE_API moe_status moe_grouped_swiglu(const moe_shape *shape, const moe_bf16 *x_perm,
                              const int32_t *offsets, const moe_bf16 *W1, const moe_bf16 *W3,
                              const moe_bf16 *W2, moe_bf16 *h, moe_bf16 *y_perm, void *ws,
                              size_t ws_bytes, moe_stream_t stream);

/* Gate-weighted combine.  Source: "Mixtral and Mixture-of-Experts,
 * Explained", "How it works" (y = sum_i G(x)_i Expert_i(x)).
 *   y[t] = sum over j with slot_pos[t*k+j] >= 0 of
 *          topk_w[t, j] * y_perm[slot_pos[t*k+j]]
 * accumulated in fp32 in slot order, stored bf16; y[t] = 0 when every slot
 * of t was dropped.  The remaining weights are not renormalised.
 * Precondition (not checked): every slot_pos entry is -1 or a row < T * k of
 * y_perm, as moe_permute writes them. */
MOE_API moe_status moe_combine(const moe_shape *shape, const moe_bf16 *y_perm, const int32_t *slot_pos,
                       const float *topk_w, moe_bf16 *y, moe_stream_t stream);

/* The whole layer: router, capacity, grouping, experts, combine, all
 * intermediates in the workspace.  y [T, d] bf16 (out).  topk_idx_out
 * [T, k] and counts_out [E] (both may be NULL) receive the routing. */
MOE_API moe_status moe_layer_forward(const moe_shape *shape, const moe_bf16 *x, const float *Wg,
                             const moe_bf16 *W1, const moe_bf16 *W3, const moe_bf16 *W2,
                             moe_bf16 *y, int32_t *topk_idx_out, int32_t *counts_out, void *ws,
                             size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward, also recording CUDA events on `stream` between its
 * kernels, for timing each kernel inside a real forward pass.  events[6]
 * are cudaEvent_t handles the caller created (timing enabled):
 *   [0] before the router        [1] after the router
 *   [2] after capacity selection and grouping by expert
 *   [3] after the gate/up-projection GEMM (SiLU * mul fused)
 *   [4] after the down-projection GEMM    [5] after the combine.
 * The two expert GEMMs also record, from their first CTA, the SM cycle
 * counter and the global nanosecond timer at entry and exit: 64-bit words
 * at byte 64 of ws, {cycles, ns} at entry then at exit for the gate/up GEMM
 * (bytes 64 .. 95) and for the down GEMM (96 .. 127); (cycles difference) /
 * (ns difference) is the SM clock in GHz the GEMM ran at.  The kernels after
 * the router are not chained by programmatic launch here (the events sit
 * between them).  Same arguments and results as moe_layer_forward otherwise. */
MOE_API moe_status moe_layer_forward_profiled(const moe_shape *shape, const moe_bf16 *x,
                                              const float *Wg, const moe_bf16 *W1,
                                              const moe_bf16 *W3, const moe_bf16 *W2, moe_bf16 *y,
                                              void *const *events, void *ws, size_t ws_bytes,
                                              moe_stream_t stream);

/* The whole layer with the activations in HOST memory: copies x_host
 * [T, d] to the device (inside the workspace), runs moe_layer_forward and
 * copies y back to y_host [T, d].  Weights are device pointers.  Use
 * page-locked host buffers for asynchronous copies; y_host is valid once
 * `stream` has been synchronised.
 * Dropless calls (capacity_factor <= 0) with T >= 4096 on the CTA-pair
 * schedule run the layer on 2 to 8 consecutive groups of at least 2048
 * tokens.  Each group's copies run on two copy streams that the library
 * creates once per device and calling stream (up to 8 calling streams per
 * device; further ones share; kept for the process and invalid after a
 * device reset) and overlap the other groups' kernels.  y is the same, bit for
 * bit: in dropless mode no token's result depends on the others.  All of
 * the call's work is ordered before later work on `stream`, and it waits
 * for earlier work on `stream`.  Otherwise everything is queued on
 * `stream`.  To capture such a call in a CUDA graph, make one call on the
 * same stream outside the capture first (it creates the copy streams). */
MOE_API moe_status moe_layer_forward_host(const moe_shape *shape, const moe_bf16 *x_host,
                                  const float *Wg, const moe_bf16 *W1, const moe_bf16 *W3,
                                  const moe_bf16 *W2, moe_bf16 *y_host, void *ws,
                                  size_t ws_bytes, moe_stream_t stream);

/* Router statistics of one layer's top-k indices (device topk_idx [T, k], as
 * written by moe_router_topk or returned by moe_layer_forward):
 *   slot_counts [k, E] int32 (out): slot_counts[j][e] = number of tokens whose
 *       j-th choice (j = 0 the largest logit) is expert e.  The sum over j is
 *       the bincount of the flattened top-k indices, i.e. the layer's counts.
 *   pair_counts [E, E] int32 (out, nullable, needs k >= 2): pair_counts[a][b] =
 *       number of tokens whose first two choices are (a, b).
 * accumulate = 0 overwrites the outputs, 1 adds to them (e.g. over batches,
 * or into row `layer` of a [layers, ...] table).  The most common expert of
 * position j is the argmax of slot_counts[j].  Sources: "How Mixtral 8x7B
 * uses mixture of experts", "Expert specialization" (per-layer bincount of the
 * top-2 indices) and "Mixtral 8x7B — MoE Complete Guide", "Inspecting Expert
 * Routing" (most common expert per top-k position).  Indices outside [0, E)
 * are not counted.  Asynchronous on `stream`; allocates nothing.  T == 0
 * only clears the outputs (accumulate = 0). */
MOE_API moe_status moe_router_stats(const moe_shape *shape, const int32_t *topk_idx, int32_t *slot_counts,
                                    int32_t *pair_counts, int32_t accumulate, moe_stream_t stream);

/* ------------------------------------------------------ expert parallelism
 * Sources: "How Mixtral 8x7B uses mixture of experts", "Tensor parallelism vs
 * expert parallelism" (the experts are divided among the GPUs; an all-to-all
 * sends every token to the ranks owning its experts and a second one brings
 * the results back; expert_parallel_forward: router, dispatch, local
 * experts, combine).
 *
 * `world` ranks, one per GPU; rank o owns experts o*epr .. o*epr+epr-1 with
 * epr = E / world (E % world == 0, world <= 32).  Dropless only.  One layer
 * step on rank r (the caller provides the collectives and barriers):
 *   1. moe_router_topk on its own tokens -> topk_idx, topk_w, counts [E];
 *   2. all-gather the counts of every rank into counts_all [world, E];
 *   3. moe_ep_plan -> recv_off [E] and owner_off [epr + 1];
 *   4. moe_ep_dispatch: stores each slot's token row into its owner's
 *      receive buffer x_recv (peer memory) and records the row in ret_row;
 *   5. barrier; moe_grouped_swiglu on this rank's x_recv with owner_off, its
 *      local experts' weights, a shape with E = epr, k = 1 and T = the
 *      receive buffer's rows, writing y_recv;
 *   6. barrier; moe_ep_combine: y[t] = sum_j w[t, j] * y_recv of the owner at
 *      ret_row (peer memory), fp32 in slot order, one bf16 rounding.
 * An owner's receive buffer holds its experts' rows expert by expert, the
 * source ranks in rank order within an expert, each in token order; it needs
 * room for every slot that can reach it (at most the sum over ranks of T*k).
 * The dispatch and combine kernels never wait on another rank. */

/* counts_all [world, E] int32 (device) -> recv_off [E]: start row of this
 * rank's slots of expert e in the receive buffer of e's owner; owner_off
 * [epr + 1]: row ranges of this rank's local experts in its own receive
 * buffer. */
MOE_API moe_status moe_ep_plan(const int32_t *counts_all, int32_t E, int32_t rank, int32_t world,
                               int32_t *recv_off, int32_t *owner_off, moe_stream_t stream);

/* shape: this rank's T, the global E, k (capacity_factor must be <= 0; with
 * a capacity use moe_ep_dispatch_cap).
 * x [T, d], topk_idx [T, k], counts [E] from moe_router_topk; recv_off from
 * moe_ep_plan; peer_x: DEVICE array of `world` device pointers, entry o the
 * receive buffer [rows, d] bf16 of rank o (this rank's own included).
 * ret_row [T, k] int32 (out).  ws: at least moe_workspace_size(shape).
 * Precondition (not checked): counts and recv_off come from this step's
 * moe_router_topk and moe_ep_plan, and every owner's buffer has room for the
 * rows the plan gives it. */
MOE_API moe_status moe_ep_dispatch(const moe_shape *shape, int32_t world, const moe_bf16 *x,
                                   const int32_t *topk_idx, const int32_t *counts, const int32_t *recv_off,
                                   moe_bf16 *const *peer_x, int32_t *ret_row, void *ws, size_t ws_bytes,
                                   moe_stream_t stream);

/* peer_y: DEVICE array of `world` device pointers, entry o the expert output
 * buffer y_recv [rows, d] bf16 of rank o.  y [T, d] bf16 (out). */
MOE_API moe_status moe_ep_combine(const moe_shape *shape, int32_t world, const int32_t *topk_idx,
                                  const float *topk_w, const int32_t *ret_row, const moe_bf16 *const *peer_y,
                                  moe_bf16 *y, moe_stream_t stream);

/* Expert parallelism with a capacity (capacity_factor > 0; policies
 * MOE_DROP_BY_PROB and MOE_DROP_BY_ORDER).  Sources: "How Mixtral 8x7B uses
 * mixture of experts", "Routing without auxiliary loss" (each expert keeps at
 * most cf x (tokens x k / E) slots, the rest are dropped) and "Tensor
 * parallelism vs expert parallelism".  The ranks' tokens form one batch,
 * their concatenation in rank order (token t of rank r is token
 * t_base(r) + t, t_base(r) = the tokens of ranks 0 .. r-1), and the layer is
 * the single-device layer on that batch: cap = floor(cf * T_all * k / E)
 * with T_all the tokens of all ranks, and the kept slots of an expert are
 * the cap of largest full-softmax probability (ties: the smaller batch
 * index) or the first cap in batch order.  Only the owner of an expert sees
 * all of its slots, so it decides:
 *   1. moe_router_topk, counts all-gathered, moe_ep_plan (as dropless);
 *   2. moe_ep_dispatch_cap: every slot's row to its owner as in
 *      moe_ep_dispatch, and (by probability) its priority key to the same
 *      row of the owner's key buffer;
 *   3. barrier; on the owner, moe_ep_select: row_map [rows] (kept row or -1)
 *      and kept_off [epr + 1], the kept rows gathered into x_kept; then
 *      moe_grouped_swiglu on x_kept with kept_off;
 *   4. barrier; moe_ep_combine_cap: as moe_ep_combine, each slot's row
 *      passed through its owner's row_map; a dropped slot adds zero and the
 *      other gates are not renormalised.
 * Buffers of `rows` rows (the sum over ranks of T*k at most): x_recv, keys,
 * row_map and the kept-row output y_kept must be reachable by every rank
 * (peer arrays); x_kept and h are the owner's own. */

/* shape: this rank's T, the global E, k, capacity_factor > 0 and the drop
 * policy; counts_all [world, E] as for moe_ep_plan; topk_p [T, k] from
 * moe_router_topk (by probability); peer_keys: DEVICE array of `world`
 * device pointers to the owners' key buffers [rows] uint64 (by probability;
 * may be NULL by order).  Other arguments and preconditions as
 * moe_ep_dispatch.  The next-best fallback policies give
 * MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_ep_dispatch_cap(const moe_shape *shape, int32_t world, int32_t rank,
                                       const int32_t *counts_all, const moe_bf16 *x, const int32_t *topk_idx,
                                       const float *topk_p, const int32_t *counts, const int32_t *recv_off,
                                       moe_bf16 *const *peer_x, uint64_t *const *peer_keys, int32_t *ret_row,
                                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Owner side of the capacity (after the dispatch's barrier).  shape: the
 * global E, k, d_model, capacity_factor and policy (T is not used);
 * counts_all and owner_off from this step; keys [rows] this rank's key
 * buffer (by probability); x_recv [rows, d] its receive buffer.  Out:
 * x_kept [rows, d], kept_off [epr + 1] int32, row_map [rows] int32.
 * Allocates nothing; 1 + 1 kernels on `stream`. */
MOE_API moe_status moe_ep_select(const moe_shape *shape, int32_t world, const int32_t *counts_all,
                                 const int32_t *owner_off, const uint64_t *keys, const moe_bf16 *x_recv,
                                 moe_bf16 *x_kept, int32_t *kept_off, int32_t *row_map, moe_stream_t stream);

/* peer_map: DEVICE array of `world` device pointers to the owners' row_map;
 * peer_y: to the owners' outputs of moe_grouped_swiglu on x_kept.  Otherwise
 * as moe_ep_combine. */
MOE_API moe_status moe_ep_combine_cap(const moe_shape *shape, int32_t world, const int32_t *topk_idx,
                                      const float *topk_w, const int32_t *ret_row,
                                      const int32_t *const *peer_map, const moe_bf16 *const *peer_y,
                                      moe_bf16 *y, moe_stream_t stream);

/* ---------------------------------------------------------------- 4-bit experts
 * Sources: "How Mixtral 8x7B uses mixture of experts", "Deployment tradeoffs
 * you'll actually hit" / "Quantization asymmetry" (keep the router in 16-bit
 * precision, quantise the experts to 4 bits) and "Mixtral 8x7B — MoE
 * Complete Guide", "4-bit Quantization for Single GPU" (4-bit weights, bf16
 * arithmetic, block-wise absmax scales).
 *
 * Format of one 4-bit matrix W [E, R, K] (K a multiple of 64, R of 8):
 *   codes  [E, R, K/2] bytes, 16-byte aligned.  The codes of inputs 8g ..
 *          8g+7 of a row fill one little-endian 32-bit word: nibble m (bits
 *          4m .. 4m+3) holds input 8g + 2m, nibble m + 4 input 8g + 2m + 1.
 *   scales [E, K/64, R] bf16, 16-byte aligned: one scale per 64 consecutive
 *          inputs of a row, stored block-major.
 *   w = (code - 8) * scale, code in 0 .. 15.
 * The expert matrices are W1, W3 [E, d_ff, d_model] and W2 [E, d_model, d_ff]
 * as in the bf16 entry points; the router stays fp32.  Arithmetic on the
 * GPU: at token tiles of 16 and 32 (16 while the mean slots per expert,
 * T k / E, fit it, 32 up to a mean of 22, else twice the mean rounded up
 * to 16: T <= 88 for 8 experts and top-2), the weights stay
 * exact integers (code - 8) and each token slot's
 * activations are rounded to 16-bit integers with one fp32 scale per slot
 * (error at most half a step, 1.5e-5 of the slot's largest value); the
 * per-64-input integer sums are exact and are scaled and added in fp32.  For
 * larger tiles each dequantised weight is rounded to bf16 and the GEMM
 * accumulates in fp32. */

/* Quantises W [E, R, K] bf16 (device) into codes and scales (device, out):
 * per 64-input block s = bf16(absmax / 7) and code = 8 + clamp(round half to
 * even(w / s), -8, 7), both divisions IEEE fp32; an all-zero block gets s = 0
 * and codes 8.  Requires 1 <= E <= 32, 8 <= R <= 65536 with R % 8 == 0,
 * 64 <= K <= 65536 with K % 64 == 0, finite weights.  Asynchronous on
 * `stream`; allocates nothing. */
MOE_API moe_status moe_quantize_q4(const moe_bf16 *W, int32_t E, int32_t R, int32_t K, uint8_t *codes,
                                   moe_bf16 *scales, moe_stream_t stream);

/* Workspace bytes the 4-bit entry points need for `shape` (0 if the shape is
 * invalid); for token tiles of 16 and 32 it includes the quantised
 * activations.  gemm_variant is ignored: the 4-bit GEMMs stream the weights. */
MOE_API size_t moe_workspace_size_q4(const moe_shape *shape);

/* moe_grouped_swiglu with 4-bit expert weights (W1c/W1s, W3c/W3s, W2c/W2s
 * in the format above).  h [T*k, d_ff] and y_perm [T*k, d_model] bf16 out;
 * ws of at least moe_workspace_size_q4 bytes.  Same precondition on offsets
 * as moe_grouped_swiglu. */
MOE_API moe_status moe_grouped_swiglu_q4(const moe_shape *shape, const moe_bf16 *x_perm,
                                         const int32_t *offsets, const uint8_t *W1c,
                                         const moe_bf16 *W1s, const uint8_t *W3c, const moe_bf16 *W3s,
                                         const uint8_t *W2c, const moe_bf16 *W2s, moe_bf16 *h,
                                         moe_bf16 *y_perm, void *ws, size_t ws_bytes,
                                         moe_stream_t stream);

/* moe_layer_forward with 4-bit expert weights; the router, grouping and
 * combine are those of the bf16 layer.  ws of at least moe_workspace_size_q4
 * bytes. */
MOE_API moe_status moe_layer_forward_q4(const moe_shape *shape, const moe_bf16 *x, const float *Wg,
                                        const uint8_t *W1c, const moe_bf16 *W1s, const uint8_t *W3c,
                                        const moe_bf16 *W3s, const uint8_t *W2c, const moe_bf16 *W2s,
                                        moe_bf16 *y, int32_t *topk_idx_out, int32_t *counts_out,
                                        void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward_q4 with the activations in HOST memory, as
 * moe_layer_forward_host: copies x_host [T, d] into the workspace, runs the
 * 4-bit layer and copies y back to y_host [T, d], all queued on `stream`.
 * The workspace is the one of moe_workspace_size_q4.  Use page-locked host
 * buffers; y_host is valid once the stream has been synchronised. */
MOE_API moe_status moe_layer_forward_q4_host(const moe_shape *shape, const moe_bf16 *x_host,
                                             const float *Wg, const uint8_t *W1c, const moe_bf16 *W1s,
                                             const uint8_t *W3c, const moe_bf16 *W3s, const uint8_t *W2c,
                                             const moe_bf16 *W2s, moe_bf16 *y_host, void *ws,
                                             size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward_q4 recording six CUDA events (cudaEvent_t) on `stream`
 * between its stages and the GEMMs' clock records in ws, as
 * moe_layer_forward_profiled. */
MOE_API moe_status moe_layer_forward_q4_profiled(const moe_shape *shape, const moe_bf16 *x,
                                                 const float *Wg, const uint8_t *W1c,
                                                 const moe_bf16 *W1s, const uint8_t *W3c,
                                                 const moe_bf16 *W3s, const uint8_t *W2c,
                                                 const moe_bf16 *W2s, moe_bf16 *y,
                                                 void *const *events, void *ws, size_t ws_bytes,
                                                 moe_stream_t stream);

/* Self-test of the failure reporting of the device-side waits (the pages
 * have no counterpart).  Queues one small kernel that makes an mbarrier wait
 * and a look-back wait -- the two kinds of bounded wait in the layer's
 * kernels -- give up after `limit_us` microseconds (1 .. 10^7) on a barrier
 * and a word that nothing completes.  Each records MOE_ERR_TIMEOUT in the
 * status word at the start of `ws` (the first 256 bytes are used) and returns;
 * nothing traps, and the context stays usable.  Afterwards
 * moe_read_device_status(ws) returns MOE_ERR_TIMEOUT and the 32-bit word at
 * byte offset 128 of `ws` holds 2 (the number of waits that gave up). */
MOE_API moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t limit_us,
                                             moe_stream_t stream);

/* Synchronises `stream`, then returns the device status word of the last
 * call that used this workspace (MOE_OK or MOE_ERR_TIMEOUT), or
 * MOE_ERR_CUDA if the stream reports an error. */
MOE_API moe_status moe_read_device_status(const void *ws, moe_stream_t stream);

/* ------------------------------------------------------------ debug build
 * The pages have no counterpart of this section.  The library also builds as
 * libmoe_debug.so (compiled with MOE_DEBUG): the same entry points, plus
 *   - in-kernel bounds checks on the indices the kernels derive on the device
 *     (grouped rows below offsets[e+1] and below T * k, slot rows read by the
 *     combine below T * k, token indices below T).  A failed check skips the
 *     access and records MOE_ERR_BOUNDS in the status word; nothing traps;
 *   - a 256-byte guard after each workspace region past the control region
 *     (the debug build's moe_workspace_size includes them);
 *   - a host-side stage-failure hook: with the environment variable
 *     MOE_DEBUG_FAIL_STAGE=n (1 router, 2 capacity / grouping, 3 expert
 *     GEMMs, 4 combine, 5 output copies), the whole-layer entry points return
 *     MOE_ERR_CUDA just before queuing stage n, so nothing from stage n on is
 *     queued.
 * The release library returns 0 from moe_debug_build and MOE_ERR_UNSUPPORTED
 * from the two guard calls. */
MOE_API int32_t moe_debug_build(void);

/* Debug build: fill the guards of a workspace laid out for `shape` (q4 != 0:
 * the layout of moe_workspace_size_q4) with a fixed byte pattern, queued on
 * `stream`. */
MOE_API moe_status moe_debug_workspace_arm(const moe_shape *shape, void *ws, size_t ws_bytes,
                                           int32_t q4, moe_stream_t stream);

/* Debug build: synchronise `stream` and check that every guard still holds
 * the pattern: MOE_OK, or MOE_ERR_WORKSPACE if any byte changed. */
MOE_API moe_status moe_debug_workspace_check(const moe_shape *shape, const void *ws, size_t ws_bytes,
                                             int32_t q4, moe_stream_t stream);

/* Static English text of a status code. */
MOE_API const char *moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
