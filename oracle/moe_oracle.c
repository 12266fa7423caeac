/*
 * CPU ORACLE of the Mixtral-style sparse mixture-of-experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load or run this code.  It shares
 * no code, header, table or helper with the GPU path, and the GPU path never
 * calls it.
 *
 * Every step is the plain definition, computed in double precision from the
 * same bf16 / fp32 input bytes the GPU consumes, in the order the pages state
 * it; nothing is blocked, fused or reordered.  Sources (web pages, by title):
 *
 *  [P1] "How Mixtral 8x7B uses mixture of experts" (n4n.ai)
 *       - "The architecture in one diagram": router logits -> softmax -> top-2
 *         -> renormalise; outputs weighted and summed.
 *       - "Routing without auxiliary loss": capacity factor; excess tokens are
 *         dropped; each expert keeps its slots in order of router probability
 *         until it is full.
 *  [P2] "Mixtral and Mixture-of-Experts, Explained" (automatone.win)
 *       - "How it works": G(x) = Softmax(TopK(x . W_g)), logits outside the
 *         top-k set to -inf; y = sum_i G(x)_i . Expert_i(x).
 *  [P3] "Mixtral" (vanos001.github.io)
 *       - "MoE Layer": MixtralMoE.forward (top-k of logits, softmax over the
 *         k kept logits) and MixtralExpert.forward: w2(silu(w1 x) * w3 x),
 *         all nn.Linear without bias.
 *       - "SwiGLU Experts": SwiGLU(x) = SiLU(x W1) (.) (x W3), output @ W2.
 *       - "MixtralBlock": the MoE output is added to the residual stream.
 *  [P4] "Mixtral 8x7B" (interview.clozo.ai)
 *       - "Step 2: A router picks 2 experts and mixes their outputs": the
 *         worked example (scores 2.1 0.3 1.4 -0.5 0.0 0.9 -1.2 0.2 -> weights
 *         0.6682 / 0.3318).
 *  [P5] "Mixtral 8x7B — MoE Complete Guide" (webcoderspeed.com)
 *       - "4-bit Quantization for Single GPU": 4-bit expert weights with
 *         bf16 arithmetic (the 4-bit section at the end of this file).
 *
 * Readings taken where the pages are silent or disagree (each is also tested):
 *  - Gate: [P1] (softmax over all E, top-k, renormalise), [P2] (-inf mask then
 *    softmax) and [P3] (softmax of the k largest logits) are the same function
 *    except under exact ties; this file computes the [P3] form.
 *  - Top-k order and ties: slot j = 0 holds the largest logit; equal logits
 *    are ordered by the smaller expert index.
 *  - Experts are numbered from 0 ([P4] calls the first and third scores
 *    experts 1 and 3; here they are indices 0 and 2).
 *  - SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a)).
 *  - Capacity per expert = floor(cf * T * k / E) (the pages' cf * T / E per
 *    slot of top-k); cf <= 0 means no capacity limit (dropless).
 *  - Which slots overflow: policy 0 keeps, per expert, the `cap` slots with
 *    the largest full-softmax router probability ([P1]'s sketch orders each
 *    expert's tokens by it), ties to the smaller token index; policy 1 keeps the first
 *    `cap` slots in token order.
 *  - A dropped slot contributes zero (the token passes on the residual path,
 *    [P3] MixtralBlock); the remaining gate weights are not renormalised.
 *
 * Parity unpinned (readings the pages leave open; each function is pinned
 * only against its own stated rule, by brute force and invariants, not
 * against anything the pages fix):
 *  - which slots overflow: policy 0 (router probability) against policy 1
 *    (token order); only [P1]'s comment supports policy 0;
 *  - the next-best fallback's rule (one move per dropped slot to the token's
 *    next router ranks, competing for the capacity left), which [P1] names
 *    without stating;
 *  - the bits of the 4-bit format, which [P1] and [P5] name but do not give.
 *
 * Layouts (row-major): x [T, d] bf16 bits; Wg [E, d] fp32 (logit = x . Wg[e]);
 * W1, W3 [E, f, d] bf16 bits; W2 [E, d, f] bf16 bits.  Slot s = t * k + j.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Router logits [P2] "How it works" (x . W_g) with [P3] "MoE Layer" storage
 * (nn.Linear(d_model, num_experts, bias=False) keeps W as [E, d]):
 * logits[t, e] = sum_i x[t, i] * Wg[e, i], summed in index order. */
void oracle_router_logits(int64_t T, int32_t d, int32_t E, const uint16_t *x, const float *Wg,
                          double *logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int32_t i = 0; i < d; ++i)
        acc += bf16_to_double(x[t * d + i]) * (double)Wg[(int64_t)e * d + i];
      logits[t * E + e] = acc;
    }
  }
}

/* Top-k [P3] "MoE Layer" (router_logits.topk(top_k)): the k experts with the
 * largest logits, slot j = 0 the largest; equal logits -> smaller index first.
 * Plain selection: k passes, each taking the best expert not yet chosen. */
void oracle_topk(int64_t T, int32_t E, int32_t k, const double *logits, int32_t *idx) {
  for (int64_t t = 0; t < T; ++t) {
    const double *l = logits + t * E;
    for (int32_t j = 0; j < k; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e) {
        int taken = 0;
        for (int32_t q = 0; q < j; ++q) taken |= (idx[t * k + q] == e);
        if (taken) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep smaller e */
      }
      idx[t * k + j] = best;
    }
  }
}

/* Gate weights [P3] "MoE Layer": softmax over the k kept logits,
 *   w_j = exp(l_j - m) / sum_{q<k} exp(l_q - m),  m = l_{idx_0}.
 * Router probability [P1] "The architecture in one diagram" (softmax over all
 * E logits) of each chosen expert, used as the capacity priority:
 *   p_j = exp(l_j - M) / sum_{e<E} exp(l_e - M),  M = max_e l_e. */
void oracle_gates(int64_t T, int32_t E, int32_t k, const double *logits, const int32_t *idx,
                  double *w, double *p) {
  for (int64_t t = 0; t < T; ++t) {
    const double *l = logits + t * E;
    double m = l[idx[t * k]];
    double zk = 0.0;
    for (int32_t q = 0; q < k; ++q) zk += exp(l[idx[t * k + q]] - m);
    double M = l[0];
    for (int32_t e = 1; e < E; ++e)
      if (l[e] > M) M = l[e];
    double zE = 0.0;
    for (int32_t e = 0; e < E; ++e) zE += exp(l[e] - M);
    for (int32_t j = 0; j < k; ++j) {
      w[t * k + j] = exp(l[idx[t * k + j]] - m) / zk;
      p[t * k + j] = exp(l[idx[t * k + j]] - M) / zE;
    }
  }
}

typedef struct {
  double p;
  int64_t t;
  int64_t s;
} prio_t;

/* (p descending, then t ascending) */
static int prio_cmp(const void *a, const void *b) {
  const prio_t *x = (const prio_t *)a, *y = (const prio_t *)b;
  if (x->p > y->p) return -1;
  if (x->p < y->p) return 1;
  return (x->t < y->t) ? -1 : (x->t > y->t);
}

/* Capacity [P1] "Routing without auxiliary loss": each expert takes at most
 * cap = floor(cf * T * k / E) slots; the excess is dropped.  policy 0 keeps
 * the cap slots of highest router probability p (ties: smaller token first),
 * policy 1 keeps the first cap slots in token order.  cf <= 0: keep all.
 * kept[s] = 1 / 0.  Returns cap, or -1 when dropless. */
int64_t oracle_capacity(int64_t T, int32_t E, int32_t k, double cf, int32_t policy,
                        const int32_t *idx, const double *p, uint8_t *kept) {
  int64_t S = T * k;
  if (cf <= 0.0) {
    for (int64_t s = 0; s < S; ++s) kept[s] = 1;
    return -1;
  }
  int64_t cap = (int64_t)floor(cf * (double)T * (double)k / (double)E);
  prio_t *list = (prio_t *)malloc(sizeof(prio_t) * (size_t)(S > 0 ? S : 1));
  for (int64_t s = 0; s < S; ++s) kept[s] = 0;
  for (int32_t e = 0; e < E; ++e) {
    int64_t n = 0;
    for (int64_t s = 0; s < S; ++s)
      if (idx[s] == e) {
        list[n].p = p[s];
        list[n].t = s / k;
        list[n].s = s;
        ++n;
      }
    if (policy == 0) qsort(list, (size_t)n, sizeof(prio_t), prio_cmp);
    /* policy 1: list is already in token order */
    for (int64_t r = 0; r < n && r < cap; ++r) kept[list[r].s] = 1;
  }
  free(list);
  return cap;
}

/* Next-best-expert fallback [P1] "Routing without auxiliary loss": slots
 * beyond a full expert's capacity go to a fallback, usually the token's
 * next-best expert.  Reading: after the capacity pass of oracle_capacity,
 * the dropped slots of token t, in slot order, move to t's next experts in
 * the router order (logit descending, index ascending) past its top k: the
 * first dropped slot to rank k, the second to rank k + 1, and so on (none
 * past rank E - 1).  At each expert the moved slots compete for the capacity
 * the first pass left (cap minus its kept slots) under the same policy:
 * policy 0 by the full router probability of the new expert (ties: smaller
 * token first), policy 1 in token order.  A moved slot keeps its gate weight;
 * one that does not fit is dropped.  expert[s] = the expert that processes
 * slot s (its top-k choice, or the fallback it moved to), kept[s] = 1 / 0.
 * order_override (may be NULL) [T, E]: a row whose first entry is >= 0
 * replaces that token's router order (the comparison rule for tokens with
 * near-tied logits).  Returns cap, or -1 when dropless. */
int64_t oracle_capacity_fallback(int64_t T, int32_t E, int32_t k, double cf, int32_t policy,
                                 const double *logits, const int32_t *idx, const double *p,
                                 const int32_t *order_override, int32_t *expert, uint8_t *kept) {
  int64_t S = T * k;
  int64_t cap = oracle_capacity(T, E, k, cf, policy, idx, p, kept);
  for (int64_t s = 0; s < S; ++s) expert[s] = idx[s];
  if (cap < 0) return cap;
  int64_t *used = (int64_t *)calloc((size_t)E, sizeof(int64_t));
  for (int64_t s = 0; s < S; ++s)
    if (kept[s]) used[idx[s]] += 1;
  /* candidates: moved slot s goes to cand_e[s] with probability cand_p[s] */
  int32_t *cand_e = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S > 0 ? S : 1));
  double *cand_p = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
  int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
  for (int64_t t = 0; t < T; ++t) {
    const double *l = logits + t * E;
    /* router order of all E experts: logit descending, index ascending */
    if (order_override && order_override[t * E] >= 0) {
      for (int32_t e = 0; e < E; ++e) order[e] = order_override[t * E + e];
    } else {
      for (int32_t e = 0; e < E; ++e) order[e] = e;
      for (int32_t a = 1; a < E; ++a) {
        int32_t v = order[a], b = a - 1;
        while (b >= 0 && (l[order[b]] < l[v] || (l[order[b]] == l[v] && order[b] > v))) {
          order[b + 1] = order[b];
          --b;
        }
        order[b + 1] = v;
      }
    }
    double M = l[0], zE = 0.0;
    for (int32_t e = 1; e < E; ++e)
      if (l[e] > M) M = l[e];
    for (int32_t e = 0; e < E; ++e) zE += exp(l[e] - M);
    int32_t moved = 0;
    for (int32_t j = 0; j < k; ++j) {
      int64_t s = t * k + j;
      cand_e[s] = -1;
      if (kept[s]) continue;
      int32_t r = k + moved;
      ++moved;
      if (r >= E) continue;
      cand_e[s] = order[r];
      cand_p[s] = exp(l[order[r]] - M) / zE;
    }
  }
  prio_t *list = (prio_t *)malloc(sizeof(prio_t) * (size_t)(S > 0 ? S : 1));
  for (int32_t e = 0; e < E; ++e) {
    int64_t n = 0;
    for (int64_t s = 0; s < S; ++s)
      if (cand_e[s] == e) {
        list[n].p = cand_p[s];
        list[n].t = s / k;
        list[n].s = s;
        ++n;
      }
    if (policy == 0) qsort(list, (size_t)n, sizeof(prio_t), prio_cmp);
    int64_t room = cap - used[e];
    for (int64_t r = 0; r < n && r < room; ++r) {
      kept[list[r].s] = 1;
      expert[list[r].s] = e;
    }
  }
  free(list);
  free(order);
  free(cand_p);
  free(cand_e);
  free(used);
  return cap;
}

/* Grouping of slots by expert [P1] "The architecture in one diagram" (batch
 * tokens by expert, run the experts, scatter back): for e = 0..E-1, the kept
 * slots routed to e in ascending token order form rows offsets[e] ..
 * offsets[e+1]-1 of the grouped layout.  counts[e] = routed slots (the
 * per-expert histogram), kept_counts[e] = kept slots, perm_slot[row] = slot,
 * slot_pos[slot] = row or -1 when dropped. */
void oracle_permute(int64_t T, int32_t E, int32_t k, const int32_t *idx, const uint8_t *kept,
                    int32_t *counts, int32_t *kept_counts, int32_t *offsets, int32_t *perm_slot,
                    int32_t *slot_pos) {
  int64_t S = T * k;
  int64_t row = 0;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) {
    counts[e] = 0;
    kept_counts[e] = 0;
    for (int64_t s = 0; s < S; ++s) {
      if (idx[s] != e) continue;
      counts[e] += 1;
      if (kept[s]) {
        kept_counts[e] += 1;
        perm_slot[row] = (int32_t)s;
        slot_pos[s] = (int32_t)row;
        ++row;
      } else {
        slot_pos[s] = -1;
      }
    }
    offsets[e + 1] = (int32_t)row;
  }
}

/* One expert on one token [P3] "MoE Layer" (MixtralExpert.forward) and
 * "SwiGLU Experts":  a = W1 x,  b = W3 x,  h = SiLU(a) * b,  o = W2 h,
 * SiLU(a) = a / (1 + exp(-a)).  W1e, W3e [f, d]; W2e [d, f].  h [f], o [d]. */
void oracle_expert_row(int32_t d, int32_t f, const uint16_t *xrow, const uint16_t *W1e,
                       const uint16_t *W3e, const uint16_t *W2e, double *h, double *o) {
  for (int32_t n = 0; n < f; ++n) {
    double a = 0.0, b = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      double xi = bf16_to_double(xrow[i]);
      a += bf16_to_double(W1e[(int64_t)n * d + i]) * xi;
      b += bf16_to_double(W3e[(int64_t)n * d + i]) * xi;
    }
    h[n] = a / (1.0 + exp(-a)) * b;
  }
  for (int32_t c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int32_t n = 0; n < f; ++n) acc += bf16_to_double(W2e[(int64_t)c * f + n]) * h[n];
    o[c] = acc;
  }
}

/* Layer output [P2] "How it works": y = sum_i G(x)_i * Expert_i(x), G zero off
 * the top-k; with capacity, a dropped slot adds nothing.  Computed for the
 * tokens listed in rows[0..n_rows): y[r, :] for token rows[r].
 * Optional outputs (may be NULL): h_out [n_rows, k, f] and o_out
 * [n_rows, k, d], the expert hidden state and output of each slot (zeros for
 * a dropped slot). */
void oracle_layer_rows(int64_t T, int32_t d, int32_t f, int32_t E, int32_t k, const uint16_t *x,
                       const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                       const int32_t *idx, const double *w, const uint8_t *kept, int64_t n_rows,
                       const int64_t *rows, double *y, double *h_out, double *o_out) {
  (void)T;
  (void)E;
#pragma omp parallel
  {
    double *h = (double *)malloc(sizeof(double) * (size_t)f);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t t = rows[r];
      double *yr = y + r * d;
      for (int32_t c = 0; c < d; ++c) yr[c] = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int64_t s = t * k + j;
        double *hs = h_out ? h_out + (r * k + j) * (int64_t)f : NULL;
        double *os = o_out ? o_out + (r * k + j) * (int64_t)d : NULL;
        if (!kept[s]) {
          if (hs) memset(hs, 0, sizeof(double) * (size_t)f);
          if (os) memset(os, 0, sizeof(double) * (size_t)d);
          continue;
        }
        int64_t e = idx[s];
        oracle_expert_row(d, f, x + t * d, W1 + e * f * d, W3 + e * f * d, W2 + e * d * f, h, o);
        for (int32_t c = 0; c < d; ++c) yr[c] += w[s] * o[c];
        if (hs) memcpy(hs, h, sizeof(double) * (size_t)f);
        if (os) memcpy(os, o, sizeof(double) * (size_t)d);
      }
    }
    free(h);
    free(o);
  }
}

/* Router statistics [P1] "Expert specialization" (get_expert_activations:
 * per layer, the bincount of the top-2 expert indices over all tokens) and
 * [P5] "Inspecting Expert Routing" (the most common expert in each top-k
 * position).  slot_counts[j * E + e] = number of tokens whose j-th choice is
 * e; pair_counts[a * E + b] = number of tokens whose first two choices are
 * (a, b) (k >= 2; may be NULL).  Summing slot_counts over j gives the
 * bincount of the flattened top-k indices. */
void oracle_router_stats(int64_t T, int32_t E, int32_t k, const int32_t *idx, int32_t *slot_counts,
                         int32_t *pair_counts) {
  for (int64_t i = 0; i < (int64_t)k * E; ++i) slot_counts[i] = 0;
  if (pair_counts)
    for (int64_t i = 0; i < (int64_t)E * E; ++i) pair_counts[i] = 0;
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t j = 0; j < k; ++j) slot_counts[j * E + idx[t * k + j]] += 1;
    if (pair_counts && k >= 2) pair_counts[idx[t * k] * E + idx[t * k + 1]] += 1;
  }
}

/* ------------------------------------------------------------------------
 * 4-bit expert weights.
 *  [P1] "Deployment tradeoffs you'll actually hit", "Quantization asymmetry":
 *       the router stays in 16-bit precision, the experts are quantised to 4
 *       bits.
 *  [P5] "4-bit Quantization for Single GPU" and "Memory Requirements": 4-bit
 *       weights with block-wise absmax scales, arithmetic in bf16.
 * Reading (the pages name formats, not their bits): symmetric 4-bit codes,
 * one scale per 64 consecutive inputs of a weight row.  For a block b of row
 * r of expert e:
 *   s     = bf16(absmax_b / 7)            (fp32 division, then round to bf16)
 *   q     = clamp(round_half_even(w / s), -8, 7)   (fp32 division; q = 0 if s = 0)
 *   code  = q + 8                         (0 .. 15)
 *   w_hat = (code - 8) * s
 * Storage of W [E, R, K] (K a multiple of 64):
 *   codes  [E, R, K/2] bytes.  The codes of inputs 8g .. 8g+7 of a row fill
 *          one little-endian 32-bit word: nibble m (bits 4m .. 4m+3) holds
 *          input 8g + 2m and nibble m + 4 holds input 8g + 2m + 1 (m = 0..3).
 *   scales [E, K/64, R] bf16 bits (block-major: the scales of one block of
 *          consecutive rows are adjacent).
 * ------------------------------------------------------------------------ */

static float q4_bf16_round(float v) {  /* fp32 -> nearest-even bf16, as fp32 */
  uint32_t u;
  memcpy(&u, &v, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  float r;
  memcpy(&r, &u, 4);
  return r;
}

/* byte offset and bit shift of input k's code inside its row */
static void q4_locate(int64_t k, int64_t *byte, int *shift) {
  int64_t g = k / 8;
  int j = (int)(k % 8);
  int nib = j / 2 + 4 * (j % 2);
  *byte = g * 4 + nib / 2;
  *shift = 4 * (nib % 2);
}

void oracle_q4_quantize(int32_t E, int32_t R, int32_t K, const uint16_t *W, uint8_t *codes,
                        uint16_t *scales) {
  int32_t nb = K / 64;
  memset(codes, 0, (size_t)E * R * (K / 2));
#pragma omp parallel for collapse(2) schedule(static)
  for (int32_t e = 0; e < E; ++e)
    for (int32_t r = 0; r < R; ++r)
      for (int32_t b = 0; b < nb; ++b) {
        const uint16_t *wr = W + ((int64_t)e * R + r) * K + (int64_t)b * 64;
        float amax = 0.0f;
        for (int i = 0; i < 64; ++i) {
          float v = fabsf((float)bf16_to_double(wr[i]));
          if (v > amax) amax = v;
        }
        float s = q4_bf16_round(amax / 7.0f);
        uint32_t sb;
        memcpy(&sb, &s, 4);
        scales[((int64_t)e * nb + b) * R + r] = (uint16_t)(sb >> 16);
        uint8_t *cr = codes + ((int64_t)e * R + r) * (K / 2);
        for (int i = 0; i < 64; ++i) {
          int q = 0;
          if (s != 0.0f) {
            float v = nearbyintf((float)bf16_to_double(wr[i]) / s);
            q = v < -8.0f ? -8 : v > 7.0f ? 7 : (int)v;
          }
          int64_t byte;
          int shift;
          q4_locate((int64_t)b * 64 + i, &byte, &shift);
          cr[byte] |= (uint8_t)((q + 8) << shift);
        }
      }
}

/* w_hat of input k of row r, expert slice (codes_e [R, K/2], scales_e [K/64, R]) */
static double q4_weight(const uint8_t *codes_e, const uint16_t *scales_e, int32_t R, int32_t K,
                        int64_t r, int64_t k) {
  int64_t byte;
  int shift;
  q4_locate(k, &byte, &shift);
  int code = (codes_e[r * (K / 2) + byte] >> shift) & 0xF;
  return (double)(code - 8) * bf16_to_double(scales_e[(k / 64) * R + r]);
}

void oracle_q4_dequant(int32_t E, int32_t R, int32_t K, const uint8_t *codes,
                       const uint16_t *scales, double *out) {
  for (int32_t e = 0; e < E; ++e) {
    const uint8_t *ce = codes + (int64_t)e * R * (K / 2);
    const uint16_t *se = scales + (int64_t)e * (K / 64) * R;
    for (int64_t r = 0; r < R; ++r)
      for (int64_t k = 0; k < K; ++k) out[((int64_t)e * R + r) * K + k] = q4_weight(ce, se, R, K, r, k);
  }
}

/* One expert on one token with 4-bit weights: the expert of [P3] "MoE Layer"
 * with every weight read as w_hat.  Expert slices: W1 / W3 codes [f, d/2],
 * scales [d/64, f]; W2 codes [d, f/2], scales [f/64, d]. */
void oracle_expert_row_q4(int32_t d, int32_t f, const uint16_t *xrow, const uint8_t *W1c,
                          const uint16_t *W1s, const uint8_t *W3c, const uint16_t *W3s,
                          const uint8_t *W2c, const uint16_t *W2s, double *h, double *o) {
  for (int32_t n = 0; n < f; ++n) {
    double a = 0.0, b = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      double xi = bf16_to_double(xrow[i]);
      a += q4_weight(W1c, W1s, f, d, n, i) * xi;
      b += q4_weight(W3c, W3s, f, d, n, i) * xi;
    }
    h[n] = a / (1.0 + exp(-a)) * b;
  }
  for (int32_t c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int32_t n = 0; n < f; ++n) acc += q4_weight(W2c, W2s, d, f, c, n) * h[n];
    o[c] = acc;
  }
}

/* oracle_layer_rows with 4-bit expert weights (same combine, [P2] "How it works"). */
void oracle_layer_rows_q4(int64_t T, int32_t d, int32_t f, int32_t E, int32_t k, const uint16_t *x,
                          const uint8_t *W1c, const uint16_t *W1s, const uint8_t *W3c,
                          const uint16_t *W3s, const uint8_t *W2c, const uint16_t *W2s,
                          const int32_t *idx, const double *w, const uint8_t *kept, int64_t n_rows,
                          const int64_t *rows, double *y, double *h_out, double *o_out) {
  (void)T;
  (void)E;
#pragma omp parallel
  {
    double *h = (double *)malloc(sizeof(double) * (size_t)f);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t t = rows[r];
      double *yr = y + r * d;
      for (int32_t c = 0; c < d; ++c) yr[c] = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int64_t slot = t * k + j;
        double *hs = h_out ? h_out + (r * k + j) * (int64_t)f : NULL;
        double *os = o_out ? o_out + (r * k + j) * (int64_t)d : NULL;
        if (!kept[slot]) {
          if (hs) memset(hs, 0, sizeof(double) * (size_t)f);
          if (os) memset(os, 0, sizeof(double) * (size_t)d);
          continue;
        }
        int64_t e = idx[slot];
        int64_t w13 = e * (int64_t)f * (d / 2), s13 = e * (int64_t)(d / 64) * f;
        int64_t w2 = e * (int64_t)d * (f / 2), s2 = e * (int64_t)(f / 64) * d;
        oracle_expert_row_q4(d, f, x + t * d, W1c + w13, W1s + s13, W3c + w13, W3s + s13, W2c + w2,
                             W2s + s2, h, o);
        for (int32_t c = 0; c < d; ++c) yr[c] += w[slot] * o[c];
        if (hs) memcpy(hs, h, sizeof(double) * (size_t)f);
        if (os) memcpy(os, o, sizeof(double) * (size_t)d);
      }
    }
    free(h);
    free(o);
  }
}

/* Number of OpenMP threads the oracle runs with (reported with its timing). */
int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      extern int omp_get_num_threads(void);
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}
