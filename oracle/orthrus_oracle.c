/*
 * Plain fp64 CPU oracle for the Orthrus dual-view decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or table with the CUDA
 * library; the two meet only in the seeded input generators.
 *
 * Sources (web pages about "Orthrus: Memory-Efficient Parallel Token
 * Generation via Dual-View Diffusion", arXiv 2605.12825):
 *   [GIST]  gist.science summary of the paper, "Technische samenvatting",
 *           sections 2.1 (dual-view attention), 2.2 (block mask M_diff),
 *           2.3 (inference consensus, items 1-3), 3 (contributions).
 *   [HN]    Hacker News thread "Orthrus-Qwen3: up to 7.8x tokens/forward on
 *           Qwen3, identical output distribution", co-author summary quoted in
 *           post #21.
 *   [ABS]   the paper's abstract (codewithpapers page): shared KV cache,
 *           exact consensus, O(1) cache overhead.
 *
 * Every function is written the slow, obvious way: one output element at a
 * time, sums in index order, double precision throughout.  OpenMP only runs
 * independent output rows on separate threads; it never splits or reorders a
 * sum.  Inputs arrive as fp64, fp32 or raw bf16 bits (converted exactly to
 * fp64 on read), chosen by a dtype code, so the oracle reads the very bits
 * the GPU reads without a 5 GB fp64 copy of the LM-head matrix.
 *
 * Parity pins for each function live in the CPU test suite: SDPA in torch
 * float64, the K=1 and row-by-row reductions, closed forms, brute force and
 * the toy-model losslessness loop.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)
#define ORC_ECAPACITY (-5)

#define ORC_F64 0
#define ORC_BF16 1
#define ORC_F32 2

#define ORC_MASK_DIFF 0
#define ORC_MASK_AR 1

/* Read element i of a buffer of the given dtype as an exact double. */
static double rd(const void *p, size_t i, int dtype) {
  if (dtype == ORC_F64) return ((const double *)p)[i];
  if (dtype == ORC_F32) return (double)((const float *)p)[i];
  /* bf16: the upper 16 bits of an IEEE binary32; widening is exact. */
  uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int oracle_version(void) { return 1; }

/* Number of OpenMP threads a parallel region of this library will use. */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Block-query attention over the shared KV cache.
 *
 * [GIST 2.1, 2.2, 2.3 items 1-2; HN #21; ABS]: both views read one KV cache.
 * The diffusion view (mask_mode DIFF) lets every block position see the whole
 * committed prefix and every position of the block in both directions
 * ("causal context" + "bidirectional block" rules of M_diff).  The AR view
 * (mask_mode AR) verifies all K positions in one pass; position i sees the
 * prefix and block positions 0..i (ordinary causal attention).
 *
 * Layouts (row-major):
 *   q        [B, K, Hq, d]
 *   kc, vc   [B, Hkv, cap, d]   slots [0, L_b) committed, [L_b, L_b+K) block
 *   ctx_lens [B]                L_b, the committed length of sequence b
 *   out      [B, K, Hq, d]      fp64
 *   lse      [B, K, Hq] or NULL natural-log log-sum-exp of the scaled scores
 *
 * For query head h the KV head is g = h / (Hq / Hkv) (contiguous GQA groups).
 * Scores are (q . k_j) * scale with scale = 1/sqrt(d) unless scale > 0 is
 * given.  Key range: j < L_b + K (DIFF) or j < L_b + i + 1 (AR).
 * Returns ORC_ECAPACITY if L_b + K > cap for some b (nothing is written).
 */
int oracle_block_attn(const void *q, int q_dtype, const void *kc, const void *vc,
                      int kv_dtype, const int32_t *ctx_lens, int B, int K, int Hq,
                      int Hkv, int cap, int d, int mask_mode, double scale,
                      double *out, double *lse) {
  if (B < 0 || K < 1 || Hq < 1 || Hkv < 1 || d < 1 || cap < 0) return ORC_EINVAL;
  if (Hq % Hkv != 0) return ORC_EINVAL;
  if (mask_mode != ORC_MASK_DIFF && mask_mode != ORC_MASK_AR) return ORC_EINVAL;
  for (int b = 0; b < B; ++b)
    if (ctx_lens[b] < 0 || (long)ctx_lens[b] + K > cap) return ORC_ECAPACITY;
  const int G = Hq / Hkv;
  const double sc = scale > 0 ? scale : 1.0 / sqrt((double)d);
  const long nrows = (long)B * K * Hq;
  int err = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (long row = 0; row < nrows; ++row) {
    const int h = (int)(row % Hq);
    const int i = (int)((row / Hq) % K);
    const int b = (int)(row / ((long)Hq * K));
    const int g = h / G;
    const long L = ctx_lens[b];
    const long e = (mask_mode == ORC_MASK_DIFF) ? L + K : L + i + 1;
    double *s = (double *)malloc(sizeof(double) * (size_t)e);
    if (!s) {
#pragma omp atomic write
      err = ORC_ENOMEM;
      continue;
    }
    const size_t qoff = (size_t)row * d; /* [b][i][h] flattened == row */
    const size_t kvbase = ((size_t)b * Hkv + g) * (size_t)cap * d;
    /* scores s_j = (q . k_j) * scale */
    double m = -INFINITY;
    for (long j = 0; j < e; ++j) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c)
        acc += rd(q, qoff + c, q_dtype) * rd(kc, kvbase + (size_t)j * d + c, kv_dtype);
      s[j] = acc * sc;
      if (s[j] > m) m = s[j];
    }
    /* p_j = exp(s_j - m) / sum_j exp(s_j - m);  o = sum_j p_j v_j */
    double denom = 0.0;
    for (long j = 0; j < e; ++j) {
      s[j] = exp(s[j] - m);
      denom += s[j];
    }
    double *o = out + (size_t)row * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (long j = 0; j < e; ++j) {
      const double p = s[j] / denom;
      for (int c = 0; c < d; ++c) o[c] += p * rd(vc, kvbase + (size_t)j * d + c, kv_dtype);
    }
    if (lse) lse[row] = m + log(denom);
    free(s);
  }
  return err;
}

/*
 * Greedy choice of each row: the smallest column index attaining the row's
 * maximum ([GIST 2.3 item 3]: a drafted token is kept only if it equals the
 * greedy prediction of the frozen AR head).  top1 receives the maximum and gap
 * the difference to the best value at any other index (0 on an exact tie).
 * Either of top1/gap may be NULL.  NaN entries are never chosen.
 */
static void greedy_row(const double *x, int V, int32_t *arg, double *top1, double *gap) {
  int best = -1;
  double bv = -INFINITY;
  for (int v = 0; v < V; ++v)
    if (!isnan(x[v]) && (best < 0 || x[v] > bv)) {
      best = v;
      bv = x[v];
    }
  double second = -INFINITY;
  for (int v = 0; v < V; ++v)
    if (v != best && !isnan(x[v]) && x[v] > second) second = x[v];
  *arg = best;
  if (top1) *top1 = bv;
  if (gap) *gap = bv - second;
}

/*
 * LM head with fused greedy choice ([GIST 2.3 items 2-3]: the AR head yields
 * the target distribution for all K positions; acceptance compares with its
 * greedy prediction).
 *   h [R, H], W [V, H] (nn.Linear layout) -> logits[r, v] = sum_k h[r,k] W[v,k]
 *   argmax [R] int32; top1 [R], gap [R] fp64 (NULL allowed).
 * Row r is computed on one thread; the logits never leave this function.
 */
int oracle_lmhead_argmax(const void *h, int h_dtype, const void *W, int w_dtype, int R,
                         int H, int V, int32_t *argmax, double *top1, double *gap) {
  if (R < 0 || H < 1 || V < 1) return ORC_EINVAL;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < R; ++r) {
    double *logit = (double *)malloc(sizeof(double) * (size_t)V);
    double *hr = (double *)malloc(sizeof(double) * (size_t)H);
    if (!logit || !hr) {
      free(logit);
      free(hr);
#pragma omp atomic write
      err = ORC_ENOMEM;
      continue;
    }
    for (int k = 0; k < H; ++k) hr[k] = rd(h, (size_t)r * H + k, h_dtype);
    for (int v = 0; v < V; ++v) {
      double acc = 0.0;
      for (int k = 0; k < H; ++k) acc += hr[k] * rd(W, (size_t)v * H + k, w_dtype);
      logit[v] = acc;
    }
    greedy_row(logit, V, &argmax[r], top1 ? &top1[r] : NULL, gap ? &gap[r] : NULL);
    free(logit);
    free(hr);
  }
  return err;
}

/* Greedy choice over given logits [R, V] (fp64 or fp32). */
int oracle_row_argmax(const void *logits, int dtype, int R, int V, int32_t *argmax,
                      double *top1, double *gap) {
  if (R < 0 || V < 1) return ORC_EINVAL;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < R; ++r) {
    double *x = (double *)malloc(sizeof(double) * (size_t)V);
    if (!x) {
#pragma omp atomic write
      err = ORC_ENOMEM;
      continue;
    }
    for (int v = 0; v < V; ++v) x[v] = rd(logits, (size_t)r * V + v, dtype);
    greedy_row(x, V, &argmax[r], top1 ? &top1[r] : NULL, gap ? &gap[r] : NULL);
    free(x);
  }
  return err;
}

/*
 * Exact consensus ([GIST 2.3 item 3]; [HN #21]: accept the longest matching
 * prefix).  Row i of the AR pass predicts the token after block position i, so
 * argmax[b,i] is compared with draft[b,i].  Scanning i = 0, 1, ... the first
 * index where they differ is the accepted length a_b (K if none differs).
 * The correction token is the AR choice at that index; when the whole block
 * matches, the last drafted token becomes the next anchor.
 *   argmax, draft [B, K] -> accept_len [B], next_tok [B]
 */
int oracle_verify(const int32_t *argmax, const int32_t *draft, int B, int K,
                  int32_t *accept_len, int32_t *next_tok) {
  if (B < 0 || K < 1) return ORC_EINVAL;
  for (int b = 0; b < B; ++b) {
    const int32_t *am = argmax + (size_t)b * K;
    const int32_t *dr = draft + (size_t)b * K;
    int a = 0;
    while (a < K && dr[a] == am[a]) ++a;
    accept_len[b] = a;
    next_tok[b] = (a < K) ? am[a] : dr[K - 1];
  }
  return ORC_OK;
}

/*
 * KV commit by moving the length pointer ([GIST 2.3 item 3]: commit the
 * synchronised prefix and shorten the cache; [ABS]: O(1) cache overhead).
 * The verify pass cached the anchor and drafts 0..K-2 in slots
 * [L, L+K); the anchor plus the a accepted drafts stay, so L advances by
 * min(a+1, K).  No KV element moves.  If the advance would pass cap the
 * length is clamped to cap and *status (if given) is set to ORC_ECAPACITY;
 * an accept length outside [0, K] sets ORC_EINVAL and leaves L unchanged.
 */
int oracle_kv_commit(int32_t *ctx_lens, const int32_t *accept_len, int B, int K, int cap,
                     int32_t *status) {
  if (B < 0 || K < 1 || cap < 0) return ORC_EINVAL;
  int st = ORC_OK;
  for (int b = 0; b < B; ++b) {
    const int a = accept_len[b];
    if (a < 0 || a > K) {
      st = ORC_EINVAL;
      continue;
    }
    const long adv = (a + 1 < K) ? a + 1 : K;
    long nl = (long)ctx_lens[b] + adv;
    if (nl > cap) {
      nl = cap;
      st = ORC_ECAPACITY;
    }
    ctx_lens[b] = (int32_t)nl;
  }
  if (status) *status = st;
  return ORC_OK;
}

/*
 * Block Q/K/V append: the step just before block attention, which writes the
 * block's keys and values into the scratch slots [L_b, L_b + K) of the shared
 * cache ([GIST 2.1, 2.3 item 1]: the block's K/V live in the one cache;
 * [ABS]: O(1) overhead).  The pages do not describe the projections' epilogue;
 * this follows the plain definitions of the Qwen3 family the build targets
 * (per-head RMS normalisation of q and k, then rotary position embedding):
 *
 * Token i of sequence b sits at position p = L_b + i.  qkv is packed per token
 * as [Hq heads of q | Hkv heads of k | Hkv heads of v], each head d values.
 *   norm (q and k heads, only if the weight pointer is non-NULL):
 *     x_c <- x_c / sqrt((1/d) sum_c x_c^2 + eps) * w_c
 *   rotary embedding, coordinate j paired with j + d/2 (j < d/2):
 *     a_j = p * theta^(-2j/d)                   (exactly, in fp64)
 *     y_j       = x_j cos a_j - x_{j+d/2} sin a_j
 *     y_{j+d/2} = x_{j+d/2} cos a_j + x_j sin a_j
 *   q_out[b, i, h, :] = rotary(norm_q(q));   k_cache[b, g, p, :] = rotary(norm_k(k));
 *   v_cache[b, g, p, :] = v.
 * The caches are fp64 [B, Hkv, cap, d] and only slots [L_b, L_b + K) are
 * written.  Returns ORC_ECAPACITY (writing nothing) if some L_b + K > cap.
 */
int oracle_qkv_append(const void *qkv, int qkv_dtype, const void *q_w, const void *k_w,
                      int w_dtype, double theta, double eps, const int32_t *ctx_lens, int B,
                      int K, int Hq, int Hkv, int d, int cap, double *q_out, double *k_cache,
                      double *v_cache) {
  if (B < 0 || K < 1 || Hq < 1 || Hkv < 1 || d < 2 || d % 2 || cap < 0 || theta <= 0 ||
      eps < 0)
    return ORC_EINVAL;
  if (Hq % Hkv != 0) return ORC_EINVAL;
  for (int b = 0; b < B; ++b)
    if (ctx_lens[b] < 0 || (long)ctx_lens[b] + K > cap) return ORC_ECAPACITY;
  const int G = Hq / Hkv;
  const int W = Hq + 2 * Hkv; /* heads per token in qkv */
  const long ntok = (long)B * K;
  int err = ORC_OK;

#pragma omp parallel for schedule(static)
  for (long t = 0; t < ntok; ++t) {
    const int b = (int)(t / K), i = (int)(t % K);
    const long pos = (long)ctx_lens[b] + i;
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    if (!x || !y) {
      free(x);
      free(y);
#pragma omp atomic write
      err = ORC_ENOMEM;
      continue;
    }
    for (int hh = 0; hh < W; ++hh) {
      const int is_q = hh < Hq, is_k = !is_q && hh < Hq + Hkv;
      for (int c = 0; c < d; ++c) x[c] = rd(qkv, ((size_t)t * W + hh) * d + c, qkv_dtype);
      if (is_q || is_k) {
        const void *w = is_q ? q_w : k_w;
        if (w) {
          double ss = 0.0;
          for (int c = 0; c < d; ++c) ss += x[c] * x[c];
          const double r = 1.0 / sqrt(ss / d + eps);
          for (int c = 0; c < d; ++c) x[c] = x[c] * r * rd(w, (size_t)c, w_dtype);
        }
        for (int j = 0; j < d / 2; ++j) {
          const double a = (double)pos * pow(theta, -2.0 * j / d);
          const double cs = cos(a), sn = sin(a);
          y[j] = x[j] * cs - x[j + d / 2] * sn;
          y[j + d / 2] = x[j + d / 2] * cs + x[j] * sn;
        }
      } else {
        for (int c = 0; c < d; ++c) y[c] = x[c];
      }
      if (is_q) {
        double *o = q_out + (((size_t)b * K + i) * Hq + hh) * d;
        for (int c = 0; c < d; ++c) o[c] = y[c];
      } else {
        const int g = is_k ? hh - Hq : hh - Hq - Hkv;
        double *dst = (is_k ? k_cache : v_cache) + (((size_t)b * Hkv + g) * cap + pos) * d;
        for (int c = 0; c < d; ++c) dst[c] = y[c];
      }
    }
    free(x);
    free(y);
  }
  (void)G;
  return err;
}
