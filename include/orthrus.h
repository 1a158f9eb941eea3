/*
 * orthrus.h -- C ABI of the B200 (sm_100a) hot path of the Orthrus dual-view
 * decode step.
 *
 * Method sources (web pages about "Orthrus: Memory-Efficient Parallel Token
 * Generation via Dual-View Diffusion", arXiv 2605.12825):
 *   [GIST]  gist.science summary, "Technische samenvatting": 2.1 dual-view
 *           attention over one shared KV cache, 2.2 block mask M_diff
 *           (causal context + bidirectional block), 2.3 inference consensus
 *           (item 1 parallel projection of anchor + K-1 masks, item 2 AR check
 *           of all K positions in one pass, item 3 longest greedy-matching
 *           prefix, correction token, cache shortening).
 *   [HN]    Hacker News thread "Orthrus-Qwen3: up to 7.8x tokens/forward on
 *           Qwen3, identical output distribution", post #21 (K = 32, shared
 *           KV cache, AR head accepts the longest matching prefix).
 *   [ABS]   the paper's abstract: shared KV cache, exact consensus, O(1)
 *           memory overhead.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, row-major
 *     and densely packed.  bf16 means IEEE bfloat16 bits.  The caller owns
 *     every buffer, including workspaces; the library allocates no device
 *     memory.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  Every call is asynchronous on `stream` and never synchronises.
 *   - Return value: ORTHRUS_OK (0) or a negative orthrus_status.  Host-side
 *     validation happens before any launch; on an error nothing is launched
 *     and no output is touched.  ORTHRUS_ECUDA reports a launch failure.
 *   - Conditions only the device can see (a committed length that would pass
 *     the cache capacity, an accept length out of range) never trap: the
 *     kernel clamps and, if `dev_status` is non-NULL, stores the first error
 *     code there (atomically, only if it is still 0).  Callers zero it first.
 *   - Waits inside kernels are bounded; a wait that gives up stores
 *     ORTHRUS_ETIMEOUT in dev_status (when given) and the kernel returns.
 *   - The library is built for sm_100a only.
 */
#ifndef ORTHRUS_H_
#define ORTHRUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ORTHRUS_OK = 0,
  ORTHRUS_EINVAL = -1,       /* bad argument value (NULL pointer, K out of range, ...) */
  ORTHRUS_ESHAPE = -2,       /* inconsistent shapes (Hq % Hkv != 0, cap < K, ...)      */
  ORTHRUS_EUNSUPPORTED = -3, /* valid but not implemented (head_dim not 64/128, ...)  */
  ORTHRUS_ECUDA = -4,        /* a CUDA runtime/driver call failed                     */
  ORTHRUS_ECAPACITY = -5,    /* device: ctx_len + K would pass the cache capacity     */
  ORTHRUS_EWORKSPACE = -6,   /* workspace missing or smaller than the size query says */
  ORTHRUS_EALIGN = -7,       /* a pointer is not 16-byte aligned                      */
  ORTHRUS_ETIMEOUT = -8      /* device: a bounded wait inside a kernel gave up        */
} orthrus_status;

typedef enum {
  /* [GIST 2.2, 2.3 item 1] diffusion view: block row i sees keys [0, L+K):
   * the whole committed prefix plus every block position, bidirectionally. */
  ORTHRUS_MASK_DIFF = 0,
  /* [GIST 2.3 item 2; HN #21] AR view: block row i sees keys [0, L+i+1):
   * the prefix plus block positions 0..i.  K = 1 is ordinary decoding. */
  ORTHRUS_MASK_AR = 1
} orthrus_mask_mode;

/* Option bit OR-ed into mask_mode of orthrus_block_attn (no counterpart in
 * the method: an implementation choice).  By default the CTAs that share a
 * (sequence, KV head) segment claim its last ~quarter of key groups
 * dynamically, which balances their finish times but makes the fp32
 * summation order, hence the last bits of the output, vary between calls.
 * With this bit every CTA takes a fixed key range and repeated calls on the
 * same inputs are bitwise identical. */
#define ORTHRUS_ATTN_DETERMINISTIC 0x100

/*
 * One layer's view of the shared KV cache ([GIST 2.1, 3]; [ABS]).
 *   k, v      bf16 [B, Hkv, cap, d] device.  Slots [0, ctx_lens[b]) hold the
 *             committed prefix of sequence b; before block attention the
 *             caller writes the block's K/V (either view's projections) into
 *             slots [ctx_lens[b], ctx_lens[b] + K).  Slots beyond that are
 *             never read and may hold anything, including NaN.
 *   ctx_lens  int32 [B] device: committed length L_b per sequence.  One array
 *             serves all layers; orthrus_kv_commit advances it once per step.
 * Rows of k and v (d * 2 bytes) and the base pointers must be 16-byte aligned.
 */
typedef struct {
  void *k;
  void *v;
  int32_t *ctx_lens;
  int B;
  int Hkv;
  int cap;
  int d;
} orthrus_kv_cache;

/* Human-readable name of a status code (static storage, never NULL). */
const char *orthrus_status_str(int status);

/* ABI version of this header/library pair (incremented on any change). */
int orthrus_abi_version(void);

/*
 * Process-wide limit, in nanoseconds, after which a bounded wait inside any
 * kernel of this library gives up: the kernel then stores ORTHRUS_ETIMEOUT in
 * dev_status, lets its in-flight copies and MMAs finish, frees its tensor
 * memory and returns (its outputs are then undefined, and an attention
 * workspace must be zeroed again).  Read at every launch; 0 restores the
 * default of 2 s.  The kernels' real waits take microseconds, so only a
 * watchdog or a test of the timeout path needs another value.  Always
 * returns ORTHRUS_OK.  (No counterpart in the method: failure handling.)
 */
int orthrus_set_wait_limit_ns(uint64_t ns);

/*
 * Workspace bytes orthrus_block_attn needs on the CURRENT device for these
 * shapes (split-KV partial results; independent of the context lengths).
 * Returns ORTHRUS_OK and writes *bytes, or a validation error.
 */
int orthrus_block_attn_workspace_size(int B, int Hq, int Hkv, int d, int K, size_t *bytes);

/*
 * Block-query attention over the shared KV cache ([GIST 2.1-2.3 items 1-2]).
 *
 * For sequence b, block row i in [0, K), query head h in [0, Hq), KV head
 * g = h / (Hq / Hkv) (contiguous GQA groups):
 *     s_j = (q[b,i,h,:] . k[b,g,j,:]) / sqrt(d)  for j < e,
 *     e   = L_b + K        (ORTHRUS_MASK_DIFF)
 *     e   = L_b + i + 1    (ORTHRUS_MASK_AR)
 *     out[b,i,h,:] = sum_j softmax(s)_j * v[b,g,j,:]
 * with bf16 inputs, fp32 accumulation and softmax, bf16 output.
 *
 *   q          bf16 [B, K, Hq, d] device (post-RoPE queries)
 *   cache      KV cache view (host struct; its pointers are device pointers)
 *   Hq, K      query heads (multiple of cache->Hkv), block size 1..32
 *   mask_mode  orthrus_mask_mode, optionally | ORTHRUS_ATTN_DETERMINISTIC
 *   out        bf16 [B, K, Hq, d] device
 *   workspace  device, >= orthrus_block_attn_workspace_size(...) bytes, zero
 *              filled before the first call.  Its head (at a fixed place for
 *              every shape) holds a grid-barrier counter and, per (sequence,
 *              KV head, head chunk) segment, a completion counter and a
 *              work-claim counter.  Every completed call leaves them in the
 *              state the next call starts from (grid counter a multiple of the
 *              grid size, completion counters multiples of 2^20, claim
 *              counters 0; the comparisons survive 64-bit wrap-around), so a
 *              workspace is zeroed once, not per call, and serves any sequence
 *              of shapes whose size query it satisfies.  Zero it again after an
 *              ORTHRUS_ETIMEOUT and before using it on a device with a
 *              different SM count.  The rest holds per-call partial results.
 *              Calls that share a workspace must be stream-ordered.
 *   dev_status int32 device or NULL (see conventions; ORTHRUS_ECAPACITY when
 *              L_b + K > cap, in which case L_b is clamped to cap - K)
 * Supported: d in {64, 128}; 1 <= K <= 32; Hq / Hkv <= 128.
 * Runs as one persistent split-KV kernel (one CTA per SM, tcgen05 MMAs with
 * TMEM accumulators, TMA-staged K/V tiles) whose CTAs merge their partial
 * results by log-sum-exp: per segment, behind that segment's counter, when
 * every segment gets its own CTAs; after a grid barrier otherwise.  Every CTA
 * must be resident at once.  With programmatic dependent launch on (the
 * default) the launch is plain, so back-to-back calls overlap; work that other
 * streams run at the same time can then hold SMs some CTAs wait for (past the
 * wait limit: ORTHRUS_ETIMEOUT).  Setting ORTHRUS_ATTN_COOPERATIVE (or
 * ORTHRUS_NO_PDL) before the first call makes every launch cooperative.
 */
int orthrus_block_attn(const void *q, const orthrus_kv_cache *cache, int Hq, int K,
                       int mask_mode, void *out, void *workspace, size_t ws_bytes,
                       int32_t *dev_status, void *stream);

/*
 * Causal attention over a prompt chunk: the AR view's pre-filling pass
 * ([GIST 2.1] item 1: the frozen AR head's only job is to pre-fill the context
 * into the shared cache both views read; [ABS]: the autoregressive head
 * executes context pre-filling).
 *
 * For sequence b with L_b = ctx_lens[b], chunk row i in [0, P) at position
 * L_b + i, query head h, KV head g = h / (Hq / Hkv):
 *     out[b,i,h,:] = sum_j softmax(s)_j * v[b,g,j,:],
 *     s_j = (q[b,i,h,:] . k[b,g,j,:]) / sqrt(d),   j < L_b + i + 1
 * -- orthrus_block_attn's AR mask with the chunk in place of the block (L_b = 0
 * for a whole prompt, L_b > 0 for a later chunk of a long one), bf16 inputs,
 * fp32 accumulation and softmax, bf16 output.
 *   q          bf16 [B, P, Hq, d] device (post-RoPE queries of the chunk)
 *   cache      KV cache view; the caller has written the chunk's K/V into slots
 *              [L_b, L_b + P) (orthrus_block_qkv_append with K = P does so with
 *              the Qwen3 epilogue).  ctx_lens is read, not changed: advance it
 *              by P afterwards.
 *   Hq, P      query heads (multiple of cache->Hkv), chunk length (>= 1)
 *   out        bf16 [B, P, Hq, d] device
 *   dev_status int32 device or NULL: ORTHRUS_ECAPACITY when L_b + P > cap
 *              (L_b is then clamped to cap - P)
 * Supported: d in {64, 128}.  No workspace.  One CTA per pair of query heads of
 * a KV group and 128 positions (tcgen05 MMAs, TMEM accumulators, TMA-staged
 * Q/K/V), latest positions first.
 */
int orthrus_prefill_attn(const void *q, const orthrus_kv_cache *cache, int Hq, int P, void *out,
                         int32_t *dev_status, void *stream);

/*
 * Workspace bytes orthrus_lmhead_argmax needs on the CURRENT device.
 */
int orthrus_lmhead_workspace_size(int R, int V, size_t *bytes);

/*
 * LM head with fused greedy choice ([GIST 2.3 items 2-3]: the frozen AR head
 * gives the target at all K positions; a draft is kept only if it equals the
 * greedy prediction).
 *     logits[r, v] = sum_k h[r,k] * W[v,k]   (fp32 accumulation of bf16 products)
 *     argmax[r]    = smallest v attaining max_v logits[r, v]
 * The logits never reach HBM: the argmax is reduced in the GEMM epilogue.
 *
 *   h          bf16 [R, H] device (final hidden states of the R = B*K rows)
 *   W          bf16 [V, H] device (nn.Linear weight layout)
 *   argmax     int32 [R] device (output)
 *   max_logit  fp32 [R] device or NULL (output: the maximum logit per row)
 *   workspace  device, >= orthrus_lmhead_workspace_size(R, V) bytes
 *   dev_status int32 device or NULL (ORTHRUS_ETIMEOUT if a bounded wait gave up)
 * Supported: 1 <= R; H % 64 == 0; 1 <= V < 2^31.  Rows are processed in
 * passes of at most 256.
 */
int orthrus_lmhead_argmax(const void *h, const void *W, int R, int H, int V, int32_t *argmax,
                          float *max_logit, void *workspace, size_t ws_bytes,
                          int32_t *dev_status, void *stream);

/*
 * orthrus_lmhead_argmax for callers that cannot allocate device memory.
 * (The paper has no counterpart: this is a deployment convenience.)
 *
 * Callers such as a plain C host program with no device allocator, a serving
 * loop whose memory plan is frozen after start-up (cudaMalloc synchronises the
 * device and may fail under fragmentation), or a runtime that owns all device
 * memory cannot pass a workspace.  This variant keeps its scratch -- the
 * per-CTA argmax candidates -- in a fixed 512 KB array inside the library's
 * own device memory (held on every GPU that loads the library until the
 * process exits) and otherwise behaves exactly like orthrus_lmhead_argmax.
 *   - It allocates nothing and calls no allocating routine.
 *   - The first call on each device looks up the array's device address once;
 *     make that first call before any stream capture.
 *   - All calls share the array (it keeps the last call's contents; nothing
 *     in it has to start zeroed).  Calls that overlap on the GPU race: order
 *     them on one stream.
 *   - Works on devices with up to 256 SMs (the array's capacity); returns
 *     ORTHRUS_EWORKSPACE, launching nothing, on a device with more.
 * Arguments as for orthrus_lmhead_argmax, without the workspace.
 */
int orthrus_lmhead_argmax_noalloc(const void *h, const void *W, int R, int H, int V,
                                  int32_t *argmax, float *max_logit, int32_t *dev_status,
                                  void *stream);

/*
 * Greedy choice over precomputed fp32 logits (a test helper for verifying
 * from given logits).  logits fp32 [R, V] device -> argmax int32 [R] device
 * (smallest index of the maximum; NaN entries are never chosen).
 */
int orthrus_row_argmax_f32(const float *logits, int R, int V, int32_t *argmax, void *stream);

/*
 * Exact consensus ([GIST 2.3 item 3]; [HN #21]).
 * argmax[b,i] is the AR greedy token predicted by block row i (the token after
 * block position i); draft[b,i] is the drafted token for the same position.
 *     accept_len[b] = min { i : draft[b,i] != argmax[b,i] }, or K if none
 *     next_tok[b]   = argmax[b, accept_len[b]]  if accept_len[b] < K
 *                     draft[b, K-1]             otherwise
 * next_tok is the new anchor (last emitted token, not yet in the cache).
 *   argmax, draft  int32 [B, K] device;  accept_len, next_tok int32 [B] device.
 * Supported: 1 <= K <= 32.  One warp per sequence, bit-exact.
 */
int orthrus_verify(const int32_t *argmax, const int32_t *draft, int B, int K,
                   int32_t *accept_len, int32_t *next_tok, void *stream);

/*
 * KV commit by moving the length pointer ([GIST 2.3 item 3]: commit the
 * synchronised prefix, shorten the cache; [ABS]: O(1) overhead).
 * The verify pass cached the anchor and draft[0..K-2] in slots [L, L+K); the
 * anchor plus the accepted drafts stay, so
 *     ctx_lens[b] += min(accept_len[b] + 1, K)
 * No KV element is moved or cleared: rejected slots are overwritten by the
 * next block.  A length that would pass cache->cap is clamped to cap
 * (ORTHRUS_ECAPACITY in dev_status); an accept length outside [0, K] leaves
 * the length unchanged (ORTHRUS_EINVAL in dev_status).
 *   cache       host struct; uses cache->ctx_lens, cache->B, cache->cap
 *   accept_len  int32 [B] device
 */
int orthrus_kv_commit(const orthrus_kv_cache *cache, const int32_t *accept_len, int K,
                      int32_t *dev_status, void *stream);

/*
 * orthrus_verify followed by orthrus_kv_commit in one launch (one warp per
 * sequence).  Same arguments and results as the two calls in sequence.
 */
int orthrus_verify_commit(const int32_t *argmax, const int32_t *draft, int B, int K,
                          int32_t *accept_len, int32_t *next_tok,
                          const orthrus_kv_cache *cache, int32_t *dev_status, void *stream);

/*
 * Block Q/K/V append: the step just before orthrus_block_attn, writing the
 * block's keys and values into the scratch slots [L_b, L_b + K) of the shared
 * cache ([GIST 2.1, 2.3 item 1]: both views use one cache; [ABS]: O(1)
 * overhead).  The pages leave the projections' epilogue open; this applies the
 * Qwen3 family's: for token i of sequence b at position p = L_b + i and every
 * head's d values x,
 *   q and k heads: x_c <- x_c / sqrt(mean_c x_c^2 + rms_eps) * w_c  (skipped
 *                  when both weights are NULL), then the rotary embedding
 *                  y_j = x_j cos a_j - x_{j+d/2} sin a_j,
 *                  y_{j+d/2} = x_{j+d/2} cos a_j + x_j sin a_j,
 *                  a_j = p * rope_theta^(-2j/d) (angles in double precision);
 *   v heads:       copied.
 *   qkv         bf16 [B*K, (Hq + 2 Hkv) d] device, row = token b*K + i, heads
 *               packed q (Hq) | k (Hkv) | v (Hkv)
 *   q_norm_w, k_norm_w  bf16 [d] device, both or neither
 *   rope_theta  > 0; rms_eps >= 0
 *   Hq, K       query heads (multiple of cache->Hkv), block tokens (>= 1)
 *   cache       KV cache view: k/v[b, g, L_b + i, :] receive the rotated k
 *               and the v of KV head g; other slots are untouched
 *   q_out       bf16 [B, K, Hq, d] device: the rotated queries, the layout
 *               orthrus_block_attn reads
 *   dev_status  int32 device or NULL: ORTHRUS_ECAPACITY when L_b + K > cap (L_b
 *               is then clamped to cap - K, exactly as orthrus_block_attn does)
 * Supported: d in {64, 128}.  Pointers 16-byte aligned.  No workspace.
 */
int orthrus_block_qkv_append(const void *qkv, const void *q_norm_w, const void *k_norm_w,
                             float rope_theta, float rms_eps, int Hq, int K,
                             const orthrus_kv_cache *cache, void *q_out, int32_t *dev_status,
                             void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ORTHRUS_H_ */
