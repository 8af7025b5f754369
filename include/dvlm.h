/*
 * dvlm.h -- C ABI of the B200 (sm_100a) block-diffusion decode step.
 *
 * The method (Fast-dVLM / Fast-dLLM v2 block diffusion):
 *   - the answer is produced in blocks of B tokens; inside a block every
 *     masked position is denoised in parallel, blocks follow one another
 *     autoregressively over an exact KV cache
 *     [Fast-dVLM technical overview (ocdem.com), sections 1.2 and 2.2.1];
 *   - attention follows three rules: noisy tokens of one block see each other
 *     (N2N, bidirectional), noisy tokens see the clean tokens of preceding
 *     blocks including the vision tokens (N2C), clean tokens are token-level
 *     causal (C2C) [same page, section 2.2.1; Fast-dVLM walkthrough
 *     (itsolotime.com), section 4.1];
 *   - each masked position is scored by its top-1 softmax probability over
 *     the vocabulary [Look Only When Needed (LOWN), method step (1)] and is
 *     committed when that confidence reaches the threshold (0.9), at least one
 *     per step [Fast-dVLM overview, section 4.1 recommended configuration];
 *   - the linear self-speculative variant drafts the block by diffusion,
 *     verifies it with a causal pass, keeps the longest agreeing prefix and
 *     truncates the KV cache [Fast-dVLM overview, section 2.3.1];
 *   - the certificate scan visits positions by descending anchor confidence
 *     and stops at the first disagreement [LOWN, method step (2)].
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host".
 *     The caller owns all memory; the library never allocates or frees device
 *     memory.  Workspaces are sized with the matching *_workspace_size() call
 *     and must be zero-filled once before their first use; every successful
 *     call leaves them ready for the next (counters return to zero).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Arguments are validated on the host before any
 *     launch; a bad argument returns an error status and launches nothing.
 *   - Errors found on the device (a bounded wait that ran out, an index out of
 *     range) are written to `*dev_status` (device int, first error wins, may
 *     be NULL); nothing traps or aborts.  Read it after synchronising.
 *   - Results are deterministic: the same inputs give bitwise-identical
 *     outputs (fixed reduction orders, no floating-point atomics).
 *   - Layouts are row-major; "[a, b, c]" lists dimensions outermost first.
 *     bf16 tensors hold IEEE bfloat16, fp32 tensors IEEE binary32.
 *   - The bf16 path runs on tcgen05 tensor cores with TMA-staged operands and
 *     needs every tensor base 16-byte aligned; the fp32 path (for the tiny
 *     fp32 model) runs on CUDA cores.
 */
#ifndef DVLM_H_
#define DVLM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DVLM_API __attribute__((visibility("default")))
#else
#define DVLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dvlm_status {
  DVLM_OK = 0,
  DVLM_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, bad enum value       */
  DVLM_ERR_SHAPE = 2,         /* sizes inconsistent or out of the supported range */
  DVLM_ERR_UNSUPPORTED = 3,   /* valid request the library does not implement     */
  DVLM_ERR_CACHE_OVERFLOW = 4,/* the step would write past Lmax                   */
  DVLM_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out               */
  DVLM_ERR_CUDA = 6,          /* a CUDA runtime/driver call failed                */
  DVLM_ERR_WORKSPACE = 7,     /* workspace missing or smaller than required       */
  DVLM_ERR_BOUNDS = 8         /* a device-side index check failed (e.g. token id) */
} dvlm_status;

/* DVLM_FP8_W8A8: the four projections of every layer are FP8 W8A8 (E4M3
 * weight codes with one scale per output row, activations quantised per
 * token on the fly); embedding, LM head, activations and the KV cache are
 * bf16 [Fast-dVLM technical overview (ocdem.com), section 2.3.2]. */
typedef enum dvlm_dtype { DVLM_BF16 = 0, DVLM_FP32 = 1, DVLM_FP8_W8A8 = 2 } dvlm_dtype;

typedef void* dvlm_stream; /* cudaStream_t */

/* Human-readable name of a status code (static string). */
DVLM_API const char* dvlm_status_string(int status);
/* Library version: major*10000 + minor*100 + patch. */
DVLM_API int dvlm_version(void);
/* Number of SMs the kernels size their grids for on the current device
 * (queried once per process); -1 when no device is visible. */
DVLM_API int dvlm_device_sm_count(void);

/* ------------------------------------------------------------------------
 * Block-masked GQA attention of one step's rows against the KV cache.
 *
 * q        [n_batch, n_rows, Hq, D]   queries, RoPE already applied.
 * out      [n_batch, n_rows, Hq, D]   attention output (same dtype).
 * k_cache  [n_batch, Hkv, Lmax, D]    keys; slots [L, L+n_rows) already hold
 *                                     this step's keys.
 * v_cache  [n_batch, Hkv, D, Lmax]    values, stored TRANSPOSED (value
 *                                     feature-major) so both tensor-core
 *                                     products read K-major operands.
 * Rows 0..n_clean-1 are clean and causal: row t sits at slot L+t and sees
 * slots 0..L+t (C2C).  Rows n_clean..n_rows-1 are the noisy block: each sees
 * every slot 0..L+n_rows-1, i.e. the whole cache (N2C: vision, prompt and
 * committed tokens) and the whole block (N2N).  Query head h uses KV head
 * h / (Hq/Hkv).  scale multiplies q.k (normally 1/sqrt(D)); softmax in fp32.
 * Slots at or beyond L+n_rows are never read into a result, whatever they
 * hold (NaN poison included).
 * bf16 path: D == 128, Hq == 8*Hkv, Lmax % 8 == 0.  fp32 path: D <= 128.
 * Errors: INVALID_ARG (null/misaligned), SHAPE (L+n_rows > Lmax, n_clean >
 * n_rows, Hq % Hkv), UNSUPPORTED (bf16 head shapes other than the above).
 * Defined by: Fast-dVLM technical overview (ocdem.com), section 2.2.1 (the
 * N2N / N2C / C2C attention rules of block diffusion over an exact KV
 * cache); Fast-dVLM walkthrough (itsolotime.com), section 4.1.
 */
DVLM_API dvlm_status dvlm_block_attn(const void* q, void* out, const void* k_cache, const void* v_cache,
                            int n_batch, int n_rows, int n_clean, int L, int Lmax, int Hq, int Hkv,
                            int D, float scale, dvlm_dtype dt, int* dev_status, dvlm_stream stream);

/* ------------------------------------------------------------------------
 * Fused LM head + top-1 confidence + threshold commit (+ certificate scan).
 *
 * For each row r < R: logits l = s_r * (hidden[r] . W^T) over the whole
 * vocabulary, streamed tile by tile and never written to memory; s_r is the
 * final RMSNorm factor 1/sqrt(mean(hidden[r]^2)+eps) when apply_rmsnorm != 0,
 * else 1.  Outputs (each pointer may be NULL):
 *   top1_id[r]   = lowest id attaining max l,
 *   top1_prob[r] = max softmax probability = 1 / sum_v exp(l_v - max l),
 *   commit[r]    = 1 if row r is committed this call, else 0,
 *   n_commit[0]  = number of committed rows.
 * Commit rule: among rows with masked[r] != 0 (all rows when masked is
 * NULL), every row with top1_prob >= threshold; if none passes, the masked
 * row with the highest top1_prob (lowest r on ties).  threshold <= -1
 * commits every masked row (the speculative draft).  When `tokens` is
 * non-NULL the commit is applied in place: tokens[r] = top1_id[r] and
 * masked[r] = 0 for committed rows (masked must then be non-NULL).
 * Certificate (when anchor_id, anchor_conf and cert_len are all non-NULL):
 * the rows that are masked on entry are visited in descending anchor_conf
 * (lower r first on ties); cert_len[0] = number visited before the first
 * row whose top1_id differs from anchor_id.
 * hidden [R, H], w [V, H] (same dtype).  1 <= R <= 128.
 * bf16 path: H % 64 == 0.  Workspace: dvlm_lmhead_workspace_size().
 * Defined by: Look Only When Needed, method step (1) (top-1 confidence = the
 * largest softmax probability) and step (2) (the certificate scan);
 * Fast-dVLM technical overview (ocdem.com), section 4.1 (threshold 0.9,
 * at least one position committed per step).
 */
DVLM_API size_t dvlm_lmhead_workspace_size(int R, int V, int H, dvlm_dtype dt);
DVLM_API dvlm_status dvlm_lmhead_conf_commit(const void* hidden, const void* w, int R, int H, int V,
                                    dvlm_dtype dt, int apply_rmsnorm, float eps, uint8_t* masked,
                                    int32_t* tokens, float threshold, int32_t* top1_id,
                                    float* top1_prob, uint8_t* commit, int32_t* n_commit,
                                    const int32_t* anchor_id, const float* anchor_conf,
                                    int32_t* cert_len, void* workspace, size_t ws_bytes,
                                    int* dev_status, dvlm_stream stream);

/* Same computation as dvlm_lmhead_conf_commit on the bf16 path, for callers
 * that cannot allocate device memory when they call it (a process whose
 * device memory is reserved up front by another framework's caching
 * allocator; a real-time control loop that forbids cudaMalloc after start-up
 * because an allocation can synchronise the device).  No counterpart on the
 * method's pages: this is a deployment variant.  It takes no workspace: its
 * scratch is one fixed 6 MiB device array inside the library.  The CUDA
 * runtime creates that array on a GPU when it loads the library's device
 * code there -- with lazy module loading, the CUDA default, during the first
 * call on that GPU -- and keeps it until the process exits.  Limits: R <= 32
 * and a scratch layout (about 17 KiB per SM plus 4 bytes per 128 vocabulary
 * rows) within 6 MiB, e.g. V <= 262144 and H <= 8192 on a 148-SM B200;
 * larger requests return DVLM_ERR_WORKSPACE and launch nothing.  The first
 * call on a device (and the first after a device reset) looks the array's
 * device address up: make one warm-up call at start-up, before any stream
 * capture.  Every call shares the one array and finds the previous call's
 * contents there (the counters it needs at zero are cleared on the stream
 * first): calls that overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller.  Allocates nothing; calls no
 * allocating routine. */
DVLM_API dvlm_status dvlm_lmhead_conf_commit_static(const void* hidden, const void* w, int R, int H, int V,
                                                   int apply_rmsnorm, float eps, uint8_t* masked,
                                                   int32_t* tokens, float threshold, int32_t* top1_id,
                                                   float* top1_prob, uint8_t* commit, int32_t* n_commit,
                                                   const int32_t* anchor_id, const float* anchor_conf,
                                                   int32_t* cert_len, int* dev_status, dvlm_stream stream);

/* dvlm_block_attn computed by `splits` independent CTAs per (batch entry,
 * 16-row group, KV head), bf16 only: the keys are dealt to the splits in
 * 128-key chunks (chunk j to split j % splits, by absolute slot, so a causal
 * row's result does not depend on n_rows), each split streams its chunks,
 * and the last split to finish merges all partials in split order.  The
 * bandwidth-bound form, for long caches and batches of caches.  workspace
 * (device, 16-byte aligned, zero-filled before the first call; it is zero
 * again after each call) of dvlm_block_attn_split_workspace_size bytes;
 * calls sharing a workspace must not overlap.  Arguments and errors
 * otherwise as dvlm_block_attn (DVLM_ERR_WORKSPACE for a small workspace;
 * splits 1..64). */
DVLM_API size_t dvlm_block_attn_split_workspace_size(int n_batch, int n_rows, int Hkv, int splits);
DVLM_API dvlm_status dvlm_block_attn_split(const void* q, void* out, const void* k_cache, const void* v_cache,
                                          int n_batch, int n_rows, int n_clean, int L, int Lmax, int Hq, int Hkv,
                                          int D, float scale, int splits, void* workspace, size_t ws_bytes,
                                          int* dev_status, dvlm_stream stream);

/* Block-masked attention over PAGED KV caches [Fast-dVLM technical overview
 * (ocdem.com), section 2.3.2: paged KV cache management], bf16: the rules of
 * dvlm_block_attn for each of n_batch sequences, whose caches live in 64-slot
 * pages.  Logical slot s of sequence b is row s % 64 of page
 * block_table[b * max_pages + s / 64] (device int32 [n_batch, max_pages]);
 * k_pages [n_pages, Hkv, 64, D], v_pages [n_pages, Hkv, D, 64] (transposed);
 * lens (device int32 [n_batch]) gives each sequence's cache length L_b, its
 * rows' K/V already at slots L_b..L_b+n_rows-1; q [n_batch, n_rows, Hq, D],
 * out likewise.  Ragged lengths are the point: every sequence is the
 * per-sequence definition and sees only its own pages.  D == 128, Hq == 8 *
 * Hkv, n_rows <= 64.  A page id outside 0..n_pages-1 or a length the table
 * cannot hold sets DVLM_ERR_BOUNDS in *dev_status (that chunk then reads page
 * 0 / the length is clamped; no out-of-range access).  Asynchronous. */
DVLM_API dvlm_status dvlm_block_attn_paged(const void* q, void* out, const void* k_pages, const void* v_pages,
                                          const int32_t* block_table, const int32_t* lens, int n_batch,
                                          int n_rows, int n_clean, int n_pages, int max_pages, int Hq, int Hkv,
                                          int D, float scale, int* dev_status, dvlm_stream stream);

/* ------------------------------------------------------------------------
 * Top-k commit [Look Only When Needed, background: the baseline dVLM
 * schedule unmasks the k most confident masked positions per step].
 *
 * Among rows r < R with masked[r] != 0, the k of highest top1_prob[r] (lower
 * row first on equal values) are committed: tokens[r] = top1_id[r] and
 * masked[r] = 0; every other row keeps its token and mask.  commit[r] = 1 for
 * the committed rows, 0 otherwise; *n_commit = min(k, number of masked rows).
 * top1_prob [R] (finite), top1_id [R]: device, as written by
 * dvlm_lmhead_conf_commit; masked [R] (uint8, in/out), tokens [R] (int32,
 * in/out): device; commit [R] and n_commit [1]: device, may be NULL.
 * 1 <= R <= 128, k >= 0.  Errors: DVLM_ERR_INVALID_ARG (a required pointer is
 * NULL), DVLM_ERR_SHAPE (R or k out of range).  One small kernel on `stream`,
 * asynchronous; dev_status is unused (no device-side failure mode).
 */
DVLM_API dvlm_status dvlm_topk_commit(const float* top1_prob, const int32_t* top1_id, uint8_t* masked,
                                      int32_t* tokens, int R, int k, uint8_t* commit, int32_t* n_commit,
                                      int* dev_status, dvlm_stream stream);

/* Divergence-first commit of certificate-guided routing's FULL branch [Look
 * Only When Needed, method step (3)]: as dvlm_topk_commit over the FULL
 * pass's rows (full_prob, full_id), except that masked rows whose TEXT-ONLY
 * top-1 text_id[r] differs from full_id[r] rank before every agreeing row;
 * inside each group descending full_prob, lower row first.  Committed rows
 * take full_id.  text_id [R]: device int32.  Same shapes, ownership and
 * errors as dvlm_topk_commit.  (The certified-prefix branch needs no entry
 * of its own: dvlm_topk_commit over the anchors' confidences and ids with k
 * = the certificate length unmasks exactly that prefix.) */
DVLM_API dvlm_status dvlm_divergence_first_commit(const float* full_prob, const int32_t* full_id,
                                                  const int32_t* text_id, uint8_t* masked, int32_t* tokens, int R,
                                                  int k, uint8_t* commit, int32_t* n_commit, int* dev_status,
                                                  dvlm_stream stream);

/* ------------------------------------------------------------------------
 * Speculative verify + longest-prefix accept + in-place KV truncation.
 *
 * For each sequence i < b: v_j = argmax_v verify_logits[i, j, :] (lowest id
 * on ties; NaN logits never win) when verify_logits [b, B, V] (bf16) is
 * non-NULL, else v_j = verify_ids[i, j] ([b, B] int32).  accept_len[i] = k =
 * the longest prefix length with v_j == draft_ids[i, j] for all j < k.
 * When cache_len is non-NULL it is updated in place from L0+B (the verify
 * pass wrote B slots) to L0+k, i.e. cache_len[i] -= B - k.  When
 * poison_tail != 0 the truncated slots [L0+k, L0+B) of every layer are
 * overwritten with bf16 NaN in k_cache [n_layers, b, Hkv, Lmax, D] and
 * v_cache [n_layers, b, Hkv, D, Lmax] (a debugging aid: attention never reads
 * them).  Workspace: dvlm_spec_workspace_size().
 * Defined by: Fast-dVLM technical overview (ocdem.com), section 2.3.1
 * (linear self-speculative decoding: a causal verify pass, the longest
 * agreeing prefix kept, the KV cache truncated to it).
 */
DVLM_API size_t dvlm_spec_workspace_size(int b, int B, int V);
DVLM_API dvlm_status dvlm_spec_verify_accept(const void* verify_logits, const int32_t* verify_ids,
                                    const int32_t* draft_ids, int b, int B, int V,
                                    int32_t* accept_len, int32_t* cache_len, int poison_tail,
                                    void* k_cache, void* v_cache, int n_layers, int Hkv, int D,
                                    int Lmax, void* workspace, size_t ws_bytes, int* dev_status,
                                    dvlm_stream stream);

/* ------------------------------------------------------------------------
 * Decoder model and decode engine.
 *
 * dvlm_model holds non-owning views of device weights, all [out, in]
 * row-major in the model dtype:
 *   embed   [V, H]                 token embeddings
 *   wqkv    [n_layers, (Hq+2*Hkv)*D, H]  rows: Hq query heads, Hkv key
 *                                  heads, Hkv value heads (D rows each)
 *   wo      [n_layers, H, Hq*D]
 *   wgate   [n_layers, I, H]       SwiGLU gate
 *   wup     [n_layers, I, H]       SwiGLU up
 *   wdown   [n_layers, H, I]
 *   lm_head [V, H]                 untied output projection
 * Each layer: x += Wo.attn(RoPE(Wqkv.rmsnorm(x))); x += Wdown.(silu(Wgate.n)
 * * Wup.n) with n = rmsnorm(x); RMSNorm gain 1; RoPE rotate-half with base
 * rope_base at absolute slot positions; final RMSNorm before the LM head.
 * bf16 storage points: q/k/v after RoPE, attention output, the residual
 * stream after each add, the SwiGLU activation; all sums in fp32.
 * bf16 path: H % 128 == 0, I % 64 == 0, D == 128, Hq == 8*Hkv.
 * FP8 W8A8 path: the bf16 path's shapes with I % 128 == 0; the projection
 * y = x W^T becomes y[t,o] = a_t * s_o * sum_k E4M3(h_tk / a_t) * code_ok
 * with a_t = max_k |h_tk| / 448 over the projection's input row h_t (the
 * RMS-normed row, the attention output or the SwiGLU activation) and s_o the
 * weight row scale; prefill runs in 16-row forwards.
 */
typedef struct dvlm_model {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, inter, vocab;
  int mask_id;       /* id of [MASK]; its embedding row feeds masked positions */
  float rope_base, eps;
  int dtype;         /* dvlm_dtype */
  const void* embed;
  const void* wqkv;
  const void* wo;
  const void* wgate;
  const void* wup;
  const void* wdown;
  const void* lm_head;
  /* DVLM_FP8_W8A8 only: wqkv..wdown hold E4M3 codes (uint8, same shapes) and
   * these their per-row fp32 scales ([n_layers, rows] each, e.g. from
   * dvlm_quantize_rows_e4m3); NULL otherwise. */
  const float* sqkv;
  const float* so;
  const float* sgate;
  const float* sup;
  const float* sdown;
} dvlm_model;

/* DVLM_MODE_SPEC_QUAD: quadratic self-speculative decoding [Fast-dVLM
 * technical overview (ocdem.com), section 2.3.1: draft and verify fused into
 * one forward at O(B^2) cost].  The first round of a run drafts with one
 * diffusion pass; every round then runs one forward over B + B*B rows: the
 * draft's B verify rows (causal, K/V to the cache) and, for each possible
 * accepted length k = 1..B, a candidate block of B [MASK] rows at positions
 * L+k..L+k+B-1 that sees the context, the verify rows 0..k-1 and itself (its
 * K/V stay out of the cache).  The longest agreeing prefix k is kept (L += k)
 * and the next draft is the verifier's token v_k followed by the top-1 of
 * candidate block k-1's rows 0..B-2.  Output = greedy AR output.  bf16
 * engines whose compute-bound prefill is supported, with B + B*B <= max_ctx. */
/* DVLM_MODE_ROUTE: certificate-guided visual routing inside block decoding
 * [Look Only When Needed, method steps (1)-(3)].  Per block (first token the
 * AR seed): a FULL noisy pass sets the anchors (top-1 id and probability of
 * every masked position) and unmasks the route_k most confident; each later
 * step runs a TEXT-ONLY pass (cache slots 0..route_n_vis-1 hidden, positions
 * unchanged) and scans the masked positions in descending anchor confidence
 * while its top-1 equals the anchor: a certified prefix of at least
 * min(route_k, masked) positions is unmasked whole with the anchor ids;
 * otherwise a FULL pass refreshes every anchor and min(route_k, masked)
 * positions are unmasked with the FULL ids, those whose TEXT-ONLY top-1
 * differs first (each group by confidence, lower position first on ties).
 * A causal pass appends the block.  bf16 engines; one host read of the
 * certified length per TEXT-ONLY pass. */
enum { DVLM_MODE_THRESHOLD = 0, DVLM_MODE_SPEC_LINEAR = 1, DVLM_MODE_AR = 2, DVLM_MODE_SPEC_QUAD = 3,
       DVLM_MODE_ROUTE = 4 };

typedef struct dvlm_decode_cfg {
  int block_size;     /* B, 1..16 */
  float threshold;    /* commit threshold (0.9) */
  int mode;           /* DVLM_MODE_* */
  int ar_seed;        /* 1: the block's first token is the AR prediction, committed outright */
  int max_new_tokens; /* generation stops after exactly this many tokens */
  int use_graphs;     /* 1: replay each forward as a captured CUDA graph */
  int route_k;        /* DVLM_MODE_ROUTE: positions unmasked per step (>= 1) */
  int route_n_vis;    /* DVLM_MODE_ROUTE: vision rows at the front of the cache (multiple of 8) */
} dvlm_decode_cfg;

#define DVLM_HIST 17
typedef struct dvlm_stats {
  int64_t nfe;                    /* decoder forwards (noisy iterations + causal passes) */
  int64_t n_tokens;               /* tokens emitted */
  int64_t n_iters;                /* threshold iterations (noisy passes) */
  int64_t n_rounds;               /* blocks (threshold/AR) or draft+verify rounds (spec) */
  int64_t commit_hist[DVLM_HIST]; /* iterations that committed c tokens, c = 0..16 */
  int64_t accept_hist[DVLM_HIST]; /* spec rounds that accepted k tokens, k = 0..16 */
  int64_t n_launches;             /* kernel launches issued (graph replays included) */
  int64_t n_text_passes;          /* DVLM_MODE_ROUTE: TEXT-ONLY noisy passes (counted in nfe too) */
} dvlm_stats;

typedef struct dvlm_engine dvlm_engine;

/* Workspace for an engine serving contexts up to Lmax slots, blocks up to
 * max_block (<= 16) rows and prompts (vision + ids) up to max_ctx rows. */
DVLM_API size_t dvlm_engine_workspace_size(const dvlm_model* m, int Lmax, int max_block, int max_ctx);
/* Builds the host-side engine (tensor maps, launch plans) over the caller's
 * buffers and zero-fills the workspace on `stream`.  k_cache [n_layers, Hkv,
 * Lmax, D] and v_cache [n_layers, Hkv, D, Lmax] (transposed) hold the exact
 * KV cache.  The engine keeps pointers, not copies. */
DVLM_API dvlm_status dvlm_engine_create(const dvlm_model* m, void* k_cache, void* v_cache, int Lmax,
                               int max_block, int max_ctx, void* workspace, size_t ws_bytes,
                               dvlm_stream stream, dvlm_engine** out);
DVLM_API dvlm_status dvlm_engine_destroy(dvlm_engine* e);
/* Causal pass over the context [vision rows | text ids] starting at slot 0
 * (vision [n_vision, H] in the model dtype, ids [n_ids] int32, both device),
 * in chunks of max_block rows; leaves L = n_vision + n_ids and the AR seed
 * (argmax of the LM head at the last context row) on the device. */
DVLM_API dvlm_status dvlm_prefill(dvlm_engine* e, const void* vision, int n_vision, const int32_t* ids,
                         int n_ids, dvlm_stream stream);
/* Decodes one block (threshold/AR modes: B tokens; spec mode: one draft +
 * verify round, 1..B tokens).  Tokens go to out_tokens (device, >= B
 * entries); *n_out (host) receives their count.  Synchronises the stream
 * once per noisy iteration (threshold mode) or round.  stats accumulate.
 * Returns DVLM_ERR_TIMEOUT when a block needs more than B - 1 noisy
 * iterations or a speculative round keeps no token: both mean a device-side
 * wait gave up (the status word, dvlm_engine_check, says where).
 * Defined by: Fast-dVLM technical overview (ocdem.com), sections 2.2.1-2.2.2
 * (block-wise decoding over the KV cache, the block's first token the AR
 * prediction), 2.3.1 (self-speculative variants) and 4.1 (block 16,
 * threshold 0.9); Look Only When Needed, method steps (1)-(3) (routing). */
DVLM_API dvlm_status dvlm_decode_block(dvlm_engine* e, const dvlm_decode_cfg* cfg, int32_t* out_tokens,
                              int32_t* n_out, dvlm_stats* stats, dvlm_stream stream);
/* Decodes exactly cfg->max_new_tokens tokens into out_tokens (device).
 * Errors as dvlm_decode_block. */
DVLM_API dvlm_status dvlm_generate(dvlm_engine* e, const dvlm_decode_cfg* cfg, int32_t* out_tokens,
                          dvlm_stats* stats, dvlm_stream stream);
/* End to end from HOST buffers: copies vision_host [n_vision, H] (model
 * dtype) and ids_host [n_ids] to the device, prefills, generates
 * cfg->max_new_tokens tokens and copies them to out_host.  Pinned host
 * buffers make the copies asynchronous.  Returns after the stream drained. */
DVLM_API dvlm_status dvlm_generate_host(dvlm_engine* e, const dvlm_decode_cfg* cfg, const void* vision_host,
                               int n_vision, const int32_t* ids_host, int n_ids,
                               int32_t* out_host, dvlm_stats* stats, dvlm_stream stream);
/* Cache length and pending seed token (host copies; synchronises). */
DVLM_API dvlm_status dvlm_engine_get_position(dvlm_engine* e, int32_t* L, int32_t* seed, dvlm_stream stream);
/* Rewinds to an earlier (L, seed); slots [0, L) must still hold that context. */
DVLM_API dvlm_status dvlm_engine_set_position(dvlm_engine* e, int32_t L, int32_t seed, dvlm_stream stream);
/* Synchronises, returns the first device-side error recorded since the last
 * call (DVLM_OK if none) and clears it. */
DVLM_API dvlm_status dvlm_engine_check(dvlm_engine* e, dvlm_stream stream);

/* One forward pass of n_rows rows at slots [L, L+n_rows) through layers
 * [first_layer, first_layer+n_layers_run) (test and profiling hook).  Input
 * rows: x_in [n_rows, H] (model dtype) when non-NULL, else the embeddings of
 * tokens [n_rows] (rows with masked[r] != 0 take the [MASK] embedding).
 * Rows 0..n_clean-1 are causal, the rest one noisy block.  Writes this
 * step's K/V to slots [L, L+n_rows) of the layers it runs, the resulting
 * residual stream to x_out [n_rows, H] (may be NULL) and, when
 * advance != 0, sets L += n_rows. */
DVLM_API dvlm_status dvlm_forward(dvlm_engine* e, const void* x_in, const int32_t* tokens,
                         const uint8_t* masked, int n_rows, int n_clean, int first_layer,
                         int n_layers_run, int advance, void* x_out, dvlm_stream stream);

/* Paged KV cache for an engine [Fast-dVLM technical overview (ocdem.com),
 * section 2.3.2: paged KV cache management]: from now on the engine's cache
 * is k_pages [n_layers, n_pages, Hkv, 64, D] and v_pages [n_layers, n_pages,
 * Hkv, D, 64] (bf16, device, caller-owned), logical slot s living in row
 * s % 64 of page block_table[s / 64] (device int32 [max_pages], read at each
 * launch: the caller may extend it between calls).  Attention reads each
 * 64-slot page through the table and the QKV projection writes each new K/V row
 * through it; results equal those of the contiguous cache bit for bit.
 * Prefill runs in 16-row forwards; DVLM_MODE_SPEC_QUAD, DVLM_MODE_ROUTE and
 * dvlm_forward_text_only are unsupported on a paged engine.  max_pages * 64
 * must cover the engine's Lmax (DVLM_ERR_SHAPE).  A page id outside
 * 0..n_pages-1 is reported as DVLM_ERR_BOUNDS in the status word. */
DVLM_API dvlm_status dvlm_engine_set_paged(dvlm_engine* e, void* k_pages, void* v_pages,
                                          const int32_t* block_table, int n_pages, int max_pages);

/* Test hook: the fused draft+verify forward of quadratic self-speculative
 * decoding alone, over draft [B] (device int32, copied into the engine's
 * block tokens) at slots L..L+B-1: writes the verify rows' K/V to the cache
 * (L is not advanced) and the final residual stream of all B + B*B rows
 * (verify rows, then candidate blocks 0..B-1) to x_out [B + B*B, H] (bf16,
 * device).  UNSUPPORTED where DVLM_MODE_SPEC_QUAD is; SHAPE for B outside
 * 1..16 or B + B*B > max_ctx; CACHE_OVERFLOW if L + B + B > Lmax. */
DVLM_API dvlm_status dvlm_forward_quad(dvlm_engine* e, const int32_t* draft, int B, void* x_out,
                                      dvlm_stream stream);

/* Launch-configuration knobs of a bf16 engine (defaults are chosen at
 * creation from occupancy queries).  Names and values:
 *   "qkv_cluster", "o_cluster", "down_cluster": CTAs per cluster of the
 *       cluster split-K projections (2..16; 0 = stream-K kernel instead);
 *   "down_stages", "gateup_stages": TMA pipeline depth, 5 or 10 (not both 5:
 *       UNSUPPORTED);
 *   "gateup_ctas_per_sm": 1, or 2 with 5 gate/up stages;
 *   "attn_cluster": CTAs per attention cluster, 8 or 16;
 *   "pdl": 1/0, programmatic dependent launch between kernels;
 *   "attn_split": 0 = cluster attention, 1..32 = split attention with that
 *       many CTAs per KV head (dvlm_block_attn_split);
 *   "prefill_gemm": 1/0, the compute-bound prefill (where supported);
 *   "persistent": 1/0, every decoder layer of a forward in one launch on
 *       all SMs: the first layer's QKV, then per layer attention (64-key
 *       chunk units), its merge, O-projection, gate/up, down and the next
 *       layer's QKV as phases separated by grid barriers, the weight stream
 *       running ahead across them (bf16 weights, 128-wide heads, 8 query
 *       heads per KV head, contiguous cache; TEXT-ONLY passes and paged
 *       caches use the per-kernel path; UNSUPPORTED where one CTA per SM
 *       cannot be resident on all SMs).
 * Results do not depend on the knobs except through fp32 summation order
 * (cluster sizes, stream-K splits) and, with "persistent", attention's P
 * held in bf16 (fp16 in the per-kernel attention).  Changing a knob drops the captured CUDA graphs.
 * Errors: INVALID_ARG (unknown name), SHAPE (bad value), UNSUPPORTED (the
 * device cannot launch that configuration, or an fp32 engine). */
DVLM_API dvlm_status dvlm_engine_set_option(dvlm_engine* e, const char* name, int value);
/* Current value of a knob (-1 for an unknown name). */
DVLM_API int dvlm_engine_get_option(dvlm_engine* e, const char* name);

/* Failure-detection self-test.  Every device-side wait of the library is
 * bounded: on expiry it writes DVLM_ERR_TIMEOUT to the status word, abandons
 * the rest of its work and lets the kernel end (no trap, no hang).  This
 * launches one CTA whose wait can never be satisfied (an mbarrier expecting
 * two arrivals receives one) with a budget of budget_cycles SM cycles
 * (1..4e9); afterwards *dev_status (device) holds DVLM_ERR_TIMEOUT and
 * *gave_up (device int) holds 1. */
DVLM_API dvlm_status dvlm_selftest_wait_timeout(long long budget_cycles, int* dev_status, int* gave_up,
                                               dvlm_stream stream);

/* TEXT-ONLY noisy pass of certificate-guided routing [Look Only When Needed,
 * method step (2): the vision rows removed, position ids kept]: one forward
 * of n_rows noisy rows (tokens, masked as in dvlm_forward) at slots L..L+n-1
 * over all layers in which attention does not see cache slots
 * 0..n_hidden-1 (the vision rows at the front of the cache); RoPE positions
 * and the K/V written for the rows stay absolute.  L is not advanced.
 * x_out [n_rows, H] (bf16, may be NULL) receives the final residual stream.
 * bf16 engines only (DVLM_ERR_UNSUPPORTED otherwise); 0 <= n_hidden <= L,
 * n_hidden % 8 == 0 (DVLM_ERR_SHAPE otherwise).  Reads L to the host
 * (synchronises the stream) and launches eagerly. */
DVLM_API dvlm_status dvlm_forward_text_only(dvlm_engine* e, const int32_t* tokens, const uint8_t* masked,
                                           int n_rows, int n_hidden, void* x_out, dvlm_stream stream);

/* FP8 row quantisation for the W8A8 projections [Fast-dVLM technical
 * overview (ocdem.com), section 2.3.2: the served model is quantised to W8A8
 * FP8].  For each row r of a (bf16 [rows, K], device, row-major): scales[r]
 * = max_k |a[r,k]| / 448 (1 for an all-zero row; fp32, device [rows]) and
 * codes[r,k] = E4M3(a[r,k] / scales[r]) (device uint8 [rows, K]; E4M3 finite
 * variant, round to nearest even, formed from the exact quotient in fp64).
 * Rows are a weight matrix's output channels.  Errors: INVALID_ARG (NULL
 * pointer), SHAPE (rows or K < 1).  One launch on `stream`, asynchronous. */
DVLM_API dvlm_status dvlm_quantize_rows_e4m3(const void* a, int rows, int K, uint8_t* codes, float* scales,
                                            dvlm_stream stream);

/* Trace of the decode driver (test hook).  When set, every forward that
 * dvlm_decode_block / dvlm_generate run (noisy, causal append, draft, verify,
 * AR) appends one record to buf (device, caller-owned, 16-byte aligned) and
 * increments *count (device int32, zeroed by the caller); records past the
 * capacity bytes / dvlm_engine_trace_record_bytes(m) are dropped and the
 * count stops there.  A record holds 112 int32 words and then the final
 * residual stream of the forward's rows before the final RMSNorm (16 x H
 * values in the model's dtype):
 *   [0] kind (1 noisy, 2 causal append, 3 speculative draft, 4 speculative
 *   verify, 5 AR), [1] cache length L at the forward, [2] rows, [3] clean
 *   rows, [4] LM-head rows R; [8..23] block tokens before the forward,
 *   [24..39] masked flags before (1 = still masked); [40..55] the LM head's
 *   top-1 id of rows 0..R-1 and [56..71] their top-1 probability (fp32
 *   bits); [72..87] block tokens after the LM head's commit, [88..103]
 *   masked flags after; [104] the pending AR seed and [105] the cache length
 *   after the forward.
 * The kernels run inside the captured CUDA graphs (setting or clearing the
 * trace drops them).  buf == NULL clears the trace.  Errors: INVALID_ARG,
 * WORKSPACE (room for less than one record).  Decisions and outputs of the
 * decode do not change. */
DVLM_API size_t dvlm_engine_trace_record_bytes(const dvlm_model* m);
DVLM_API dvlm_status dvlm_engine_set_trace(dvlm_engine* e, void* buf, size_t bytes, int32_t* count);

/* Profiling hook: one forward pass like dvlm_forward over all layers (L is
 * not advanced), launched eagerly with a CUDA event pair around every kernel
 * on `stream`.  ms_out[8] receives the device time per kernel class summed
 * over layers and counts_out[8] the launches: [0] embedding, [1] QKV GEMM,
 * [2] attention, [3] O-projection GEMM, [4] gate/up GEMM, [5] down GEMM,
 * [6] fused LM head (run when with_lm_head != 0, rows 0..n_rows-1, no
 * commit), [7] persistent forward (option "persistent": every decoder
 * layer in one launch; classes 1 to 5 are then empty).
 * Synchronises the stream. */
DVLM_API dvlm_status dvlm_profile_forward(dvlm_engine* e, const int32_t* tokens, const uint8_t* masked,
                                          int n_rows, int n_clean, int with_lm_head, float* ms_out,
                                          int* counts_out, dvlm_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* DVLM_H_ */
