/*
 * dsa.h -- C ABI of libdsa.so: DeepSeek Sparse Attention (DSA) on one
 * NVIDIA B200 (sm_100a).
 *
 * The method has three stages, all on the GPU:
 *   1. lightning indexer: for every causal (query t, key s) pair
 *        I[t,s] = sum_h w[t,h] * ReLU(scale * q[t,h] . k[s])
 *      over a 128-wide FP8 (e4m3) indexer key cache
 *      ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理", section 4, step 2;
 *       FP8 and ReLU: "m.gxzdkb.com/media/457.html", section "秘密武器");
 *   2. top-k: each query keeps its k best keys (k = 2048 by default), or
 *      every key when it sees at most k of them (page 3, section 4, step 3
 *      and section 2 "风险边界明确"); ties go to the smaller key index;
 *   3. sparse MLA: softmax attention over the selected keys only, against a
 *      512 + 64 wide bf16 latent cache whose first 512 dims are the values
 *      (page 3, section 4, step 4 and section 3 "稀疏多潜在注意力").
 *
 * Conventions shared by every entry point
 *  - All pointers are DEVICE pointers of the current CUDA device unless a
 *    parameter says otherwise. The caller owns every buffer, including any
 *    workspace; the library never allocates or frees device memory.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and the call returns without synchronising.
 *  - Arguments are checked on the host before anything is launched; a call
 *    that fails a check returns DSA_ERR_INVALID_ARG (or DSA_ERR_UNSUPPORTED)
 *    and launches nothing. A failed launch returns DSA_ERR_CUDA.
 *  - Faults found by the kernels (an index or block id out of range, which
 *    is then skipped; a bounded wait that gave up, after which the kernel
 *    returns early) are recorded in a per-device error word and reported by
 *    dsa_get_device_error(). While a timeout is recorded, every kernel of
 *    this library returns at once, so read and clear the word after a
 *    failure.
 *  - Buffers handed to the tensor memory accelerator must be 16-byte
 *    aligned; row pitches are fixed by the layouts below (128 B for FP8
 *    rows, 1152 B for 576-wide bf16 rows).
 *  - Index sets are returned sorted by key index (ascending), then padded
 *    with -1. Sets, not orders, are the result.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = -1,     /* bad pointer, size, alignment or layout */
  DSA_ERR_UNSUPPORTED = -2,     /* valid but not supported (e.g. head count) */
  DSA_ERR_WORKSPACE = -3,       /* workspace missing or too small */
  DSA_ERR_CUDA = -4,            /* a CUDA runtime call failed */
  DSA_ERR_TIMEOUT = -5,         /* a kernel's bounded wait gave up */
  DSA_ERR_DEVICE_BOUNDS = -6,   /* a kernel met an out-of-range index */
  DSA_ERR_NOT_IMPLEMENTED = -7
} dsa_status_t;

typedef void *dsa_stream_t; /* cudaStream_t */

/* Fixed widths of the caches. */
#define DSA_D_INDEX 128   /* indexer key / query width (e4m3) */
#define DSA_D_QK 576      /* MLA key width: 512 latent + 64 rope (bf16) */
#define DSA_D_V 512       /* MLA value width: the latent dims */
#define DSA_BLOCK 64      /* tokens per block of the paged cache */

/* Human-readable name of a status code. Never NULL. */
const char *dsa_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int dsa_version(void);

/*
 * Text of the last CUDA runtime error an entry point of this thread turned
 * into DSA_ERR_CUDA ("" if none). The string is owned by the library and
 * stays valid until the next failing call on the same thread.
 */
const char *dsa_last_error_string(void);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word. Returns DSA_OK, DSA_ERR_TIMEOUT (takes precedence) or
 * DSA_ERR_DEVICE_BOUNDS; DSA_ERR_CUDA if the synchronisation itself failed.
 */
int dsa_get_device_error(dsa_stream_t stream);

/*
 * Debug aid for failure handling; the pages have no counterpart. With a bit
 * of `mask` set, every later launch of the named kernel on the current
 * device first makes its MMA-issuing thread wait on a barrier that nothing
 * arrives at. That wait, bounded like every wait in the library (1 s), runs
 * out; the kernel records DSA_ERR_TIMEOUT in the device's error word and
 * leaves through its give-up path (every CTA drains its own copies in
 * flight and frees its tensor memory), and later kernels of the library
 * return at once until dsa_get_device_error() clears the word. Nothing
 * faults or traps. mask = 0 restores normal operation.
 *   DSA_DEBUG_STALL_INDEXER  the indexer (dsa_indexer_scores, and the
 *                            indexer launches inside dsa_forward,
 *                            dsa_forward_fused and dsa_decode_paged)
 *   DSA_DEBUG_STALL_MLA      the sparse MLA (every entry point that runs it)
 * Synchronises the device. Returns DSA_ERR_INVALID_ARG for unknown bits.
 */
#define DSA_DEBUG_STALL_INDEXER 1u
#define DSA_DEBUG_STALL_MLA 2u
int dsa_debug_stall(unsigned mask);

/*
 * Stage 1, lightning indexer scores (section 4 step 2 of page 3).
 *
 *   q8      [T][Hi][128] e4m3 codes of the indexer queries
 *   q_scale [T] fp32 per-token dequantisation scale, or NULL (= 1)
 *   k8      [S][128] e4m3 codes of the indexer key cache
 *   k_scale [S] fp32 per-token scale, or NULL (= 1); must be > 0
 *   w       [T][Hi] fp32 per-head weights (any sign)
 *   T, S    query rows and cached keys; query row t sits at position
 *           q_pos0 + t and sees keys 0 .. min(q_pos0 + t, S - 1)
 *   Hi      indexer heads: 1, 2, 4, 8, 16, 32 or 64
 *   scale   positive score scale
 *   scores  [T][ld] fp32 out: scores[t][s] = I[t,s] for every visible key
 *           s; entries of later keys are unspecified (a key past the query
 *           in the same 128-key tile reads -inf, others are not written)
 *   ld      row pitch of `scores` in elements, >= S, multiple of 4
 * All positive scales commute with ReLU, so they are applied after the
 * head sum: I = k_scale[s] * sum_h (w * scale * q_scale[t]) * ReLU(q8 . k8).
 */
int dsa_indexer_scores(const void *q8, const float *q_scale, const void *k8,
                       const float *k_scale, const float *w, int T, int S,
                       int Hi, int q_pos0, float scale, float *scores,
                       int64_t ld, dsa_stream_t stream);

/*
 * Stage 2, per-query top-k (section 4 step 3 of page 3).
 *
 *   scores  [T][ld] fp32 as written by dsa_indexer_scores; only the first
 *           min(q_pos0 + t + 1, S) entries of row t are read
 *   k       keys to keep per query, 1 .. 65536, multiple of 4
 *   idx     [T][k] int32 out: the keys with the k largest scores (ties to
 *           the smaller index), or every visible key when there are at
 *           most k, sorted by key index and padded with -1
 *   ld      multiple of 4; `scores` 16-byte aligned
 */
int dsa_topk(const float *scores, int T, int S, int64_t ld, int q_pos0, int k,
             int32_t *idx, dsa_stream_t stream);

/*
 * Stage 3, sparse MLA forward (section 4 step 4 of page 3).
 *
 *   q       [T][H][576] bf16 queries (absorbed MLA form: every head
 *           attends over the shared latent row)
 *   kv      [S][576] bf16 latent cache; values are kv[:, :512]
 *   idx     [T][k] int32 selected key positions in [0, S); -1 entries are
 *           skipped; k multiple of 4
 *   H       heads, 1 .. 128
 *   out     [T][H][512] bf16 out: softmax(sm_scale * q . kv[idx]) kv[idx, :512]
 *   lse     [T][H] fp32 out (natural log of the softmax denominator,
 *           including the max), or NULL; -inf when no key is selected
 */
int dsa_sparse_mla_fwd(const void *q, const void *kv, const int32_t *idx,
                       int T, int S, int H, int k, float sm_scale, void *out,
                       float *lse, dsa_stream_t stream);

/*
 * Step 1 of the workflow (page 3, section 4 "步骤一：查询与键的投影"; page 5,
 * section "第一步"): the hidden states are projected to the indexer's queries
 * and keys, rotary position encoding is applied to both, and each indexer
 * head gets a weight a_h, a linear map of the same hidden state. The outputs
 * are the FP8 inputs dsa_indexer_scores takes.
 *
 *   h       [T][d] bf16 hidden states, d a multiple of 8; T at most
 *           65535 * 128 (the GEMM's row tiles)
 *   wt      [Hi*128 + 128 + Hi][d] bf16: the rows of W_Q (Hi heads x 128),
 *           then W_K (128), then W_a (Hi), each row one output's weights
 *   rope    [T][64][2] fp32 (cos, sin) of each token's position for the 64
 *           dimension pairs (2i, 2i+1) of a 128-wide head; pair i of q (every
 *           head) and of k becomes (y0 cos - y1 sin, y0 sin + y1 cos)
 *   q8      [T][Hi][128] e4m3 out, q_scale [T] fp32 out
 *   k8      [T][128] e4m3 out, k_scale [T] fp32 out
 *   a       [T][Hi] fp32 out (a_h, not scaled)
 *   Scales are per token, over all of its q (or k) values: scale = amax / 448
 *   (1 when amax = 0); codes are e4m3(y / scale), rounded to nearest even and
 *   saturated at +-448.
 *   workspace  >= dsa_project_workspace_size(T, Hi) bytes, 16-byte aligned,
 *              caller-owned (fp32 rotated q and k, per-token maxima)
 * Hi in {1, 2, 4, ..., 64}; the library has no counterpart for the widths,
 * which the pages leave open.
 */
size_t dsa_project_workspace_size(int T, int Hi);
int dsa_project_indexer_inputs(const void *h, const void *wt, const float *rope, int T,
                               int d, int Hi, void *q8, float *q_scale, void *k8,
                               float *k_scale, float *a, void *workspace, size_t ws_bytes,
                               dsa_stream_t stream);

/*
 * The indexer's warm-up objective (page 2, section "四、训练的两步走冷启动"):
 * dense attention is run, the weight distribution each token receives is the
 * target, and the indexer alone is trained to fit it with a KL divergence.
 * The target of query t is read as the dense causal attention distribution
 * averaged over heads; the indexer's distribution is softmax(I[t, s]) over
 * the same keys. Row t sits at position q_pos0 + t and sees keys 0 .. that
 * position (clamped to S - 1). fp32 results.
 *
 * dsa_attention_probs_mean:
 *   p[t][s] = (1/H) sum_h exp(sm_scale q[t,h] . kv[s] - lse[t][h]), 0 past the
 *   row's keys; q [T][H][576] bf16, kv [S][576] bf16, lse [T][H] the natural
 *   log normaliser of each head, as dsa_sparse_mla_fwd returns it over index
 *   sets covering every causal key (dsa_window_indices with window >= S);
 *   p [T][ldp] fp32 out. The logits q . kv go through a tensor-core GEMM into
 *   the caller's workspace of dsa_attention_probs_workspace_size(T, S, H)
 *   bytes (T * H rows of S fp32, S rounded up to 4); T * H at most 65535 * 128.
 * dsa_indexer_kl:
 *   loss[t] = sum_s p[t][s] (log p[t][s] - log r[t][s]), r = softmax(I[t, :]);
 *   grad[t][s] = r[t][s] - p[t][s] (dloss/dI), 0 past the row's keys.
 *   I [T][ldi], p [T][ldp], grad [T][ldg] fp32; loss [T] fp32.
 * dsa_indexer_backward:
 *   through I = sum_h w * ReLU(scale * qf . kf) with qf = q8 * q_scale and
 *   kf = k8 * k_scale (the FP8 inputs dsa_indexer_scores takes), given
 *   grad = dloss/dI [T][ldg]: dq [T][Hi][128] (w.r.t. qf), dk [S][128]
 *   (w.r.t. kf), dw [T][Hi], all fp32, caller-owned, dq and dk 16-byte
 *   aligned; dk sums over the T rows given (a caller splitting the rows into
 *   chunks adds the chunks' dk). The products q8 . k8, dq and dk are tensor-
 *   core GEMMs through the caller's workspace of
 *   dsa_indexer_backward_workspace_size(T, S, Hi) bytes, about
 *   T * Hi * S * 10 bytes (keep T * Hi * S near 2^28 or below by chunking the
 *   rows); T * Hi and S at most 65535 * 128 (the GEMM's row tiles).
 * Each returns DSA_ERR_INVALID_ARG (nothing launched) on bad arguments,
 * DSA_ERR_WORKSPACE for a missing or short workspace, and
 * DSA_ERR_UNSUPPORTED for an indexer head count outside {1, 2, 4, ..., 64}.
 */
size_t dsa_attention_probs_workspace_size(int T, int S, int H);
int dsa_attention_probs_mean(const void *q, const void *kv, const float *lse, int T, int S,
                             int H, int q_pos0, float sm_scale, float *p, int64_t ldp,
                             void *workspace, size_t ws_bytes, dsa_stream_t stream);
int dsa_indexer_kl(const float *I, int64_t ldi, const float *p, int64_t ldp, int T, int S,
                   int q_pos0, float *loss, float *grad, int64_t ldg, dsa_stream_t stream);
size_t dsa_indexer_backward_workspace_size(int T, int S, int Hi);
int dsa_indexer_backward(const void *q8, const float *q_scale, const void *k8,
                         const float *k_scale, const float *w, int T, int S, int Hi, int q_pos0,
                         float scale, const float *grad, int64_t ldg, float *dq, float *dk,
                         float *dw, void *workspace, size_t ws_bytes, dsa_stream_t stream);

/*
 * Index sets for sliding-window and dense causal attention, to run through
 * dsa_sparse_mla_fwd in place of the top-k selection. Sliding-window
 * attention keeps a fixed number of the keys just before each token (page 1,
 * section "秘密武器"; page 4, section "Sparse Attention"), and DSA generalises
 * it; a window covering the whole causal prefix is dense causal attention,
 * the full interface page 2 (section "六、实测表现与取舍") keeps beside DSA.
 *
 *   row t (position p = min(q_pos0 + t, S - 1)) gets the keys
 *   max(0, p - window + 1) .. p in increasing order, then -1 up to k.
 *
 *   window  1 .. k; keys per row, the query's own position included
 *   k       row length of idx, multiple of 4
 *   idx     [T][k] int32 out, 16-byte aligned, caller-owned
 * Returns DSA_ERR_INVALID_ARG (nothing launched) for window > k or other bad
 * arguments.
 */
int dsa_window_indices(int T, int S, int q_pos0, int window, int k, int32_t *idx,
                       dsa_stream_t stream);

/*
 * Dense causal MLA, the full interface page 2 keeps beside DSA ("六、实测表现与
 * 取舍"): the same kernel as dsa_sparse_mla_fwd with every causal key selected,
 * the slots generated in the kernel (no index sets in memory). It is the
 * baseline DSA is measured against: attention whose cost grows with the whole
 * context, where DSA's grows with k (page 1, section "秘密武器").
 *
 * dsa_dense_causal_mla: query row t (position q_pos0 + t) attends to keys
 *   0 .. min(q_pos0 + t, S - 1) of kv [S][576]; q, out, lse as for
 *   dsa_sparse_mla_fwd.
 * dsa_dense_causal_mla_decode_paged: query j of sequence b attends to its
 *   sequence's keys 0 .. seq_len[b] - nq + j through the block table;
 *   arguments as for dsa_sparse_mla_decode_paged without idx and k.
 * Both return DSA_ERR_INVALID_ARG (nothing launched) for bad arguments and
 * DSA_ERR_UNSUPPORTED for H outside 1 .. 128.
 */
int dsa_dense_causal_mla(const void *q, const void *kv, int T, int S, int H, int q_pos0,
                         float sm_scale, void *out, float *lse, dsa_stream_t stream);
int dsa_dense_causal_mla_decode_paged(const void *q, const void *kv_pool,
                                      const int32_t *block_table, const int32_t *seq_len,
                                      int B, int nq, int max_blocks, int nblk, int H,
                                      float sm_scale, void *out, float *lse,
                                      dsa_stream_t stream);

/*
 * Whole prefill path: indexer -> top-k -> sparse MLA, the chain of steps 2
 * to 4 of the four-step workflow ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
 * section 4: scores, top-k selection, attention over the selected positions
 * only) run over a whole prompt, the prefill phase page 1 distinguishes
 * from decoding ("m.gxzdkb.com/media/457.html", section "秘密武器"), for T query rows at
 * positions q_pos0 .. q_pos0 + T - 1 against S cached keys (S >= q_pos0 + T
 * for a self-contained prefill). Query rows are scored in chunks of `chunk`
 * rows (0 = all rows at once); the workspace holds the scores of two chunks
 * (one when there is a single chunk), so that the top-k of one chunk runs on
 * a library-owned side stream beside the indexer of the next. The side stream
 * and its events are created on the first multi-chunk call on a device (no
 * device memory is allocated) and joined back into `stream` before the
 * attention launch; concurrent calls on one device enqueue one at a time.
 *
 *   idx_out [T][k] int32 out (the selection), or NULL to keep it in the
 *           workspace only
 *   workspace  at least dsa_forward_workspace_size() bytes, 256-byte aligned
 *   other arguments as for the three stages.
 */
size_t dsa_forward_workspace_size(int T, int S, int Hi, int H, int k,
                                  int chunk);
int dsa_forward(const void *q8, const float *q_scale, const void *k8,
                const float *k_scale, const float *w, const void *q,
                const void *kv, int T, int S, int Hi, int H, int q_pos0, int k,
                int chunk, float scale, float sm_scale, int32_t *idx_out,
                void *out, float *lse, void *workspace, size_t ws_bytes,
                dsa_stream_t stream);

/*
 * The same prefill with the top-k fused into the indexer, so no score row
 * reaches HBM: same arguments, layouts and results as dsa_forward (the
 * selection is the k largest scores, ties to the smaller key). Per chunk of
 * `chunk` rows:
 *  - the indexer scores each row against a sample of the keys (the first 256
 *    of every 4096, copied into the workspace);
 *  - per row, a threshold from its sampled scores with, in expectation, about
 *    1.4 k of its keys at or above it;
 *  - the indexer runs again over every key, appending only the (key, score)
 *    pairs at or above the threshold to the row's candidate list;
 *  - with k to 4096 candidates the k largest are among them and are chosen
 *    exactly; any other row (rare) has its scores recomputed on CUDA cores
 *    and selected in full.
 * The workspace, dsa_forward_fused_workspace_size(...) bytes (0: not
 * supported), holds the sample, the candidate lists and one scratch score
 * row per recompute CTA: about 1.4 GB at T = S = 131072 with 4096-row chunks
 * and k = 2048 (idx included), against 5.4 GB for dsa_forward.
 * Supports k <= 2048 and S <= 131072 (DSA_ERR_UNSUPPORTED otherwise); q8 and
 * k8 16-byte aligned; the workspace 256-byte aligned.
 */
size_t dsa_forward_fused_workspace_size(int T, int S, int Hi, int H, int k, int chunk);
int dsa_forward_fused(const void *q8, const float *q_scale, const void *k8,
                      const float *k_scale, const float *w, const void *q,
                      const void *kv, int T, int S, int Hi, int H, int q_pos0, int k,
                      int chunk, float scale, float sm_scale, int32_t *idx_out,
                      void *out, float *lse, void *workspace, size_t ws_bytes,
                      dsa_stream_t stream);

/*
 * Diagnostic for dsa_forward_fused (no counterpart on the pages): how many
 * rows of the last call that used `workspace` (with the same T, S, k and
 * chunk) missed their candidate window and were recomputed on CUDA cores.
 * Synchronises `stream`; returns the count (>= 0) or a negative status.
 * Recomputed scores are summed in another order than the tensor cores', so
 * on inputs off the exact FP8 grid they equal the indexer's scores only to
 * within fp32 rounding (their selection then agrees within the tie rule).
 */
int dsa_forward_fused_fallback_rows(const void *workspace, int T, int S, int k,
                                    int chunk, dsa_stream_t stream);

/*
 * Batched decode over a paged cache (blocks of 64 tokens): the same three
 * steps (page 3, section 4, steps 2-4) for the few new tokens of each
 * sequence, the decoding phase page 1 (section "秘密武器") contrasts with
 * prefill, each new query scoring and selecting from its own sequence's
 * cached keys. The pages do not describe the cache's memory layout; the
 * paged blocks of 64 tokens with a per-sequence block table are this
 * library's layout for a batch of sequences of different lengths.
 *
 *   q8 [B][nq][Hi][128] e4m3, q_scale [B][nq] fp32 (or NULL), w [B][nq][Hi]
 *   q  [B][nq][H][576] bf16
 *   k8_pool      [nblk][64][128] e4m3; k_scale_pool [nblk][64] fp32 or NULL
 *   kv_pool      [nblk][64][576] bf16
 *   block_table  [B][max_blocks] int32: physical block of each logical
 *                block of a sequence (entries past the end are not read)
 *   seq_len      [B] int32: tokens of each sequence, nq <= seq_len[b] <=
 *                64 * max_blocks (launches are sized from max_blocks, so
 *                no host copy is needed)
 *   nq           new query tokens per sequence; query j of sequence b sits
 *                at position seq_len[b] - nq + j and sees keys 0 .. that
 *                position (causal between the new tokens)
 *   idx_out      [B][nq][k] logical key positions out, or NULL
 *   out [B][nq][H][512] bf16, lse [B][nq][H] fp32 (or NULL)
 *   workspace    scratch for the per-query score rows, at least
 *                dsa_decode_paged_workspace_size() bytes, 256-byte aligned
 */
size_t dsa_decode_paged_workspace_size(int B, int nq, int max_blocks, int Hi,
                                       int H, int k);
int dsa_decode_paged(const void *q8, const float *q_scale, const float *w,
                     const void *q, const void *k8_pool,
                     const float *k_scale_pool, const void *kv_pool,
                     const int32_t *block_table, const int32_t *seq_len,
                     int B, int nq,
                     int max_blocks, int nblk, int Hi, int H, int k,
                     float scale, float sm_scale, int32_t *idx_out, void *out,
                     float *lse, void *workspace, size_t ws_bytes,
                     dsa_stream_t stream);

/*
 * Paged decode that allocates nothing, for callers that cannot allocate
 * device memory: code running where cudaMalloc is not allowed or not safe
 * (a host callback, a plugin living inside another framework's memory
 * pool, a tool with no device allocator of its own). The pages describe no
 * such entry point; it is a convenience of this library.
 *
 * Same arguments and results as dsa_decode_paged(), without the workspace.
 * The scratch is a fixed 32 MiB array inside the library, present on every
 * GPU that loads libdsa.so until the process exits. A call whose scratch
 * need, dsa_decode_paged_workspace_size(B, nq, max_blocks, Hi, H, k), is
 * above 32 MiB is rejected with DSA_ERR_WORKSPACE before anything is
 * launched (dsa_last_error_string() says why).
 *  - The first call on each device looks up the array's device address
 *    with that device current; make that first call before any stream
 *    capture begins.
 *  - All calls on a device share the one array. Calls whose GPU work
 *    overlaps (different streams, or different host threads, without
 *    ordering between them) race on it; serialise them. Every byte a call
 *    reads from the scratch is written earlier in the same call, so the
 *    previous call's leftovers never leak into a result.
 *  - The array's device address is cached per device for the life of the
 *    process. After cudaDeviceReset() (or anything else that unloads the
 *    library's module from a device) the cached address is stale: do not
 *    call this entry point on that device again in the same process.
 */
int dsa_decode_paged_noalloc(const void *q8, const float *q_scale,
                             const float *w, const void *q,
                             const void *k8_pool, const float *k_scale_pool,
                             const void *kv_pool, const int32_t *block_table,
                             const int32_t *seq_len, int B, int nq,
                             int max_blocks, int nblk, int Hi, int H, int k,
                             float scale, float sm_scale, int32_t *idx_out,
                             void *out, float *lse, dsa_stream_t stream);

/*
 * The sparse MLA stage of the paged decode on its own (page 3, section 4,
 * step 4, and section 3 "稀疏多潜在注意力": softmax attention of every head
 * over the selected rows of the shared latent cache): like
 * dsa_sparse_mla_fwd, but `idx` [B*nq][k] holds logical positions of each
 * sequence, translated through block_table into kv_pool rows. A position
 * past the query's own position counts as out of range.
 */
int dsa_sparse_mla_decode_paged(const void *q, const void *kv_pool,
                                const int32_t *block_table,
                                const int32_t *seq_len, const int32_t *idx,
                                int B, int nq, int max_blocks, int nblk, int H,
                                int k, float sm_scale, void *out, float *lse,
                                dsa_stream_t stream);

/*
 * Splitting the work over several GPUs (host only: no CUDA call, nothing
 * launched). The pages describe no distributed step; every prefill row and
 * every decode sequence is independent given the caches, which each GPU
 * holds whole. The causal prefix makes a row's cost grow with its position,
 * so units are balanced by estimated cost (BF16-flop equivalents of one row
 * seeing n keys: 128*Hi*n for the FP8 indexer at twice the BF16 rate, plus
 * 2176*H*min(n, k) for the sparse MLA) with the longest-first greedy rule:
 * units by cost, largest first (ties: lower unit), each to the least-loaded
 * worker so far (ties: lower worker). Every worker computes the same plan,
 * so the call needs no communication; the parts are disjoint and together
 * cover every unit.
 *
 * dsa_plan_prefill_chunks: the prefill's rows 0 .. T-1 (row t at position
 *   q_pos0 + t, seeing keys 0 .. min(q_pos0 + t, S - 1)) in chunks of `chunk`
 *   rows; writes the first rows of worker `part`'s chunks (ascending) to
 *   first_rows and returns how many. Chunk c covers rows
 *   [c*chunk, min((c+1)*chunk, T)); each runs as its own dsa_forward with
 *   q_pos0 + c*chunk.
 * dsa_plan_decode_sequences: the B sequences of a decode batch (nq queries
 *   each, query j seeing seq_len[b] - nq + j + 1 keys); writes worker `part`'s
 *   sequence numbers (ascending) to seqs and returns how many.
 * Both return DSA_ERR_INVALID_ARG for bad sizes, 1 <= parts <= 4096 and
 * 0 <= part < parts violated, seq_len[b] < nq, or an output array shorter
 * than the worker's share (max_chunks / max_seqs entries).
 */
int dsa_plan_prefill_chunks(int T, int S, int q_pos0, int Hi, int H, int k, int chunk,
                            int parts, int part, int32_t *first_rows, int max_chunks);
int dsa_plan_decode_sequences(const int32_t *seq_len, int B, int nq, int Hi, int H, int k,
                              int parts, int part, int32_t *seqs, int max_seqs);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
