/*
 * dsa_indexer.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention
 * lightning indexer: dense scoring + top-k, MISA head routing, HISA
 * block-then-token filtering.
 *
 * The method (sources: "MISA: Mixture of Indexer Sparse Attention for
 * Long-Context LLM Inference", sections "Problem statement", "Methodology",
 * "Hierarchical variant (MISA-dagger)"; "HISA: Efficient Hierarchical Indexing
 * for Fine-Grained Sparse Attention" review, section 3; "DoSA: Dots Sparse
 * Attention" review, section 3, for the signed head weights):
 *
 *   For query t at absolute position p_t = q_offset + t, every key s <= p_t
 *   (s < L) is scored by H indexer heads,
 *       I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]),
 *   and the top-k keys are kept for the downstream sparse attention.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, row-major, owned by the caller.
 *     The library allocates nothing; scratch lives in a caller-provided
 *     workspace whose size the *_workspace_size functions return.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Arguments are validated on the host before any launch;
 *     a failed validation returns an error and launches nothing.
 *   - Selection: the k best candidates by (score descending, index ascending);
 *     fewer candidates than k -> all of them. Each output row lists the chosen
 *     indices in ascending order, padded with -1 (and score -inf).
 *   - The first 256 bytes of every workspace hold a device status word. Each
 *     call that passes validation clears it (stream-ordered); kernels set it
 *     if a bounded wait gave up. dsa_device_status() synchronises the stream
 *     and reports it. Zero a new workspace once before its first status read.
 *   - The workspace must be 256-byte aligned; q, k, w, q_scale and k_scale
 *     16-byte aligned.
 *   - Calls that share a workspace must not overlap in time (use one stream).
 *
 *   - Calls may come from several host threads (each with its own
 *     workspace); the current CUDA device is the one used. Device indices
 *     of 64 and above return DSA_ERR_UNSUPPORTED.
 *
 * Supported shapes: d in {64, 128}; bf16 H in {8, 16, 32, 64};
 * FP8 e4m3 (decode and prefill): d = 128, H in {32, 64}. Other shapes return
 * DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_INDEXER_H
#define DSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_EXPORT __attribute__((visibility("default")))
#else
#define DSA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DSA_BF16 = 0, DSA_FP8_E4M3 = 1 } dsa_dtype;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_ARG = -1,         /* null pointer, bad size, misaligned pointer            */
  DSA_ERR_UNSUPPORTED = -2, /* valid but not built: head count, head dim, dtype      */
  DSA_ERR_WORKSPACE = -3,   /* ws_bytes smaller than the *_workspace_size result     */
  DSA_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed           */
  DSA_ERR_TIMEOUT = -5      /* a device-side bounded wait gave up (dsa_device_status) */
} dsa_status;

/* One indexer problem: `batch` independent sequences, each with T queries at
 * positions q_offset .. q_offset+T-1 and a prefix of L keys. */
typedef struct {
  int batch;          /* independent sequences (decode: one query each)          */
  int T;              /* queries per sequence                                    */
  int L;              /* keys per sequence                                       */
  int H;              /* indexer heads                                           */
  int d;              /* head dimension                                          */
  long long q_offset; /* absolute position of query 0 (>= 0); key s is visible to
                         query t iff s <= q_offset + t                           */
  dsa_dtype qk_dtype; /* DSA_BF16: q, k bf16; DSA_FP8_E4M3: q, k e4m3 bytes       */
  const void* q;      /* [batch, T, H, d]                                        */
  const float* q_scale; /* [batch, T, H] per-(query, head) dequant scale (FP8), else NULL */
  const void* k;      /* [batch, L, d]                                           */
  const float* k_scale; /* [batch, L] per-token dequant scale (FP8), else NULL    */
  const float* w;     /* [batch, T, H] signed head weights, fp32                 */
} dsa_indexer_args;

/* Human-readable name of a status code (static storage). */
DSA_EXPORT const char* dsa_status_string(dsa_status s);

/* Synchronise `stream`, then report and clear the device status word of
 * `workspace`: DSA_ERR_TIMEOUT if a kernel's bounded wait gave up since the
 * last call that used this workspace, DSA_ERR_CUDA on a CUDA error, else OK. */
DSA_EXPORT dsa_status dsa_device_status(void* workspace, void* stream);

/* Self-test of the failure path (no counterpart on the pages): launches one
 * warp whose bounded wait on a barrier that nothing completes gives up after
 * the wait limit (2 s), records the timeout in the workspace's status word and
 * returns; dsa_device_status then reports DSA_ERR_TIMEOUT and the context
 * stays usable. Workspace: the 256-byte header only. */
DSA_EXPORT dsa_status dsa_selftest_wait_timeout(void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ dense indexer
 * indexer_score_topk: for every query of every sequence, score all visible
 * keys with all H heads and keep the top `topk`.
 *   out_idx   [batch, T, topk] int32 key indices (ascending, -1 padded)
 *   out_score [batch, T, topk] fp32 scores of those keys, or NULL
 * bf16 inputs score on tcgen05 bf16 MMAs; FP8 inputs use FP8 MMAs with
 *   I[t,s] = k_scale[s] * sum_h (w[t,h] * q_scale[t,h]) * ReLU(q8[t,h,:] . k8[s,:]).
 * Workspace: [batch*T*L] fp32 scores plus the 256-byte header. */
DSA_EXPORT size_t indexer_workspace_size(const dsa_indexer_args* a, int topk);
DSA_EXPORT dsa_status indexer_score_topk(const dsa_indexer_args* a, int topk, int32_t* out_idx,
                              float* out_score, void* workspace, size_t ws_bytes, void* stream);

/* indexer_score_topk_noalloc: the same dense score + top-k as
 * indexer_score_topk, for callers that cannot allocate device memory: a
 * plugin handed a fixed memory arena by a host runtime that owns every device
 * allocation, a latency-critical loop where cudaMalloc (which may synchronise
 * the device) is not allowed, or a caller with no allocator at all (no torch,
 * no permission to grow its device footprint). It takes no workspace: its
 * scores scratch is a 64 MiB array in the library's own device memory
 * (reserved on every GPU that loads the library, until the process exits), so
 * it accepts problems with 256 + 4 * batch * T * L <= 64 MiB (e.g. 64 decode
 * sequences of 131072 keys) and returns DSA_ERR_WORKSPACE for larger ones.
 * It allocates nothing and calls no allocating routine. Every call looks the
 * scratch's device address up (cudaGetSymbolAddress, on the current device);
 * the first call on a device also loads the library's module there, and the
 * first call of each shape class (head dim, head count, dtype, row length
 * class) sets that kernel's shared-memory attribute on the host, so make one
 * call of every shape before a phase that must not do either.
 * Every call on a device shares the one scratch array, which keeps the last
 * call's scores: calls that may overlap on the GPU (different streams, no
 * ordering between them) race and must not be issued. The status word at the
 * start of the scratch is cleared by each call; dsa_noalloc_status reads it.
 * No method page has a counterpart of this entry point; it is plumbing. */
DSA_EXPORT dsa_status indexer_score_topk_noalloc(const dsa_indexer_args* a, int topk,
                                                 int32_t* out_idx, float* out_score, void* stream);

/* Synchronise `stream`, then report and clear the status word of the static
 * scratch that indexer_score_topk_noalloc uses on the current device:
 * DSA_ERR_TIMEOUT if a bounded device wait gave up inside such a call since
 * the last read, DSA_ERR_CUDA on a CUDA error, else DSA_OK (the analogue of
 * dsa_device_status for the call that has no workspace). */
DSA_EXPORT dsa_status dsa_noalloc_status(void* stream);

/* indexer_score_topk_lists: the same selection as indexer_score_topk with the
 * scoring fused with a filter (the LiteTopK idea named in the "DoSA: Dots
 * Sparse Attention" review: scoring and filtering fused to cut memory
 * traffic), kept exact:
 *   1. every S-th visible key (S = 16, or larger so a row has at most 4096)
 *      is scored; from that sample each query gets a threshold its k-th
 *      score very likely reaches (the sample rank expected for the k-th score
 *      + 4 binomial standard deviations + 4);
 *   2. the score pass keeps no full scores: every visible score >= the
 *      query's threshold goes, with its key, to the query's candidate list;
 *   3. a query whose list holds at least min(k, visible) entries has its
 *      top-k in the list (its k-th score reaches the threshold); the other
 *      queries' groups (256 / H queries) are re-scored in full;
 *   4. top-k from the lists (or the full scores), score descending, index
 *      ascending.
 * Output and ordering as indexer_score_topk, bit for bit. bf16; rows of at
 * least 4096 keys, L a multiple of S, topk <= L / 8, else
 * DSA_ERR_UNSUPPORTED. Workspace: indexer_lists_workspace_size bytes (0
 * when unsupported). */
DSA_EXPORT size_t indexer_lists_workspace_size(const dsa_indexer_args* a, int topk);
DSA_EXPORT dsa_status indexer_score_topk_lists(const dsa_indexer_args* a, int topk, int32_t* out_idx,
                                               float* out_score, void* workspace, size_t ws_bytes, void* stream);

/* Stage 1 alone: write the scores I[t,s] of all visible keys into
 * out_scores[(b*T + t) * ld + s] (ld >= L). Entries with s > q_offset + t are
 * left untouched. Workspace: the 256-byte header only. */
DSA_EXPORT dsa_status indexer_scores(const dsa_indexer_args* a, float* out_scores, long long ld,
                          void* workspace, size_t ws_bytes, void* stream);

/* Gathered re-scoring (the MISA-dagger re-score and HISA token stages alone):
 * for every query (row r = b*T + t) and compact position c < n_slots * blk,
 * with token s = cand[r * n_slots + c / blk] * blk + c % blk,
 *     out[r * ld + c] = I[t, s]  (all H heads)  if cand[...] >= 0, s < L, s <= q_offset + t,
 *     out[r * ld + c] = -inf                      otherwise.
 * blk = 1: token candidates; blk = B: candidate blocks of B tokens (a block
 * size that is a multiple of 128 fetches whole blocks with TMA).
 *   cand [batch*T, n_slots] int32; out [batch*T, ld] fp32, ld >= n_slots * blk.
 * d = 128, H in {32, 64}; bf16 or FP8 e4m3 (FP8: 128-byte key rows, each
 * gathered key's score times its k_scale, the head weights times q_scale).
 * Workspace: the 256-byte header only. */
DSA_EXPORT dsa_status indexer_score_gathered(const dsa_indexer_args* a, const int32_t* cand,
                                             int n_slots, int blk, float* out, long long ld,
                                             void* workspace, size_t ws_bytes, void* stream);

/* Stage 2 alone: per-row top-k of fp32 scores [rows, ld]. Row r belongs to
 * query t = r % T; its candidates are positions 0 .. n_r - 1 with
 *   n_r = clamp((q_offset + t) / pstride + 1, 0, row_len)   if pstride > 0,
 *   n_r = row_len                                           if pstride == 0.
 * -inf marks an absent candidate. Selected positions j are written as
 *   cand[r * n_slots + j / blk] * blk + j % blk   if cand != NULL, else j.
 * Workspace: the 256-byte header only. */
DSA_EXPORT dsa_status indexer_topk_rows(const float* scores, long long rows, long long ld, int T,
                             long long q_offset, int pstride, int row_len, int topk,
                             const int32_t* cand, int n_slots, int blk, int32_t* out_idx,
                             float* out_score, void* workspace, size_t ws_bytes, void* stream);

/* Pooled keys: kbar[b, m, :] = bf16(mean of k[b, m*block : min((m+1)*block, L), :]),
 * m < M = ceil(L / block); mean in fp64, rounded once (nearest even). bf16 only.
 *   k [batch, L, d] bf16 -> kbar [batch, M, d] bf16. */
DSA_EXPORT dsa_status dsa_meanpool_keys(const void* k, int batch, int L, int d, int block, void* kbar,
                             void* stream);

/* ------------------------------------------------------------ MISA
 * misa_route_score_topk (MISA page, "Methodology"): split the prefix into
 * M = ceil(L / block) blocks of mean-pooled keys kbar; per query and head the
 * router affinity
 *     a[t,h] = |w[t,h]| * sum over blocks m with m*block <= p_t of ReLU(q[t,h,:] . kbar[m,:]);
 * keep the top-h heads per query (ties -> lower head); score every visible
 * token with those heads only (their original signed weights); keep the top
 * `topk` (kprime == 0), or, MISA-dagger (kprime > 0), keep the top `kprime`
 * candidates, re-score them with all H heads and keep the top `topk`.
 *   out_idx   [batch, T, topk] int32 token indices
 *   out_score [batch, T, topk] fp32 (routed scores; full-H scores for MISA-dagger) or NULL
 *   out_heads [batch, T, h] int32 chosen heads (ascending) or NULL
 *   out_cand  [batch, T, kprime] int32 MISA-dagger candidates (ascending, -1 padded) or NULL
 * h in {8, 16, 32, 64}, h <= H; MISA-dagger needs d = 128 and H in {32, 64}.
 * bf16, or FP8 e4m3 (d = 128, H in {32, 64}; a prefill chunk or the decode
 * cache): the pooled keys are kept in the cache's format (per block the fp64
 * mean of the dequantised keys, scale absmax/448, e4m3 codes of mean / scale,
 * nearest even); the router weights each pooled key by its scale and each
 * affinity by q_scale[t,h]; the routed pass reads the kept heads' e4m3 rows
 * and scales; the MISA-dagger re-score gathers 128-byte e4m3 key rows. */
DSA_EXPORT size_t misa_workspace_size(const dsa_indexer_args* a, int block, int h, int topk, int kprime);
DSA_EXPORT dsa_status misa_route_score_topk(const dsa_indexer_args* a, int block, int h, int topk,
                                 int kprime, int32_t* out_idx, float* out_score,
                                 int32_t* out_heads, int32_t* out_cand, void* workspace,
                                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ HISA
 * hisa_block_filter_topk (HISA review, section 3): block-level coarse filter,
 * then token-level refinement. Pooled keys kbar as for MISA; block score
 *     S_b[t,m] = sum_h w[t,h] * ReLU(q[t,h,:] . kbar[m,:]) for blocks with m*block <= p_t;
 * keep the top-m blocks (ties -> lower block); score the visible tokens of the
 * kept blocks with the full indexer; keep the top `topk`.
 *   out_idx    [batch, T, topk] int32 token indices
 *   out_score  [batch, T, topk] fp32 token scores or NULL
 *   out_blocks [batch, T, m] int32 kept blocks (ascending, -1 padded) or NULL
 * d = 128 and H in {32, 64}. bf16 or FP8 e4m3 (a prefill chunk or the decode
 * cache): with FP8 the pooled keys are kept in the cache's format (per block
 * the fp64 mean of the dequantised keys, scale absmax/448, e4m3 codes of
 * mean / scale, nearest even), the block scores and the token scores use FP8
 * MMAs with the per-token / per-block and per-(query, head) scales, and block
 * must be a multiple of 128. Blocks that are whole 128-key tiles are refined
 * block major (hisa_refine_scores); others one query per tile (bf16). */
DSA_EXPORT size_t hisa_workspace_size(const dsa_indexer_args* a, int block, int m, int topk);
DSA_EXPORT dsa_status hisa_block_filter_topk(const dsa_indexer_args* a, int block, int m, int topk,
                                  int32_t* out_idx, float* out_score, int32_t* out_blocks,
                                  void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ pooled-key cache
 * The pooled keys MISA and HISA read depend only on the key cache, and a
 * completed block's pooled key never changes: a decode loop can keep them
 * (pool each block once, the last, still growing block again at each step)
 * instead of pooling the whole cache at every call.
 *
 * dsa_pool_keys: pools blocks m0 .. min(m1, M) - 1 of every sequence of
 * a->k (M = ceil(L / block)) into the cache, in the form the *_pooled calls
 * read:
 *   bf16:  kbar [batch, M, d] bf16 (as dsa_meanpool_keys); kbar_scale unused (may be NULL)
 *   FP8:   kbar [batch, M, d] e4m3 codes and kbar_scale [batch, M] fp32, the
 *          format described under misa_route_score_topk (fp64 mean of the
 *          dequantised keys, scale absmax/448, codes of mean / scale)
 * Entries outside [m0, m1) are left untouched. kbar: 16-byte aligned.
 * DSA_ERR_ARG for m0 < 0, m1 < m0 or a missing buffer.
 *
 * misa_route_score_topk_pooled / hisa_block_filter_topk_pooled: the same as
 * misa_route_score_topk / hisa_block_filter_topk (same outputs, same
 * workspace size), reading the pooled keys from kbar / kbar_scale (every
 * block of every sequence, as dsa_pool_keys writes them) instead of pooling
 * the key cache. The result equals the unpooled call's bit for bit when the
 * cache holds the pooled keys of the current a->k. */
DSA_EXPORT dsa_status dsa_pool_keys(const dsa_indexer_args* a, int block, int m0, int m1, void* kbar,
                                    float* kbar_scale, void* stream);
DSA_EXPORT dsa_status misa_route_score_topk_pooled(const dsa_indexer_args* a, int block, int h, int topk,
                                                   int kprime, const void* kbar, const float* kbar_scale,
                                                   int32_t* out_idx, float* out_score, int32_t* out_heads,
                                                   int32_t* out_cand, void* workspace, size_t ws_bytes,
                                                   void* stream);
DSA_EXPORT dsa_status hisa_block_filter_topk_pooled(const dsa_indexer_args* a, int block, int m, int topk,
                                                    const void* kbar, const float* kbar_scale, int32_t* out_idx,
                                                    float* out_score, int32_t* out_blocks, void* workspace,
                                                    size_t ws_bytes, void* stream);

/* HISA token refinement alone (HISA review, section 3 and Figure 1), block
 * major: the kept blocks [batch*T, m] (block ids, -1 = empty slot) are
 * inverted into per-block lists of the queries that kept them, and each kept
 * 128-token key tile is loaded once and scored against all of those queries:
 *     out[r * ld + slot * blk + i] = I[t, blocks[r, slot] * blk + i]   (r = b*T + t)
 * and -inf where that token is past L or not visible (> q_offset + t), or the
 * slot is empty. The same values as indexer_score_gathered with these blocks
 * (which fetches every kept block once per query). hisa_block_filter_topk
 * uses this path when blk is a multiple of 128.
 * bf16 or FP8 e4m3 (scores k_scale[s] * sum_h (w * q_scale) ReLU(q8 . k8));
 * d = 128, H in {32, 64}, blk a multiple of 128. Workspace:
 * hisa_refine_workspace_size bytes (the 256-byte header plus the lists). */
DSA_EXPORT size_t hisa_refine_workspace_size(const dsa_indexer_args* a, int m, int blk);
DSA_EXPORT dsa_status hisa_refine_scores(const dsa_indexer_args* a, const int32_t* blocks, int m, int blk,
                                         float* out, long long ld, void* workspace, size_t ws_bytes,
                                         void* stream);

/* ------------------------------------------------------------ DoSA
 * dosa_score_topk ("DoSA: Dots Sparse Attention" review, section 3): the
 * dense selection of indexer_score_topk, computed with certified pruning.
 *   1. every 16th (or 32nd...) visible key is scored with all heads; from that
 *      sample each query gets a threshold thr its k-th score very likely
 *      reaches;
 *   2. screening: per query the n_screen heads with the largest
 *      |w_h| * ||q_h|| are kept exactly; the other positive-weight heads are
 *      bounded through ReLU(x) = (x + |x|) / 2 and Cauchy-Schwarz, the other
 *      negative-weight heads subtract ReLU(k . sum |w_h| q_h); the bound is
 *      evaluated on the tensor cores over n_screen + 3 augmented heads;
 *   3. a 128-key tile stays live for a group of 256 / H queries when some
 *      visible key of it has bound >= thr for some query of the group; the
 *      other tiles are not scored;
 *   4. live tiles are scored with all H heads, scores >= thr are kept per
 *      query; a query with at least min(k, visible) of them has its top-k
 *      among them (its k-th score reaches thr, and every pruned key scores
 *      below thr); other queries have their whole group re-scored;
 *   5. top-k (score descending, index ascending).
 * The selection (and out_score) equals indexer_score_topk's exactly.
 *   out_live NULL or [batch, ceil(T / (256 / H)), ceil(L / 128)] bytes: 1 for
 *            the tiles step 3 kept, 0 for the pruned ones
 * bf16; d in {64, 128}; H in {16, 32, 64}; 0 <= n_screen < H, n_screen <= 13;
 * rows long enough for sampled thresholds (L >= 4096, L a multiple of the
 * sample stride, topk <= L / 8), else DSA_ERR_UNSUPPORTED. Workspace:
 * dosa_workspace_size bytes (0 when unsupported). */
DSA_EXPORT size_t dosa_workspace_size(const dsa_indexer_args* a, int topk, int n_screen);
DSA_EXPORT dsa_status dosa_score_topk(const dsa_indexer_args* a, int topk, int n_screen, int32_t* out_idx,
                                      float* out_score, uint8_t* out_live, void* workspace, size_t ws_bytes,
                                      void* stream);

/* Launch profiling (plumbing; no counterpart on the pages). Between
 * dsa_profile_begin and dsa_profile_end every kernel the library launches, on
 * any stream, is bracketed by two CUDA events recorded on that stream and
 * filed under a name: the stage of the chain ("sample pass", "routed",
 * "re-score", "blocks", "tokens", "router"), a colon, and the kernel's label.
 * dsa_profile_end stops recording, waits for the recorded events, and writes
 * the launches in launch order: NUL-separated names into `names` (capacity
 * names_bytes) and each launch's time in milliseconds into ms; it returns
 * how many it wrote (at most max_entries), or -1 if an event could not be
 * read. Profiling adds two event records per launch; time steps without it. */
DSA_EXPORT dsa_status dsa_profile_begin(void);
DSA_EXPORT int dsa_profile_end(char* names, size_t names_bytes, float* ms, int max_entries);

/* ------------------------------------------------------------ IndexCache
 * indexcache_score_topk ("IndexCache: Accelerating Sparse Attention via
 * Cross-Layer Index Reuse", section 2): n_layers indexer layers, each marked
 * in `pattern` (n_layers characters) as 'F' (full: runs its own dense indexer,
 * as indexer_score_topk, and its top-k becomes the cached index set) or 'S'
 * (shared: skips the indexer and takes the indices of the nearest preceding F
 * layer). pattern[0] must be 'F'.
 *   layers    [n_layers] problems; an S layer's entry only needs batch and T,
 *             equal to its F layer's (q, k, w are not read)
 *   out_idx   [n_layers] pointers to [batch, T, topk] int32; an S layer whose
 *             pointer equals its F layer's shares that buffer (no copy),
 *             otherwise the indices are copied on the stream
 *   out_score NULL, or [n_layers] pointers (entries may be NULL) to fp32
 *             [batch, T, topk]; an S layer's scores are its F layer's
 * Workspace: the largest indexer_workspace_size of the F layers, reused by
 * each F layer in turn. Every argument is validated before the first launch. */
DSA_EXPORT size_t indexcache_workspace_size(const dsa_indexer_args* layers, int n_layers,
                                            const char* pattern, int topk);
DSA_EXPORT dsa_status indexcache_score_topk(const dsa_indexer_args* layers, int n_layers,
                                            const char* pattern, int topk, int32_t* const* out_idx,
                                            float* const* out_score, void* workspace, size_t ws_bytes,
                                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEXER_H */
