/*
 * csa.h -- C ABI of the compressed-sparse-attention hot path for NVIDIA B200
 * (sm_100a).
 *
 * The library computes, on the GPU, the attention step of DeepSeek-V4-style
 * hybrid long-context attention:
 *
 *   a1  compressor     pool every m consecutive projected KV rows C into one
 *                      compressed entry with per-channel softmax weights over
 *                      the block's gate logits Z (ratio 1 = unpooled copy);
 *   a2  indexer        score each query against every visible compressed
 *                      indexer key: s_j = sum_h w_h * ReLU(q_h . k_j);
 *   a3  top-k          keep the k best entries per query (score descending,
 *                      lower index first on exact ties);
 *   a4  attention      over the selected entries (CSA) or over every visible
 *                      entry (HCA), K = V = the compressed latent;
 *   a5  window + sink  the same single online softmax continues over the last
 *                      W raw tokens' SWA keys/values, plus one sink logit per
 *                      head that only enters the denominator;
 *   a6  decode step    a1..a5 for one new token of every request.
 *
 * Sources, cited by page title and section:
 *   [ILL]   "DeepSeek-V4.1-Flash, illustrated" (mxino.github.io/illustrations/
 *           deepseek-v41-flash): Equation (1) figure (C_l / Z_l compression
 *           rule; ratio 1 = unpooled main-KV projection; ratio 2 pools
 *           non-overlapping token pairs).
 *   [ATLAS] "Model architectures" atlas (llm-switchboard.icompaas.com/app/
 *           architectures): "compressed KV" entry (CSA = compress every m
 *           tokens with learned weights + lightning-indexer top-k + sliding
 *           window; HCA = stronger compression + dense attention);
 *           "Sliding-window attention" entry (rolling buffer of W tokens);
 *           "MLA" entry (attention runs over the latent directly).
 *   [TOUR]  Tech-report tour (astryx-dracula tech-report.tsx), chapter
 *           "Compressed Sparse Attention 2": "The indexer selects, SWA covers
 *           the rest" (indexer query x indexer key, top 512 per query, then
 *           attention over those entries together with the sliding-window
 *           KV); "A simpler compressor" (no overlap, no absolute position,
 *           indexer K projected from main KV); "Full, Reindex, and Reuse".
 *           Chapter "SWA Bounded Replay", "Replay only the window" (keys in
 *           [max(s, i-W+1), i]).
 *
 * Conventions shared by every entry point
 *   - Every pointer is a DEVICE pointer unless its comment says "host".  The
 *     caller owns every buffer; the library never allocates or frees memory.
 *     Scratch space comes from the caller through (workspace, workspace_bytes);
 *     csa_workspace_size() says how much a call needs.
 *   - Tensors are dense row-major; the last axis is contiguous.  Row starts
 *     of bf16/fp8 tensors must be 16-byte aligned (d and d_idx multiples of
 *     64 for FP8, of 8 for bf16, of 4 for fp32).
 *   - Every call is asynchronous on the given stream (NULL = legacy default
 *     stream).  Host-side validation of shapes, dtypes, alignment and
 *     workspace size runs before any launch; on failure nothing is launched.
 *   - Errors are returned as csa_status_t; csa_last_error() gives a message
 *     (thread-local).  No C++ exception or abort crosses the ABI.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st* csa_stream_t;

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,  /* bad pointer, shape, dtype or alignment         */
  CSA_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. a head/dim combination) */
  CSA_ERR_CAPACITY = 3,     /* workspace too small or cache capacity exceeded  */
  CSA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up              */
  CSA_ERR_CUDA = 5          /* a CUDA runtime call failed                      */
} csa_status_t;

typedef enum csa_dtype {
  CSA_F32 = 0,
  CSA_BF16 = 1,
  CSA_FP8_E4M3 = 2,         /* OCP E4M3 ('fn': no infinities, 448 max), with
                               one fp32 scale per scale_group elements        */
  CSA_MXFP4_E2M1 = 3        /* OCP E2M1 (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and
                               negatives), two per byte -- element 2i in the
                               low nibble of byte i, the sign in bit 3 of a
                               nibble -- with one E4M3 scale byte per 16
                               elements and no further scale: largest value
                               6 * 448 = 2688.  Main-KV rows only.            */
} csa_dtype_t;

/* A tensor in storage format.  value = decode(data[i]) * scale[i / scale_group]
 * for CSA_FP8_E4M3 (scale: fp32) and CSA_MXFP4_E2M1 (scale: uint8 E4M3
 * codes, scale_group 16), scale indexed in the same row-major order, one
 * scale per scale_group consecutive elements of a row; scale is ignored
 * otherwise.  CSA_MXFP4_E2M1 rows take d / 2 bytes of codes.  [TOUR] chapter
 * "Engram, DSpark, FP4", section "FP4 main KV cache" (E2M1 elements, one
 * E4M3 scale per 16 channels, no second-level scale, dequantised before
 * attention; SWA KV stays 8-bit).                                          */
typedef struct csa_tensor {
  void* data;
  void* scale;
  int32_t dtype;        /* csa_dtype_t */
  int32_t scale_group;  /* FP8 / MXFP4: elements per scale; must divide the row */
} csa_tensor_t;

/* Problem shape shared by the calls. */
typedef struct csa_params {
  int32_t m;              /* compression ratio (tokens per compressed entry) >= 1 */
  int32_t d;              /* compressed-entry (= query head) dim                   */
  int32_t d_idx;          /* indexer head dim                                      */
  int32_t h_q;            /* query heads sharing the single KV head                */
  int32_t h_idx;          /* indexer heads                                         */
  int32_t topk;           /* entries kept per query; <= 0: dense over all visible  */
  int32_t window;         /* W: sliding-window length in raw tokens (0 = none)     */
  int32_t swa_cap;        /* slots of the SWA ring; position p lives in p % swa_cap */
  float softmax_scale;    /* tau: logits are tau * q . k                           */
} csa_params_t;

/* Bytes of workspace needed by a call with these shapes (scratch sizing: no
 * counterpart on the pages).
 *   n_queries    query tokens of the call (decode: batch);
 *   max_entries  largest number of visible compressed entries of any query.
 * The result covers csa_index_topk, csa_sparse_swa_attention and
 * csa_decode_step with these arguments.                                      */
size_t csa_workspace_size(const csa_params_t* p, int32_t n_queries, int64_t max_entries);

/* a1 -- compressor.  [ILL] Equation (1); [ATLAS] "compressed KV"; [TOUR]
 * "A simpler compressor".
 * For each request b and complete block j of m consecutive rows:
 *   a_i[c]    = softmax over i in block j of Z[b][i][c]   (per channel c)
 *   out[b][j][c] = sum_i a_i[c] * C[b][i][c]
 * Rows after the last complete block are ignored.  m = 1 copies C.
 *   C, Z      [batch][n_tokens][d], CSA_F32 or CSA_BF16 (same dtype).
 *   out       [batch][out_rows][d] starting at the first new entry; row
 *             stride d, request stride out_rows (>= n_tokens / m).
 *             CSA_F32, CSA_BF16, or CSA_FP8_E4M3 with scale_group 64 (the
 *             scale of a group is max|x| / 448, 1 if the group is zero;
 *             codes round to nearest even, saturating).
 *   w_ik      optional [d][d_idx] (CSA_F32 or CSA_BF16): when non-NULL the
 *             indexer key of every new entry, k = entry . W_IK (taken from the
 *             fp32 pooled entry, before storage rounding), is written to
 *   kidx_out  [batch][out_rows][d_idx]: CSA_F32, CSA_BF16, or CSA_FP8_E4M3
 *             with scale_group = d_idx (one scale per row).
 *   Pointers of out / kidx_out point at the first row to write.            */
csa_status_t csa_compress(const csa_tensor_t* C, const csa_tensor_t* Z, int32_t batch,
                          int64_t n_tokens, int32_t d, int32_t m, const csa_tensor_t* out,
                          int64_t out_rows, const csa_tensor_t* w_ik, int32_t d_idx,
                          const csa_tensor_t* kidx_out, csa_stream_t stream);

/* a2 + a3 -- lightning indexer and per-query top-k.  [ATLAS] "Trained
 * sparse attention" (DSA lightning indexer + top-k), "compressed KV"; [TOUR]
 * "The indexer selects, SWA covers the rest".
 * For query i of request r = q_req[i] with n = n_visible[i] visible entries:
 *   s_j = sum_h w[i][h] * max(0, q_idx[i][h] . k_idx[r][j]),  j < n
 * (for FP8 keys, k_idx[r][j] = codes * row scale).  out_idx[i] receives the
 * min(topk, n) indices with the largest s_j -- larger score first in value,
 * lower index first among exactly equal scores (-0 == +0).  The order of
 * the indices inside out_idx[i] is unspecified (it is a set); unused slots
 * hold -1.
 *   q_idx      [n_queries][h_idx][d_idx], CSA_F32 or CSA_BF16.
 *   w          [n_queries][h_idx] fp32.
 *   k_idx      [batch][cap][d_idx]: CSA_F32, CSA_BF16, or CSA_FP8_E4M3 with
 *              scale_group = d_idx.  cap = rows per request.
 *   q_req      [n_queries] int32 request of each query (NULL: query i uses
 *              request i).  A request outside [0, batch) scores nothing
 *              (its selection is unspecified, never out of bounds).
 *   n_visible  [n_queries] int32; values are clamped to [0, cap].
 *   out_idx    [n_queries][topk] int32.   out_score optional [n_queries][topk]
 *              fp32 (the kernel's fp32 score of each slot, -inf for padding).
 * Requires p->topk >= 1.                                                     */
csa_status_t csa_index_topk(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx,
                            const float* w, const csa_tensor_t* k_idx, int32_t batch, int64_t cap,
                            const int32_t* q_req, const int32_t* n_visible, int32_t* out_idx,
                            float* out_score, void* workspace, size_t workspace_bytes,
                            csa_stream_t stream);

/* a2 alone ([ATLAS] "Trained sparse attention": the lightning indexer) --
 * the indexer scores of csa_index_topk written out:
 * scores[i][j] = s_j for j < min(n_visible[i], cap); columns beyond are not
 * written.  scores [n_queries][ld] fp32, ld >= cap.  Same sources and
 * arguments as csa_index_topk.                                             */
csa_status_t csa_index_score(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx,
                             const float* w, const csa_tensor_t* k_idx, int32_t batch, int64_t cap,
                             const int32_t* q_req, const int32_t* n_visible, float* scores, int64_t ld,
                             csa_stream_t stream);

/* a3 alone ([TOUR] "The indexer selects, SWA covers the rest": the top-k
 * selection) -- top-k of given fp32 score rows, same order rule as above.
 *   scores   [n_rows][ld] fp32; row i has n_valid[i] (<= ld) valid columns.
 *   out_idx  [n_rows][k] int32 (-1 padded), out_score optional.
 *   workspace  optional: with at least csa_topk_workspace_size(n_rows)
 *            bytes, rows of more than 65,536 columns are each split over
 *            several CTAs (same result); without it one CTA takes a row.   */
csa_status_t csa_topk(const float* scores, int32_t n_rows, int64_t ld, const int32_t* n_valid,
                      int32_t k, int32_t* out_idx, float* out_score, void* workspace,
                      size_t workspace_bytes, csa_stream_t stream);

/* Workspace bytes that let csa_topk split long rows over several CTAs
 * (scratch sizing: no counterpart on the pages). */
size_t csa_topk_workspace_size(int32_t n_rows);

/* Hierarchical sparse indexer, first (Full) layer.  [TOUR] chapter
 * "Compressed Sparse Attention 2", section "The Hierarchical Sparse Indexer"
 * (a block's score is the maximum of its positions' scores; the best blocks
 * form a candidate pool, e.g. 2,048 blocks of 8 positions = 16,384
 * candidates at 1M context), section "Full, Reindex, and Reuse" (the Full
 * layer scores everything and builds the pool).
 * Scores s_j as csa_index_topk.  Block b of query i covers entries
 * [b*block, (b+1)*block) and scores max s_j over its visible entries; the
 * last block may be partial.  out_pool[i] receives the min(pool_blocks,
 * ceil(n_visible[i] / block)) best blocks -- larger block score first,
 * lower block id first among exactly equal scores -- as block ids in
 * ASCENDING order, padded with -1.
 *   block        power of two in [1, 128].
 *   out_pool     [n_queries][pool_blocks] int32.
 *   out_idx      optional [n_queries][p->topk] int32 (needs p->topk >= 1):
 *                the layer's own top-k, exactly as csa_index_topk;
 *   out_score    optional, with out_idx, as csa_index_topk.
 *   workspace    csa_index_pool_workspace_size(p, n_queries, cap, block,
 *                pool_blocks) bytes.
 * Other arguments, layouts and errors as csa_index_topk.                    */
csa_status_t csa_index_topk_pool(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx,
                                 const float* w, const csa_tensor_t* k_idx, int32_t batch, int64_t cap,
                                 const int32_t* q_req, const int32_t* n_visible, int32_t block,
                                 int32_t pool_blocks, int32_t* out_pool, int32_t* out_idx,
                                 float* out_score, void* workspace, size_t workspace_bytes,
                                 csa_stream_t stream);

/* Hierarchical sparse indexer, a Reindex layer.  [TOUR] chapter "Compressed
 * Sparse Attention 2", sections "Full, Reindex, and Reuse" (a Reindex layer
 * runs its own indexer query over the candidate pool only) and "The
 * Hierarchical Sparse Indexer" (later indexers search the pool, not the
 * whole context).
 * Pool position j of query i (j < pool_blocks * block) is entry
 * e = pool[i][j / block] * block + j % block; it is a candidate when
 * pool[i][j / block] >= 0 and e < n_visible[i].  The pool must be in the
 * form csa_index_topk_pool writes: block ids ascending, then -1 padding
 * (for other pools the selection is unspecified, though every index written
 * is -1 or a visible entry).  out_idx[i] receives the
 * min(topk, candidates) candidates with the largest s_e (computed as in
 * csa_index_topk, from this call's q_idx and w) as ENTRY ids -- larger
 * score first in value, the earlier pool position first among exactly equal
 * scores, which is the lower entry.  The order inside out_idx[i] is
 * unspecified; unused slots hold -1 (out_score -inf).
 *   pool         [n_queries][pool_blocks] int32 block ids (-1 = empty slot).
 *   out_idx      [n_queries][p->topk] int32; out_score optional fp32.
 *   workspace    csa_index_pool_workspace_size(...) bytes.
 * Requires p->topk >= 1.  Other arguments as csa_index_topk_pool.           */
csa_status_t csa_index_topk_reindex(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx,
                                    const float* w, const csa_tensor_t* k_idx, int32_t batch, int64_t cap,
                                    const int32_t* q_req, const int32_t* n_visible, const int32_t* pool,
                                    int32_t block, int32_t pool_blocks, int32_t* out_idx,
                                    float* out_score, void* workspace, size_t workspace_bytes,
                                    csa_stream_t stream);

/* Workspace bytes (scratch sizing: no counterpart on the pages) that
 * csa_index_topk_pool and csa_index_topk_reindex need
 * for n_queries queries with at most max_entries visible entries (0 for
 * invalid arguments).                                                       */
size_t csa_index_pool_workspace_size(const csa_params_t* p, int32_t n_queries, int64_t max_entries,
                                     int32_t block, int32_t pool_blocks);

/* a4 + a5 -- sparse (CSA) or dense (HCA) attention over compressed entries,
 * the sliding window and the sink, in one online softmax.  [ATLAS]
 * "compressed KV", "Sliding-window attention", "MLA"; [TOUR] "The indexer
 * selects, SWA covers the rest", "Replay only the window".
 * For query i of request r at absolute position t = q_pos[i], head h:
 *   E = { idx[i][0..topk) } minus -1 entries   (idx != NULL, CSA)
 *     = { 0 .. n_visible[i]-1 }                (idx == NULL, HCA)
 *   P = [max(lo, t - W + 1, 0), t], lo = swa_lo ? swa_lo[i] : 0; position p
 *       reads slot p % swa_cap of swa_k[r] / swa_v[r]
 *   l_e = tau q_h . kv[r][e],  l_p = tau q_h . swa_k[r][p % swa_cap]
 *   M = max(sink_h, l),  L = exp(sink_h - M) + sum_E exp(l_e - M) + sum_P exp(l_p - M)
 *   out[i][h] = (sum_E exp(l_e - M) kv[r][e] + sum_P exp(l_p - M) swa_v[r][p]) / L
 *   lse[i][h] = M + log L
 * (sink_h = -inf when sink == NULL; an empty softmax gives out = 0,
 * lse = -inf.)  E and P are not de-duplicated.
 *   q         [n_queries][h_q][d], CSA_F32 or CSA_BF16.
 *   kv        [batch][cap][d], CSA_F32, CSA_BF16, or CSA_FP8_E4M3 with
 *             scale_group 64.
 *   idx       [n_queries][p->topk] int32 or NULL; entries outside
 *             [0, n_visible) are skipped.  n_visible [n_queries] int32,
 *             clamped to [0, cap].  q_req as in csa_index_topk (a request
 *             outside [0, batch) attends to nothing).
 *   swa_k/v   [batch][swa_cap][d], CSA_F32 or CSA_BF16 (may alias).
 *   q_pos     [n_queries] int64.   swa_lo optional [n_queries] int64.
 *   sink      optional [h_q] fp32.
 *   out       [n_queries][h_q][d], CSA_F32 or CSA_BF16.  lse optional fp32.
 * Window positions must be resident: t - swa_cap < first window position.  */
csa_status_t csa_sparse_swa_attention(const csa_params_t* p, int32_t n_queries,
                                      const csa_tensor_t* q, const csa_tensor_t* kv, int32_t batch,
                                      int64_t cap,
                                      const int32_t* idx, const int32_t* n_visible,
                                      const int32_t* q_req, const csa_tensor_t* swa_k,
                                      const csa_tensor_t* swa_v, const int64_t* q_pos,
                                      const int64_t* swa_lo, const float* sink,
                                      const csa_tensor_t* out, float* lse, void* workspace,
                                      size_t workspace_bytes, csa_stream_t stream);

/* a4 + a5 without a caller workspace -- the pages have no counterpart; this
 * entry point exists for callers that cannot allocate device memory: a
 * plugin whose host application owns every byte of device memory, or a
 * serving loop that cannot afford cudaMalloc's implicit device-wide
 * synchronisation.  Same arguments, semantics and results as
 * csa_sparse_swa_attention, minus (workspace, workspace_bytes).  Its scratch
 * is a fixed 16 MiB device array inside the library, held by every GPU that
 * loads the library until the process exits; problems that need more
 * return CSA_ERR_CAPACITY with a message (use csa_sparse_swa_attention
 * then).  The first call made with a given device current looks up the
 * array's device address (cudaGetSymbolAddress); make that first call before
 * any stream capture.  All calls share the one array: calls that overlap on
 * the GPU (concurrent streams) race, so serialise them.  The call itself
 * allocates nothing.                                                        */
csa_status_t csa_sparse_swa_attention_noalloc(const csa_params_t* p, int32_t n_queries,
                                              const csa_tensor_t* q, const csa_tensor_t* kv,
                                              int32_t batch, int64_t cap, const int32_t* idx,
                                              const int32_t* n_visible, const int32_t* q_req,
                                              const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                              const int64_t* q_pos, const int64_t* swa_lo,
                                              const float* sink, const csa_tensor_t* out, float* lse,
                                              csa_stream_t stream);

/* Caches of a decode step (all per request, updated in place). */
typedef struct csa_decode_caches {
  csa_tensor_t kv;       /* [batch][cap][d] compressed entries                */
  csa_tensor_t kidx;     /* [batch][cap][d_idx] indexer keys                  */
  csa_tensor_t swa_k;    /* [batch][swa_cap][d] ring                          */
  csa_tensor_t swa_v;    /* [batch][swa_cap][d] ring                          */
  csa_tensor_t open_c;   /* [batch][m][d] rows of the open block, slot t % m  */
  csa_tensor_t open_z;   /* [batch][m][d]                                     */
  int64_t cap;           /* rows per request of kv / kidx                     */
} csa_decode_caches_t;

/* The new token of every request. */
typedef struct csa_decode_token {
  csa_tensor_t c;        /* [batch][d] projected KV row of the token          */
  csa_tensor_t z;        /* [batch][d] its compression gate logits            */
  csa_tensor_t k_swa;    /* [batch][d] its sliding-window key                 */
  csa_tensor_t v_swa;    /* [batch][d] its sliding-window value               */
  csa_tensor_t q;        /* [batch][h_q][d] main query                        */
  csa_tensor_t q_idx;    /* [batch][h_idx][d_idx] indexer query               */
  const float* w;        /* [batch][h_idx] indexer head weights               */
  const float* sink;     /* optional [h_q] sink logits                        */
  csa_tensor_t w_ik;     /* [d][d_idx] indexer-key projection                 */
} csa_decode_token_t;

/* a6 -- one decode step for every request.  [TOUR] "Full, Reindex, and
 * Reuse" (Full mode), "The indexer selects, SWA covers the rest".
 * For request b with its new token at absolute position t = pos[b]:
 *   1. k_swa / v_swa enter ring slot t % swa_cap; c / z enter open slot t % m.
 *   2. if (t + 1) % m == 0 the open block is pooled as in csa_compress into
 *      kv row (t+1)/m - 1 and its indexer key (entry . w_ik) into kidx.
 *   3. n = (t + 1) / m visible entries; unless p->topk <= 0 (dense / HCA),
 *      index + top-k as csa_index_topk.
 *   4. attention as csa_sparse_swa_attention with q_pos = t.
 * pos is read, never written: the caller advances it.  The step is
 * stream-ordered and writes only the caches' slots named above.
 *   out       [batch][h_q][d], CSA_F32 or CSA_BF16; lse optional [batch][h_q].
 *   out_idx   optional [batch][p->topk] int32 (sparse steps only): the
 *             selection of step 3, exactly as csa_index_topk writes it
 *             (a set, -1 padded); NULL keeps it inside the workspace.
 * Errors: CSA_ERR_INVALID_ARG for bad shapes, dtypes or alignment, or when
 * the keys of one query (topk, or cap when dense, plus window) exceed
 * 2^31 - 1; CSA_ERR_CAPACITY for a workspace below csa_workspace_size.     */
csa_status_t csa_decode_step(const csa_params_t* p, int32_t batch, const csa_decode_caches_t* caches,
                             const csa_decode_token_t* tok, const int64_t* pos,
                             const csa_tensor_t* out, float* lse, int32_t* out_idx,
                             void* workspace, size_t workspace_bytes, csa_stream_t stream);

/* Per-kernel timing (measurement support; not on the compute path, no
 * counterpart on the pages).
 * csa_profile_start(n) creates 2n CUDA events and from then on records one
 * event on the launch stream right before and right after each of the
 * library's kernel launches, for the first n launches; csa_profile_stop()
 * ends recording.  csa_profile_get(i) waits for record i to complete and
 * returns the kernel's name (static storage) and the milliseconds between
 * its two events.  Host-side state is process-wide and mutex-protected.   */
csa_status_t csa_profile_start(int32_t max_launches);
csa_status_t csa_profile_stop(void);
int32_t csa_profile_count(void);
csa_status_t csa_profile_get(int32_t i, const char** kernel_name, float* ms);

/* Message of the last failed call on this thread ("" if none; error
 * reporting, no counterpart on the pages). */
const char* csa_last_error(void);

/* (Error reporting, no counterpart on the pages.)  Synchronises `stream` and
 * reports device-side errors latched by earlier
 * calls (e.g. CSA_ERR_TIMEOUT from a bounded wait), clearing them.        */
csa_status_t csa_sync_status(csa_stream_t stream);

/* Test support for the bounded device-side waits (no counterpart on the
 * pages; never needed in normal use).  The next launch of the fused
 * tensor-core indexer (csa_index_topk, csa_index_topk_pool,
 * csa_index_topk_reindex or csa_decode_step on its tensor-core path) takes
 * this request: its CTA number `cta` does not arrive at the first
 * per-request grid barrier, and every grid-barrier wait of that launch gives
 * up after `polls` polls (about 64 ns apart; normally 2^22).  The CTAs of
 * that request then stop waiting, latch CSA_ERR_TIMEOUT for
 * csa_sync_status, leave their selection unwritten and exit; nothing faults
 * and the context stays usable.  Launches after that one run normally.
 * cta < 0 withdraws a pending request.  Process-wide, mutex-protected.     */
csa_status_t csa_test_expire_next_barrier(int32_t cta, uint32_t polls);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
