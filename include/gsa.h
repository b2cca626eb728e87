/*
 * gsa.h — C ABI of libgsa.so: the decode-time hot path of Gist Sparse
 * Attention (GSA) and its gist-causal prefill, for NVIDIA B200 (sm_100a).
 *
 * Method: "Forget, Then Recall: Learnable Compression and Selective Unfolding
 * via Gist Sparse Attention" (Mao, Li, Fox).  Citations below name the page
 * and the section that define each operation:
 *   [EN-2]  gist.science explainer (EN), section 2 "Methodology: Gist Sparse
 *           Attention" (interleaved gist tokens; gist as routing signals;
 *           selective unfolding; hybrid attention; hierarchical extension);
 *   [EN-4]  gist.science explainer (EN), section 4 "Experimental Results"
 *           (KV-cache reuse);
 *   [DE-M]  gist.science explainer (DE), section "Methodik";
 *   [DE-E]  gist.science explainer (DE), section "Ergebnisse";
 *   [SL-n]  Taki-lab slide deck (docswell), page n: 6 "GSA とは", 7 "Gist
 *           token", 9/10 "Training" (stage 1 / stage 2), 11 "H-GSA", 17 "Selective Rules
 *           Comparison", 18 "Top-k vs. Top-p".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, caller-owned DEVICE pointers (16-byte
 *    aligned), except where a declaration says HOST (gsa_decode_step_host's
 *    query and result buffers; gsa_levels_decode's arrays of pointers).  Shapes use B batch, Hq query heads, Hkv KV heads
 *    (G = Hq / Hkv query heads share one KV head: head h reads KV head h / G),
 *    d head_dim, N chunks (= gists), c raw tokens per chunk, k top-k,
 *    W uncompressed tail tokens:
 *        q        [B][Hq][d]
 *        k_gist,  v_gist  [B][Hkv][N][d]        one gist K/V per chunk
 *        k_raw,   v_raw   [B][Hkv][N][c][d]     raw K/V, chunk-major
 *        k_tail,  v_tail  [B][Hkv][W][d]        tokens after the last chunk
 *        scores   [B][Hkv][N]  fp32              routing scores
 *        idx      [B][Hkv][k]  int32             selected chunks, ascending
 *        out      [B][Hq][d]   same dtype as q
 *  - Element type: GSA_F32 or GSA_BF16 for q and every K/V tensor alike;
 *    all accumulation is fp32; the output is rounded once (RNE).
 *  - The library allocates nothing.  Between calls it keeps only small caches
 *    per host thread: launch plans and TMA descriptors, which are pure
 *    functions of the descriptor and the buffer addresses.  So calls from
 *    several host threads need no locking.  Work is enqueued on `stream` (a
 *    cudaStream_t; NULL = legacy default stream) and runs asynchronously; no
 *    entry point synchronises.
 *  - Workspace: entry points that take `ws` need a device buffer of at least
 *    the size the matching gsa_*_workspace_size() returns, 256-byte aligned.
 *    It must be ZERO-FILLED ONCE after allocation (e.g. cudaMemset); each call
 *    that completes leaves its counter words zero again.  One workspace serves
 *    one call at a time: calls that overlap on the GPU must use separate
 *    workspaces.
 *  - Errors: arguments are checked on the host before anything is enqueued;
 *    a failing check returns an error code and enqueues nothing.  A CUDA
 *    launch failure returns GSA_ERR_CUDA.  Nothing is printed, no exception
 *    crosses the ABI.  Device-side anomalies (an out-of-range chunk index
 *    passed to gsa_unfold_attn, a page index or a chunk count out of range
 *    in gsa_decode_step_paged, an expired bounded wait) never fault: the
 *    kernel clamps the value into range (or abandons the wait) and ORs a
 *    flag into an error word.  Entry points that take a workspace use the word at
 *    its start, read back by gsa_workspace_error(); the others
 *    (gsa_score, gsa_gist_prefill, gsa_decode_step_noalloc) use words of
 *    the library, read back and cleared by gsa_device_error().  A call whose
 *    wait expired has left unusable results in its outputs.
 */
#ifndef GSA_H_
#define GSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GSA_OK = 0,
    GSA_ERR_ARG = 1,        /* null pointer, k/W/chunk out of range, empty context, bad mode */
    GSA_ERR_SHAPE = 2,      /* head_dim not 64/128, Hq % Hkv != 0, G not in {1,2,4,8}, size overflow */
    GSA_ERR_DTYPE = 3,      /* dtype not supported by this entry point */
    GSA_ERR_ALIGN = 4,      /* a tensor pointer is not 16-byte aligned */
    GSA_ERR_WORKSPACE = 5,  /* ws is NULL, too small or not 256-byte aligned */
    GSA_ERR_CUDA = 6,       /* a CUDA call or launch failed */
    GSA_ERR_TIMEOUT = 7     /* device-side bounded wait expired (workspace error word) */
} gsa_status;

typedef enum { GSA_F32 = 0, GSA_BF16 = 1 } gsa_dtype;

/* Context rule of the hybrid attention.
 * GSA_ALL_GISTS        every gist once + raw tokens of the k selected chunks
 *                      + tail ([EN-2] "Hybrid Attention"; [SL-17] "AG+SR").
 * GSA_SELECTED_PAIRS   gists and raw tokens of the k selected chunks only +
 *                      tail ([SL-6]; [SL-17] "SG+SR").
 * GSA_SR_ONLY          raw tokens of the k selected chunks + tail, no gist
 *                      ([SL-17] "SR-only").
 * GSA_UNSELECTED_GISTS raw tokens of the k selected chunks + the gists of
 *                      the N - k chunks not selected + tail ([DE-M]
 *                      "Hybride Attention": a selected chunk is represented
 *                      by its raw tokens instead of its gist).
 * In GSA_UNSELECTED_GISTS mode gsa_decode_step enqueues gsa_score, gsa_topk
 * and gsa_unfold_attn (the gist attention needs the selection first); the
 * other modes are one launch on the tensor-core path.                     */
typedef enum {
    GSA_ALL_GISTS = 0,
    GSA_SELECTED_PAIRS = 1,
    GSA_SR_ONLY = 2,
    GSA_UNSELECTED_GISTS = 3
} gsa_mode;

typedef struct {
    int32_t batch, n_q_heads, n_kv_heads, head_dim;
    int32_t n_chunks;   /* N >= 0 */
    int32_t chunk;      /* c >= 1 */
    int32_t top_k;      /* 0 <= k <= N */
    int32_t tail_len;   /* W >= 0 */
    gsa_dtype dtype;
    gsa_mode mode;
    float scale;        /* softmax scale; <= 0 selects 1/sqrt(head_dim) */
} gsa_decode_desc;

/* Two-level gist-of-gist hierarchy ([EN-2] "Hierarchical Extension (H-GSA)";
 * [DE-M] "Erweiterung"; [SL-11]).  l1 describes the level-1 gists, raw chunks
 * and tail (l1.top_k = k1, l1.mode must be GSA_ALL_GISTS); level-2 gist J
 * summarises level-1 gists [J*group, (J+1)*group). n_l2 = ceil(N / group).  */
typedef struct {
    gsa_decode_desc l1;
    int32_t n_l2, group, top_k2;
} gsa_hier_desc;

/* A gist hierarchy of any depth L = levels, 2 <= L <= GSA_MAX_LEVELS ([EN-2]
 * "Hierarchical Extension (H-GSA)": gists compressed again, coarse-to-fine
 * descent; [SL-11]).  l1 describes the level-1 gists (one per chunk), raw
 * chunks and tail as for the two-level hierarchy (l1.top_k = k1, l1.mode
 * GSA_ALL_GISTS).  For i = 0 .. L-2: group[i] level-(i+1) gists make one
 * level-(i+2) gist, so level i+2 has n = ceil(n_{i+1} / group[i]) gists,
 * and top_k[i] is the selection size at level i+2.  Each level's top_k may
 * not exceed the fewest candidates the level above can yield.              */
#define GSA_MAX_LEVELS 8
typedef struct {
    gsa_decode_desc l1;
    int32_t levels;
    int32_t group[GSA_MAX_LEVELS - 1];
    int32_t top_k[GSA_MAX_LEVELS - 1];
} gsa_levels_desc;

/* Gist-causal prefill over P = N*(c+1) interleaved positions (a gist after
 * every chunk of c raw tokens). */
typedef struct {
    int32_t batch, n_q_heads, n_kv_heads, head_dim, n_chunks, chunk;
    gsa_dtype dtype;    /* GSA_BF16 only */
    float scale;        /* <= 0 selects 1/sqrt(head_dim) */
} gsa_prefill_desc;

/* Bytes of workspace gsa_unfold_attn / gsa_decode_step need for `desc`
 * (0 if the descriptor is invalid). */
size_t gsa_decode_workspace_size(const gsa_decode_desc* desc);
/* Bytes of workspace gsa_hier_decode needs (0 if invalid). */
size_t gsa_hier_workspace_size(const gsa_hier_desc* desc);
/* Bytes of workspace gsa_levels_decode needs (0 if invalid). */
size_t gsa_levels_workspace_size(const gsa_levels_desc* desc);

/* Routing scores ([EN-2] "Gist as Routing Signals"; [DE-M]
 * "Relevanz-Scoring"): the decoding query is scored against every gist key
 * by dot product; the G query heads of a KV head share one selection, so
 *     scores[b][hk][j] = sum_{h in group(hk)} q[b][h] . k_gist[b][hk][j]
 * (fp32 accumulation, no softmax scale).  Reads q, k_gist; writes scores.  */
gsa_status gsa_score(const gsa_decode_desc* desc, const void* q, const void* k_gist, float* scores,
                     void* stream);

/* Top-k chunk selection ([EN-2] "Selective Unfolding"; [SL-10] worked
 * example 0.1/0.8/0.7/0.2, k=2 -> g2, g3): per (b, hk) the k indices with the
 * largest scores; equal scores go to the lower index; -0 equals +0; NaN ranks
 * below every number.  Output ascending.  Reads scores [B][Hkv][N]; writes
 * idx [B][Hkv][k].                                                         */
gsa_status gsa_topk(const gsa_decode_desc* desc, const float* scores, int32_t* idx, void* stream);

/* Top-p (nucleus) chunk selection ([SL-18] "Top-k vs. Top-p"; [DE-E]
 * "Ergebnisse": a fixed top-p selection is compared with top-k).  The pages
 * give no formula; the reading taken: per (b, hk) the routing distribution
 * is the softmax of scale * scores (scale as in the descriptor), the chunks
 * are taken in the top-k order (higher score first, the lower index on
 * ties), and the selection is the shortest prefix of that order whose mass
 * reaches top_p, at least one chunk and at most kmax = desc->top_k chunks.
 * Weights and sums are fp32.  Reads scores [B][Hkv][N]; writes idx
 * [B][Hkv][kmax] (the selected chunks ascending, then -1) and count [B][Hkv]
 * (nullable).  0 < top_p <= 1, 1 <= kmax <= 2048; scores must be finite.   */
gsa_status gsa_topp(const gsa_decode_desc* desc, float top_p, const float* scores, int32_t* idx,
                    int32_t* count, void* stream);

/* Selective unfolding + hybrid attention ([EN-2] "Selective Unfolding",
 * "Hybrid Attention"; [DE-M] "Selektive Entfaltung", "Hybride Attention";
 * [SL-17]).  For every query head h of KV head hk the softmax of
 * scale * q_h . K over the context of desc->mode, times V, where the selected
 * chunks are idx[b][hk][0..k) (distinct, in [0, N); -1 marks an empty place
 * of a variable-size selection such as gsa_topp's and adds nothing; any other
 * index out of range is clamped into range and flagged).  lse (nullable)
 * [B][Hq] receives the natural-log sum of exp(scale * q.K) over the context. */
gsa_status gsa_unfold_attn(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                           const void* v_gist, const void* k_raw, const void* v_raw,
                           const void* k_tail, const void* v_tail, const int32_t* idx, void* out,
                           float* lse, void* ws, size_t ws_bytes, void* stream);

/* One full decode step: gsa_score -> gsa_topk -> gsa_unfold_attn in one
 * fused pass (gist keys are read once; in GSA_ALL_GISTS mode the same pass
 * accumulates the attention over all gists).  idx_out and scores_out are
 * nullable: when given they receive the selection and the routing scores.  */
gsa_status gsa_decode_step(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                           const void* v_gist, const void* k_raw, const void* v_raw,
                           const void* k_tail, const void* v_tail, int32_t* idx_out,
                           float* scores_out, void* out, void* ws, size_t ws_bytes, void* stream);

/* gsa_decode_step with the query and the result in HOST memory, for a
 * caller whose decode loop lives on the host: copies q_host [B][Hq][d] into
 * the device buffer q, runs the step, and copies out back to out_host (and
 * the selection idx_out to idx_host, when given), all enqueued on `stream`
 * in this one call; nothing synchronises, so the caller waits on the stream
 * before reading out_host.  Host buffers should be page-locked for the
 * copies to be asynchronous.  Other arguments as for gsa_decode_step (no
 * scores output).                                                           */
gsa_status gsa_decode_step_host(const gsa_decode_desc* desc, const void* q_host, void* q,
                                const void* k_gist, const void* v_gist, const void* k_raw,
                                const void* v_raw, const void* k_tail, const void* v_tail,
                                int32_t* idx_out, int32_t* idx_host, void* out, void* out_host,
                                void* ws, size_t ws_bytes, void* stream);

/* One decode step with top-p selection: gsa_score -> gsa_topp ->
 * gsa_unfold_attn (three launches on the tensor-core path).  desc->top_k is
 * kmax; idx_out [B][Hkv][kmax] receives the selection padded with -1,
 * count_out [B][Hkv] its size, scores_out the routing scores (all three
 * nullable; the workspace holds them otherwise).  Other arguments as for
 * gsa_decode_step.                                                          */
gsa_status gsa_decode_step_topp(const gsa_decode_desc* desc, float top_p, const void* q, const void* k_gist,
                                const void* v_gist, const void* k_raw, const void* v_raw,
                                const void* k_tail, const void* v_tail, int32_t* idx_out,
                                int32_t* count_out, float* scores_out, void* out, void* ws,
                                size_t ws_bytes, void* stream);

/* One decode step over a paged, multi-document raw cache ([EN-4] "KV-Cache
 * Reuse": the caches of documents are computed once and reused, and the
 * gists route the query to the relevant documents without a scan of their
 * raw caches).  The raw K/V live in page pools k_pages / v_pages
 * [n_pages][Hkv][c][d], one page per chunk holding that chunk for every KV
 * head; chunk j of sequence b is page block_table[b][j] (int32 [B][N]), so
 * sequences that hold the same document name the same pages.  seq_chunks
 * (int32 [B], nullable: every sequence has N chunks) gives each sequence's
 * chunk count nb <= N: its gists j >= nb (of k_gist / v_gist [B][Hkv][N][d],
 * which stay dense per sequence) do not exist, score -inf, are never
 * selected and are not in the context, and with nb < k the selection holds
 * all nb chunks and its other places are -1.  Table entries past nb are not
 * read.  A page index outside [0, n_pages) or a chunk count outside [0, N]
 * is clamped into range and flagged in the workspace error word
 * (GSA_WS_ERR_INDEX).  With seq_chunks given, tail_len >= 1 (a sequence
 * with no chunk keeps its tail as context).  Other arguments, the workspace
 * size and the outputs as for gsa_decode_step; n_pages * Hkv * c <= 2^30.  */
gsa_status gsa_decode_step_paged(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                                 const void* v_gist, const void* k_pages, const void* v_pages,
                                 int32_t n_pages, const int32_t* block_table,
                                 const int32_t* seq_chunks, const void* k_tail, const void* v_tail,
                                 int32_t* idx_out, float* scores_out, void* out, void* ws,
                                 size_t ws_bytes, void* stream);

/* Hierarchical decode: level-2 scores over every meta-gist -> top-k2 groups;
 * level-1 scores over the gists of those groups -> top-k1 chunks among them;
 * attention over every meta-gist, every gist of the selected groups, the raw
 * tokens of the k1 chunks and the tail.
 *   k_g2, v_g2 [B][Hkv][n_l2][d]; k_g1, v_g1 [B][Hkv][N][d]; raw and tail as
 *   above; idx2_out [B][Hkv][k2] and idx1_out [B][Hkv][k1] (nullable),
 *   ascending.                                                              */
gsa_status gsa_hier_decode(const gsa_hier_desc* desc, const void* q, const void* k_g2,
                           const void* v_g2, const void* k_g1, const void* v_g1,
                           const void* k_raw, const void* v_raw, const void* k_tail,
                           const void* v_tail, int32_t* idx2_out, int32_t* idx1_out, void* out,
                           void* ws, size_t ws_bytes, void* stream);

/* Hierarchical decode of any depth: every level-L gist is scored and the
 * top k_L taken; at each lower level the candidates are the children of the
 * level above's selection, scored and cut to that level's top-k; the raw
 * tokens of the level-1 selection are unfolded.  Attention over every
 * level-L gist, every candidate of every lower level, the raw tokens of the
 * k1 chunks and the tail (for L = 2: gsa_hier_decode's step).
 *   k_gists, v_gists: HOST arrays of L device pointers, level 1 first, level
 *   l's gists [B][Hkv][n_l][d]; raw and tail as for gsa_decode_step;
 *   idx_out: NULL or a HOST array of L nullable device pointers, level l's
 *   selection [B][Hkv][k_l] (ascending).  One launch of the tensor-core
 *   step (bf16, d = 128, up to four levels, each level's children of the
 *   selection above within 128 rows and, beyond two levels, in groups of a
 *   multiple of 8 dividing 128; k1 c <= 128); otherwise L + 1 launches of the
 *   CUDA-core passes (bf16 or fp32, d = 64 or 128).                        */
gsa_status gsa_levels_decode(const gsa_levels_desc* desc, const void* q, const void* const* k_gists,
                             const void* const* v_gists, const void* k_raw, const void* v_raw,
                             const void* k_tail, const void* v_tail, int32_t* const* idx_out,
                             void* out, void* ws, size_t ws_bytes, void* stream);

/* Stage-2 selective-finetuning forward pass ([EN-2] "Training Procedure":
 * in selective finetuning the attention mask is changed so that attention
 * goes only to the top-k selected chunks and their raw tokens; [SL-10]: the
 * suffix token's attention to the gists gives the scores, top-k picks the
 * chunks to unfold).  Reading taken: every position p of a suffix of
 * S = desc->tail_len tokens selects its own chunks exactly as a decode query
 * does (gsa_score summed over the G heads of a KV head, top-k ascending,
 * ties to the lower index) and attends to the decode context of desc->mode
 * with the suffix tokens 0..p as its tail (causal).
 *   q, out [B][S][Hq][d] (position-major, so a position's heads are
 *   contiguous); k_gist, v_gist, k_raw, v_raw as for gsa_decode_step;
 *   k_suffix, v_suffix [B][Hkv][S][d]; idx_out [B][Hkv][S][k] and
 *   scores_out [B][Hkv][S][N] nullable.  B * S * Hkv <= 65535.  Runs on the
 *   CUDA-core passes: 2 launches (3 in GSA_UNSELECTED_GISTS mode).         */
size_t gsa_suffix_workspace_size(const gsa_decode_desc* desc);
int gsa_suffix_launch_count(const gsa_decode_desc* desc);
gsa_status gsa_suffix_attn(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                           const void* v_gist, const void* k_raw, const void* v_raw,
                           const void* k_suffix, const void* v_suffix, int32_t* idx_out,
                           float* scores_out, void* out, void* ws, size_t ws_bytes, void* stream);

/* Gist-causal prefill ([EN-2] "Interleaved Gist Tokens"; [SL-7] gist causal
 * mask g1 -> x1,x2; g2 -> g1,x3,x4; g3 -> g1,g2,x5,x6,g3; [SL-9]).  Position p
 * is in chunk p / (c+1) and is a gist iff p % (c+1) == c.  Query p attends key
 * t <= p iff t == p, or t is a gist of an earlier chunk, or t is a raw token
 * of p's own chunk.
 *   q, out [B][Hq][P][d]; k, v [B][Hkv][P][d], bf16; lse (nullable)
 *   [B][Hq][P] fp32 natural-log sum of exp over the allowed keys.          */
gsa_status gsa_gist_prefill(const gsa_prefill_desc* desc, const void* q, const void* k,
                            const void* v, void* out, float* lse, void* stream);

/* gsa_decode_step without a caller-provided workspace.  No counterpart in the
 * paper: this is a deployment convenience.  Some callers cannot allocate
 * device memory at the point where they run a decode step — for instance
 * plugin or engine code whose enqueue path is forbidden to allocate, or a
 * server that plans all of its device memory up front and hands out no
 * per-call buffers.  This entry point allocates nothing: it uses a scratch
 * array of 8 MiB that is part of the library's device image (every GPU that
 * loads the library holds it until the process exits).
 *  - Arguments, layouts and results are those of gsa_decode_step.
 *  - Descriptors whose workspace (gsa_decode_workspace_size) exceeds 8 MiB
 *    are rejected with GSA_ERR_WORKSPACE.
 *  - The first call on a device looks up the array's device address for that
 *    device; make that first call before any stream capture on the device.
 *    The address is looked up again if the device's context changed (after a
 *    device reset), so that call too must come before any capture.
 *  - Each call clears the scratch words that must start at zero
 *    (cudaMemsetAsync on `stream`), then runs the decode step in it.  The
 *    array's error word is not cleared by the calls: it collects the flags
 *    of every call until gsa_device_error() reads and clears it.
 *  - All calls share the one array: calls whose work overlaps on the GPU
 *    (different streams, or different host threads) race and corrupt each
 *    other's results.  Serialise them on one stream.
 * It calls no cudaMalloc, cudaFree or other allocating routine.           */
gsa_status gsa_decode_step_noalloc(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                                   const void* v_gist, const void* k_raw, const void* v_raw,
                                   const void* k_tail, const void* v_tail, int32_t* idx_out,
                                   float* scores_out, void* out, void* stream);

/* Number of kernel launches one gsa_decode_step call with this descriptor
 * enqueues (for launch accounting and graph sizing); -1 if the descriptor is
 * invalid.  Host only, enqueues nothing. */
int gsa_decode_launch_count(const gsa_decode_desc* desc);

/* The same for one gsa_hier_decode call: 1 on the tensor-core path, 3 on the
 * CUDA-core passes; -1 if the descriptor is invalid.  Host only. */
int gsa_hier_launch_count(const gsa_hier_desc* desc);
/* The same for one gsa_levels_decode call (L + 1), -1 if invalid. */
int gsa_levels_launch_count(const gsa_levels_desc* desc);

/* Reads (synchronously, on `stream`) the workspace error word: 0, or an OR of
 * GSA_WS_ERR_* flags; returns GSA_ERR_TIMEOUT if a bounded wait expired,
 * GSA_ERR_ARG if an index was out of range, else GSA_OK.  flags_out nullable. */
#define GSA_WS_ERR_TIMEOUT 1u
#define GSA_WS_ERR_INDEX 2u
gsa_status gsa_workspace_error(const void* ws, uint32_t* flags_out, void* stream);

/* Reads (synchronously, on `stream`) and clears the library's own error
 * words on the current device: the one of the entry points without a
 * workspace (gsa_score), the prefill's (gsa_gist_prefill: a work item whose
 * bounded wait expired was abandoned and its rows of out / lse are not
 * valid) and the scratch array's of gsa_decode_step_noalloc.  flags_out
 * (nullable) receives the OR of the GSA_WS_ERR_* flags found; returns
 * GSA_ERR_TIMEOUT if a bounded wait expired, GSA_ERR_ARG if an index was out
 * of range, else GSA_OK.  Calls that overlap it on the GPU may set a flag
 * after it was read; serialise them on `stream` to attribute the flags.   */
gsa_status gsa_device_error(uint32_t* flags_out, void* stream);

/* Diagnostics: sets the time limit (ns) of the waits in which one CTA of a
 * decode launch waits for others (a row's key counter, its ticket), on the
 * current device; 0 restores the default of 2 s.  When a wait runs out the
 * kernel flags GSA_WS_ERR_TIMEOUT and finishes its launch normally.  Meant
 * for tests of that path; synchronous; do not call while a launch runs. */
gsa_status gsa_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code. */
const char* gsa_status_string(gsa_status status);

#ifdef __cplusplus
}
#endif
#endif /* GSA_H_ */
