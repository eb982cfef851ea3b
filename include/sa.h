/*
 * sa.h -- C ABI of the B200 (sm_100a) causal sparse-attention library
 * (libsa.so).
 *
 * Every query attends to its own set of earlier positions.  The set is chosen
 * by a lightweight indexer's top-k (DeepSeek-style sparse attention, with
 * IndexCache reuse across layers), fixed in advance (a recent window plus
 * dilated distances 1, 2, 4, 8, ...), or built from NSA's compressed,
 * selected and window branches.  Partial results merge by a log-sum-exp
 * softmax combine.
 *
 * Conventions shared by every call
 *  - Tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees memory.  Scratch memory is the caller's
 *    `workspace`, sized by the matching *_workspace_size() query.
 *  - Tensors are dense and row-major in the layouts written beside each
 *    argument (last dimension contiguous).  bf16 is IEEE bfloat16.
 *    Pointers to bf16/fp32 tensors must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous: they enqueue kernels and return.
 *  - Query head h reads KV head h / (Hq / Hkv).  Softmax scale `scale`
 *    multiplies q.k before any bias; pass 1/sqrt(d) for the usual scaling.
 *  - LSE outputs are natural-log log-sum-exp of the scaled (and biased)
 *    logits, fp32; an empty set gives lse = -inf and a zero output row.
 *  - Return value: SA_OK or an sa_status code.  Host-side checks (null or
 *    misaligned pointers, sizes, unsupported shapes, small workspace) fail
 *    before anything is enqueued.  Device-side problems found while running
 *    (an index past the query position or outside [0, L)) skip the offending
 *    entry and raise a bit in the library's device error word, reported by
 *    sa_check_device_status().  Every wait of a kernel on another part of
 *    itself is bounded (about one second, see sa_debug_set_spin_limit); one
 *    that runs out stops the kernel cleanly and is reported as
 *    SA_ERR_TIMEOUT, after which the call's outputs are undefined.
 *  - Supported on this build: head dim d in {64, 128}; any Hq that is a
 *    multiple of Hkv (sa_nsa_fwd: Hq/Hkv <= 16); indexer
 *    heads Hi in {1, 2, 4, 8, 16} with indexer dim di in {32, 64, 128};
 *    sm_100a only.  Anything else returns SA_ERR_UNSUPPORTED; there is no
 *    CPU fallback.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum sa_status {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, inconsistent sizes */
    SA_ERR_UNSUPPORTED = 2,    /* shape or option outside what is built */
    SA_ERR_WORKSPACE = 3,      /* workspace smaller than *_workspace_size() */
    SA_ERR_CUDA = 4,           /* CUDA launch/runtime error (see sa_last_error_string) */
    SA_ERR_DEVICE_ASSERT = 5,  /* device error word was set (bad index found on device) */
    SA_ERR_TIMEOUT = 6         /* a kernel's bounded barrier wait ran out; outputs undefined */
};

/* Fixed index set, generated inside the kernel (no index tensor).
 * SpatialLM page ("SpatialLM-Mini acelero el entrenamiento ...", section "Como
 * eligen los tokens a quien escuchar"): the token itself, its nearest
 * predecessors and the positions at distances 1, 2, 4, 8, ...; never a future
 * position.  For query position p:
 *   S_p = { p - o : 0 <= o < window, p - o >= 0 }
 *       u { p - 2^i : 2^i < p }            (only when dilated != 0)
 * `window` counts the token itself (self + 64 predecessors = 65). */
typedef struct sa_pattern {
    int32_t window;
    int32_t dilated;
} sa_pattern;

/* --------------------------------------------------------------------------
 * Indexer scores and causal top-k.
 * IndexCache page ("IndexCache: inferencia 82% mas rapida ...", body): a
 * lightweight indexer scores every earlier token and the query keeps a small
 * top-scoring subset.  HySparse2 page ("Xiaomi presenta HySparse2 ...",
 * section "Mas precision con menos memoria"): the most recent tokens are
 * forced into the set.  Score of query t (position p = q_pos0 + t) for key j:
 *   I(t, j) = sum_h w[t,h] * max(0, sum_c q_idx[t,h,c] * k_idx[j,c])
 * computed exactly in int32 (the caller keeps |I| < 2^31).
 * Forced window W = {max(0, p-window+1) .. p} (empty when window == 0); the
 * other candidates {0 .. p} \ W are ranked by (I desc, j asc) and the first
 * min(topk, count) are kept.
 *   q_idx  int8  [B, Tq, Hi, di]       k_idx int8 [B, L, di]
 *   w      int32 [B, Tq, Hi]
 *   out_idx   int32 [B, Tq, topk+window]  ascending positions, -1 padded
 *   out_count int32 [B, Tq] (nullable)    number of valid entries
 * Requires 0 <= q_pos0 and q_pos0 + Tq - 1 < L (every query has its key).
 * Selected positions are bit-exact: the selected set is unique under the
 * tie rule and is written in ascending order.
 * ------------------------------------------------------------------------ */
size_t sa_indexer_topk_workspace_size(int B, int Tq, int L, int Hi, int di,
                                      int topk, int window);
int sa_indexer_topk(const int8_t *q_idx, const int8_t *k_idx, const int32_t *w,
                    int B, int Tq, int L, int Hi, int di, int64_t q_pos0,
                    int topk, int window,
                    int32_t *out_idx, int32_t *out_count,
                    void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Gathered-KV sparse attention forward.
 * For each query t (position p = q_pos0 + t) and head h over its index set S:
 *   z_j = scale * (q[t,h] . k[j,g]) + bias(t, j, h),  j in S
 *   out[t,h] = sum_j softmax(z)_j v[j,g],   lse[t,h] = log sum_j exp z_j
 * The set comes from `idx` or, when idx == NULL, from `pattern`.
 *   q   bf16 [B, Tq, Hq, d]          k, v  bf16 [B, L, Hkv, d]
 *   idx int32 [B, Tq, idx_heads, K]  -1 = padding; entries must lie in
 *       [0, min(p, L-1)]; idx_heads is 1 (one list shared by every head) or
 *       Hkv (one list per KV head).  Any order; a repeated entry counts twice.
 *   Optional coordinate bias (SpatialLM page, same section: learnable 3-D
 *   query/key coordinates, a smaller distance giving a larger weight):
 *       bias = -beta[h] * ||cq[t,h,:] - ck[j,g,:]||^2,
 *   cq fp32 [B, Tq, Hq, 3], ck fp32 [B, L, Hkv, 3], beta fp32 [Hq]; all three
 *   NULL for no bias.
 * n_split = 1: out bf16 [B,Tq,Hq,d] and lse fp32 [B,Tq,Hq] (nullable).
 * n_split > 1 (split-KV; idx mode only): the K entries are cut into n_split
 *   contiguous pieces of ceil(K/n_split); piece s writes part_o fp32
 *   [n_split,B,Tq,Hq,d] and part_lse fp32 [n_split,B,Tq,Hq]; when `out` is
 *   non-NULL the pieces are then merged by sa_lse_combine into out/lse.
 *   part_o/part_lse may be NULL, in which case they live in `workspace`.
 * Star Attention page ("NVIDIA AI Research presenta Star Attention ...",
 * body) merges per-block results by a distributed softmax: that is the
 * split-KV mode.
 * ------------------------------------------------------------------------ */
size_t sa_sparse_attn_workspace_size(int B, int Tq, int Hq, int d, int n_split);
int sa_sparse_attn_fwd(const void *q, const void *k, const void *v,
                       int B, int Tq, int L, int Hq, int Hkv, int d, int64_t q_pos0,
                       const int32_t *idx, int idx_heads, int K,
                       const sa_pattern *pattern,
                       const float *cq, const float *ck, const float *beta,
                       float scale, int n_split,
                       void *out, float *lse,
                       float *part_o, float *part_lse,
                       void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * Backward of gathered-KV sparse attention over explicit index lists (no
 * bias).  SpatialLM page (training with the fixed sparse graph) and NSA page
 * ("Puntos Clave": the backward pass of sparse attention).  With p_j =
 * exp(z_j - lse), z_j = scale * q.k_j over the row's list (a repeated entry
 * counts twice, as in the forward):
 *   dP_j = dout . v_j,  D = dout . out,  dS_j = p_j (dP_j - D)
 *   dq = scale * sum_j dS_j k_j,  dk_j += scale * dS_j q,  dv_j += p_j dout
 *   q, out, dout bf16 [B,Tq,Hq,d]; k, v bf16 [B,L,Hkv,d]; lse fp32 [B,Tq,Hq]
 *   (the forward's outputs); idx as in sa_sparse_attn_fwd.
 *   dq fp32 [B,Tq,Hq,d] (written); dk, dv fp32 [B,L,Hkv,d] (zeroed by the
 *   call, then accumulated over every query that selected the key).
 * workspace: sa_sparse_attn_bwd_workspace_size(B, Tq, Hq) bytes.
 * ------------------------------------------------------------------------ */
size_t sa_sparse_attn_bwd_workspace_size(int B, int Tq, int Hq);
int sa_sparse_attn_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                       const void *dout, int B, int Tq, int L, int Hq, int Hkv, int d, int64_t q_pos0,
                       const int32_t *idx, int idx_heads, int K, float scale,
                       float *dq, float *dk, float *dv, void *workspace, size_t workspace_bytes,
                       void *stream);

/* --------------------------------------------------------------------------
 * Split-KV sparse attention that allocates nothing.  No page has a
 * counterpart: this is a convenience entry point of this library.
 * For callers that cannot allocate device memory at call time: a serving
 * runtime whose device memory is all handed out up front, a plugin host that
 * passes only input and output buffers, or a path where an allocation would
 * synchronise the device.  Same operation and
 * layouts as sa_sparse_attn_fwd in idx mode with n_split >= 2 and no bias;
 * the pieces are always merged into out (and lse when non-NULL).
 * The partial results live in an 8 MiB array inside the library image, one
 * per GPU that loads the library, held until the process exits:
 *   round_up(n_split*B*Tq*Hq*d*4, 256) + round_up(n_split*B*Tq*Hq*4, 256)
 * must not exceed 8388608 bytes, else SA_ERR_WORKSPACE is returned before
 * anything is enqueued.  The first call on a device looks up the array's
 * device address with that device current; make that first call before any
 * stream capture.  Every call reuses the same array: calls that may overlap
 * on the GPU (other streams, other host threads) race and must be ordered by
 * the caller.  Nothing needs clearing between calls: on a run that completes,
 * every piece writes all of its partial rows before the merge reads them.
 * After a kernel stops early (sa_check_device_status returns SA_ERR_TIMEOUT)
 * the array may hold an earlier call's partials and out/lse are undefined;
 * check the device status before using them.
 * ------------------------------------------------------------------------ */
int sa_sparse_attn_fwd_split_static(const void *q, const void *k, const void *v,
                                    int B, int Tq, int L, int Hq, int Hkv, int d, int64_t q_pos0,
                                    const int32_t *idx, int idx_heads, int K,
                                    float scale, int n_split,
                                    void *out, float *lse, void *stream);

/* --------------------------------------------------------------------------
 * Log-sum-exp combine (Star Attention page, body: distributed softmax).
 *   lse = log sum_s exp(part_lse[s]),  out = sum_s exp(part_lse[s] - lse) part_o[s]
 * A piece with part_lse = -inf contributes nothing; all empty -> out = 0,
 * lse = -inf.
 *   part_o fp32 [n_split, rows, d], part_lse fp32 [n_split, rows]
 *   out bf16 [rows, d], lse fp32 [rows] (nullable)
 * ------------------------------------------------------------------------ */
int sa_lse_combine(const float *part_o, const float *part_lse, int n_split,
                   int64_t rows, int d, void *out, float *lse, void *stream);

/* --------------------------------------------------------------------------
 * NSA forward (Native Sparse Attention page, "Puntos Clave" and "Analisis
 * Profundo"): coarse compression, fine blockwise selection, sliding window.
 *  1. Kc[i] = mean(k[i*cmp_stride .. i*cmp_stride + cmp_len - 1]) per KV
 *     head (likewise Vc), i = 0 .. (T - cmp_len) / cmp_stride.
 *  2. Compressed branch: query t attends to Kc[i] with i*cmp_stride +
 *     cmp_len - 1 <= t.
 *  3. Importance of selection block b for KV group g: the compressed-branch
 *     probabilities of tokens i with i*cmp_stride in [b*sel_block,
 *     (b+1)*sel_block), summed over those i and over the heads of the group.
 *  4. Per (t, g): the sel_topk blocks with b*sel_block <= t of largest
 *     importance (ties -> lower b; fewer candidates -> all).
 *  5. Selected branch: keys of those blocks, masked to j <= t.
 *  6. Window branch: keys max(0, t-window+1) .. t.
 *  7. out = gates[...,0]*o_cmp + gates[...,1]*o_slc + gates[...,2]*o_win.
 *   q bf16 [B,T,Hq,d], k/v bf16 [B,T,Hkv,d], gates fp32 [B,T,Hq,3]
 *   out bf16 [B,T,Hq,d]; lse_branches fp32 [B,T,Hq,3] (nullable);
 *   sel_idx_out int32 [B,T,Hkv,sel_topk] ascending, -1 padded (nullable).
 * Requires cmp_stride divides sel_block, cmp_len a multiple of cmp_stride,
 * Hq/Hkv <= 16, and sel_topk <= 32.
 * ------------------------------------------------------------------------ */
size_t sa_nsa_workspace_size(int B, int T, int Hq, int Hkv, int d, int cmp_len,
                             int cmp_stride, int sel_block, int sel_topk);
int sa_nsa_fwd(const void *q, const void *k, const void *v, const float *gates,
               int B, int T, int Hq, int Hkv, int d,
               int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
               float scale, void *out, float *lse_branches, int32_t *sel_idx_out,
               void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * NSA forward for training: sa_nsa_fwd, plus the tensors sa_nsa_bwd needs.
 *   o_branches fp32 [3,B,T,Hq,d]: the ungated branch outputs (compressed,
 *   selected, window), caller-owned; lse_branches and sel_idx_out are
 *   required here.  Same workspace as sa_nsa_fwd.
 * ------------------------------------------------------------------------ */
int sa_nsa_fwd_train(const void *q, const void *k, const void *v, const float *gates,
                     int B, int T, int Hq, int Hkv, int d,
                     int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
                     float scale, void *out, float *lse_branches, int32_t *sel_idx_out,
                     float *o_branches, void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * NSA backward (Native Sparse Attention page, "Puntos Clave": natively
 * trainable, with a faster backward pass).  The gradient of sa_nsa_fwd's
 * out for an upstream gradient dout, with the forward's block choice
 * (sel_idx) held fixed: the choice is piecewise constant in the inputs, so
 * no gradient flows through the importance or the top-k.  Per row and
 * head, branch b (gate value g_b, ungated output O_b, saved lse_b):
 *   dgates_b = dout . O_b;  the branch's upstream gradient is g_b dout;
 *   dP_j = g_b dout . v_j,  D = g_b dout . O_b,  dS_j = p_j (dP_j - D),
 *   dq += scale sum_j dS_j k_j,  dk_j += scale dS_j q,  dv_j += p_j g_b dout.
 * The compressed branch's key rows are Kc_i (mean of K[i*stride ..
 * i*stride+len-1]); each of those rows receives dKc_i / len (likewise V).
 *   q, dout bf16 [B,T,Hq,d]; k, v bf16 [B,T,Hkv,d]; gates fp32 [B,T,Hq,3];
 *   o_branches, lse_branches, sel_idx: sa_nsa_fwd_train's outputs.
 *   dq fp32 [B,T,Hq,d]; dk, dv fp32 [B,T,Hkv,d]; dgates fp32 [B,T,Hq,3];
 *   all written (not accumulated).  d = 64 or 128, any Hq/Hkv.
 * Workspace: sa_nsa_bwd_workspace_size bytes, 16-byte aligned.  A selected
 * block past the sequence sets the device error word (SA_ERR_DEVICE_ASSERT
 * from sa_check_device_status).
 * ------------------------------------------------------------------------ */
size_t sa_nsa_bwd_workspace_size(int B, int T, int Hq, int Hkv, int d, int cmp_len,
                                 int cmp_stride, int sel_block, int sel_topk);
int sa_nsa_bwd(const void *q, const void *k, const void *v, const float *gates,
               const void *dout, const float *o_branches, const float *lse_branches,
               const int32_t *sel_idx, int B, int T, int Hq, int Hkv, int d,
               int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
               float scale, float *dq, float *dk, float *dv, float *dgates,
               void *workspace, size_t workspace_bytes, void *stream);

/* --------------------------------------------------------------------------
 * A full-attention layer as an exact indexer (HySparse2 page, "Xiaomi
 * presenta HySparse2 ...", section "Que significa para la evolucion de la
 * IA": a few full-attention layers compute exact scores and guide the
 * selection of the sparse layers).
 *  1. The full layer: causal softmax attention of every head over all keys
 *     j <= t: out, lse.
 *  2. Exact score of key j for query t: the probability the full layer puts
 *     on j, summed over all Hq heads,
 *       score(t, j) = sum_h exp(scale q_{t,h}.k_{j,g(h)} - lse_{t,h}).
 *  3. Index set for the sparse layers (HySparse2 page, "Mas precision con
 *     menos memoria": the most recent tokens are forced in, score-chosen ones
 *     are added): the window {max(0, t-window+1) .. t} plus the top-k of the
 *     other keys by (score desc, j asc); ascending, -1 padded to
 *     topk + window, the layout of sa_indexer_topk (one set per query, shared
 *     by all heads; feed it to sa_sparse_attn_fwd).
 * Scores are fp32 on the device: where two keys' exact scores differ by less
 * than fp32 rounding of the sum, the order between them may differ from the
 * exact one.
 *   q bf16 [B,T,Hq,d], k/v bf16 [B,T,Hkv,d]; out bf16 [B,T,Hq,d] (nullable);
 *   lse fp32 [B,T,Hq] (nullable); out_idx int32 [B,T,topk+window].
 * d = 64 or 128.  Workspace: sa_full_attn_topk_workspace_size bytes (the
 * fp32 output, the LSE and the dense scores of a chunk of query rows,
 * at most 1 GiB), 16-byte aligned.
 * ------------------------------------------------------------------------ */
size_t sa_full_attn_topk_workspace_size(int B, int T, int Hq, int Hkv, int d, int topk,
                                        int window);
int sa_full_attn_topk(const void *q, const void *k, const void *v, int B, int T, int Hq,
                      int Hkv, int d, float scale, int topk, int window, void *out,
                      float *lse, int32_t *out_idx, void *workspace, size_t workspace_bytes,
                      void *stream);

/* --------------------------------------------------------------------------
 * IndexCache layer driver (IndexCache page, body): layers marked 'F' run the
 * indexer and top-k and overwrite the cached index buffer; layers marked 'S'
 * skip the indexer and reuse the buffer of the nearest preceding F layer.
 * pattern[0] must be 'F'.  Every layer then runs sa_sparse_attn_fwd with the
 * cached indices (split-KV with n_split pieces when n_split > 1).  Works for
 * decode (Tq = 1, q_pos0 = L - 1) and prefill alike.
 * ------------------------------------------------------------------------ */
typedef struct sa_dsa_layer {
    const void *q;          /* bf16 [B, Tq, Hq, d] */
    const void *k;          /* bf16 [B, L, Hkv, d] */
    const void *v;          /* bf16 [B, L, Hkv, d] */
    const int8_t *q_idx;    /* int8 [B, Tq, Hi, di]  (read on F layers) */
    const int8_t *k_idx;    /* int8 [B, L, di]       (read on F layers) */
    const int32_t *w;       /* int32 [B, Tq, Hi]     (read on F layers) */
    void *out;              /* bf16 [B, Tq, Hq, d] */
    float *lse;             /* fp32 [B, Tq, Hq] or NULL */
} sa_dsa_layer;

size_t sa_dsa_decode_layers_workspace_size(int B, int Tq, int L, int Hq, int d,
                                           int Hi, int di, int topk, int window,
                                           int n_split);
int sa_dsa_decode_layers(const char *pattern, int n_layers, const sa_dsa_layer *layers,
                         int B, int Tq, int L, int Hq, int Hkv, int d, int Hi, int di,
                         int64_t q_pos0, int topk, int window, float scale, int n_split,
                         int32_t *idx_cache, void *workspace, size_t workspace_bytes,
                         void *stream);

/* --------------------------------------------------------------------------
 * Sequence split across GPUs (Star Attention page, "NVIDIA AI Research
 * presenta Star Attention ...", body: the context is split across hosts and
 * their partial results are merged by a distributed softmax).  With the keys
 * of a sequence split by position over R ranks, decode queries (at the last
 * position) take the exact global selection and attention as follows:
 *   1. every rank: sa_indexer_topk over its own keys with topk + window
 *      candidates and window 0, then sa_indexer_scores_at for their scores;
 *   2. the ranks all-gather the (score, index) candidates;
 *   3. sa_topk_merge: the exact top-k of the gathered candidates by
 *      (score desc, position asc), the forced window appended (the global
 *      top-k of the non-window keys lies in the union of the local
 *      top-(k + window) sets, so this equals the single-GPU selection);
 *   4. every rank: sa_index_shard maps the selection to its rows, then
 *      sa_sparse_attn_fwd over its keys; the partial (out, lse) of the ranks
 *      are all-gathered and merged by sa_lse_combine.
 * sa_indexer_scores_at: out_score[b,t,e] = I(t, idx[b,t,e]) (exact, int32)
 *   for idx >= 0, INT_MIN for -1.  idx [B,Tq,K]; other arguments as in
 *   sa_indexer_topk.
 * sa_topk_merge: candidates [n_parts, rows, kc] (scores and part-local
 *   indices, -1 = none); part p's indices are shifted by part_off[p] (host
 *   array, n_parts <= 64) to positions.  Positions in [q_pos - window + 1, q_pos] are not
 *   ranked; they are appended.  out_idx [rows, topk + window] ascending, -1
 *   padded; out_count [rows] (nullable).  topk <= 4096 and
 *   n_parts * kc <= 24576.
 * sa_index_shard: out[i] = idx[i] - key_lo if key_lo <= idx[i] < key_hi,
 *   else -1 (n entries).
 * ------------------------------------------------------------------------ */
int sa_indexer_scores_at(const int8_t *q_idx, const int8_t *k_idx, const int32_t *w, int B, int Tq, int L, int Hi,
                         int di, const int32_t *idx, int K, int32_t *out_score, void *stream);
int sa_topk_merge(const int32_t *cand_score, const int32_t *cand_idx, const int64_t *part_off, int n_parts,
                  int64_t rows, int kc, int topk, int window, int64_t q_pos, int32_t *out_idx, int32_t *out_count,
                  void *stream);
int sa_index_shard(const int32_t *idx, int64_t n, int64_t key_lo, int64_t key_hi, int32_t *out, void *stream);

/* --------------------------------------------------------------------------
 * Status helpers.
 * sa_check_device_status: waits for `stream`, reads and clears the device
 *   error word of the current device; returns SA_ERR_TIMEOUT if a kernel
 *   since the last check stopped because a bounded wait ran out (outputs of
 *   that call undefined), else SA_ERR_DEVICE_ASSERT if one found a bad index,
 *   else SA_OK (or SA_ERR_CUDA).
 * sa_last_error_string: message of the last failing call on this host thread.
 * sa_status_string: fixed name of a status code.
 * sa_version: library ABI version (major*100 + minor).
 * sa_launch_counter: number of kernels this process has enqueued through the
 *   library so far (all devices, all threads); differences around a region
 *   count the library's launches inside it.
 * ------------------------------------------------------------------------ */
int sa_check_device_status(void *stream);

/* --------------------------------------------------------------------------
 * Debug controls (no page has a counterpart; they exist to test the failure
 * paths).  Each applies to the current device, takes effect for kernels
 * launched after it returns, and must not be called while library kernels
 * run on that device.
 * sa_debug_set_spin_limit: SM clocks a kernel's progress wait may spin
 *   before it gives up (ERR_TIMEOUT -> SA_ERR_TIMEOUT); cycles <= 0 restores
 *   the default (2e9, about one second).  Waits that drain a kernel's own
 *   copies and MMAs before it frees tensor memory keep a fixed long limit.
 * sa_debug_inject_stall: while on != 0, the NSA tensor-core branch kernels
 *   (head dim 128) issue none of their loads, so each CTA's first wait is on
 *   a barrier that nothing completes; it runs out after the spin limit and
 *   sa_nsa_fwd's outputs are undefined.  Nothing is left in flight.
 * sa_debug_exact_recompute_rows: synchronizes the current device and returns
 *   the number of rows whose top-k sa_indexer_topk took by exact recompute
 *   (the sampled-threshold candidate list was short or overflowed) since the
 *   last call, then clears the count; a negative value is -status.
 * ------------------------------------------------------------------------ */
/* --------------------------------------------------------------------------
 * Measurement helper (no page has a counterpart): the ceiling of the L2 ->
 * shared-memory row gather that bounds gathered-KV attention.  Launches
 * ctas_per_sm CTAs per SM of `warps` warps; each warp gathers `iters` stages
 * of 16 rows of 256 bytes, picked by a hash from buf (n_rows x 256 bytes,
 * device memory, 16-byte aligned), into a ring of `stages` shared-memory
 * stages, with no arithmetic on the data.  mode 0: 16-byte cp.async copies
 * (stages 2, 4 or 8); mode 1: one bulk copy (TMA engine) per row, stages
 * 2..16; mode 2: stages of one 16 KB bulk copy of 64 consecutive rows at a
 * random 64-row block (the K or V of one NSA selection block).  Bytes moved =
 * SMs * ctas_per_sm * warps * iters * S with S = 4096 (modes 0, 1) or 16384
 * (mode 2); the caller times the launch on `stream`.  sink: one device word
 * the kernel adds to.
 * ------------------------------------------------------------------------ */
int sa_probe_gather(const void *buf, int64_t n_rows, int mode, int warps, int stages, int iters,
                    int ctas_per_sm, unsigned *sink, void *stream);

int sa_debug_set_spin_limit(long cycles);
int sa_debug_inject_stall(int on);
int64_t sa_debug_exact_recompute_rows(void);
const char *sa_last_error_string(void);
const char *sa_status_string(int status);
int sa_version(void);
uint64_t sa_launch_counter(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
