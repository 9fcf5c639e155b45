/*
 * lsa.h -- C ABI of liblsa.so: the LongCat Sparse Attention (LSA) layer hot path on one
 * NVIDIA B200 (sm_100a).
 *
 * Method: "LongCat Sparse Attention: Taming the Lightning via Streaming-aware Hierarchical
 * Cross-Layer Indexing" (arXiv 2608.01662).  The layer is
 *   (1) the Lightning Indexer score  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])  (Sec. 2.2, Eq. 1),
 *   (2) Streaming-aware Indexing: a fixed sink + sliding window, and an arg-top-K over the middle
 *       region only (Sec. 3.1),
 *   (3) Hierarchical Indexing: page scores from sub-block-mean keys, top-M pages, then token
 *       scores inside the recalled pages (Sec. 3.3, Eq. 9-11),
 *   (4) Hybrid Sparse Attention: attention over the contiguous sink + window rows and the
 *       gathered dynamic rows of the MLA latent cache, merged by log-sum-exp (Sec. 4.1.1),
 *   and Cross-Layer Indexing (Sec. 3.2): a reuse layer calls lsa_attend with its owner layer's
 *   index buffer and never calls lsa_index.
 *
 * Conventions for every entry point
 *  - Positions are 0-based.  A query at position t sees keys 0..t.  Its regions are
 *      sink = [0, min(sink, t+1)),  swa = [max(sink, t-swa+1), t],  dyn = [sink, t-swa]
 *    (disjoint; with sink = swa = 0 the whole prefix is dynamic, i.e. plain DSA).
 *  - bf16 tensors are passed as device pointers to densely packed row-major arrays.
 *  - Alignment: the kernels read and write bf16 rows with 16-byte vector accesses, cp.async and
 *    TMA, so every bf16 row tensor (q_I, k_I, k_mean, q, c_kv, out, and the new rows of
 *    lsa_kv_append) and every workspace must start on a 16-byte boundary; int32 and fp32 arrays
 *    on a 4-byte one, w_I on a 2-byte one.  A pointer that breaks this returns
 *    LSA_ERR_INVALID_ARG before anything is enqueued.
 *  - Ownership: the caller owns every buffer.  The library allocates no device memory and keeps
 *    no state between calls.  Scratch memory is the caller's workspace `ws` (size from the
 *    matching *_workspace_bytes query; 256-byte aligned base).
 *  - Streams: every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns; nothing synchronises except lsa_get_error.
 *  - Errors: shapes, pointers and sizes are checked on the host before anything is enqueued;
 *    a bad argument returns LSA_ERR_INVALID_ARG (or LSA_ERR_UNSUPPORTED for a legal but
 *    unimplemented shape, LSA_ERR_WORKSPACE for a short workspace).  A failed launch returns
 *    LSA_ERR_CUDA.  Conditions only the device can see (a query position outside its sequence,
 *    a non-finite score, an index outside the query's dynamic region or out of order) set bits
 *    of a device error word kept in the workspace; lsa_get_error reads it.  No entry point
 *    traps, asserts or throws across this boundary.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,
    LSA_ERR_UNSUPPORTED = 2,
    LSA_ERR_WORKSPACE = 3,
    LSA_ERR_CUDA = 4,
    LSA_ERR_DEVICE = 5
} lsa_status;

/* Bits of the device error word (lsa_get_error). */
#define LSA_DEVERR_QPOS      0x1  /* q_pos[b,t] < 0, q_pos >= kv_len[b], or kv_len[b] > L_max   */
#define LSA_DEVERR_NONFINITE 0x2  /* a score or an attention logit was NaN or infinite          */
#define LSA_DEVERR_INDEX     0x4  /* lsa_attend: an index outside dyn, repeated, or out of order */
#define LSA_DEVERR_APPEND    0x8  /* lsa_kv_append: kv_len_old[b] + n_new > L_max                */
#define LSA_DEVERR_INTERNAL  0x10 /* an internal capacity check failed (a bug; result invalid)  */
#define LSA_DEVERR_TIMEOUT   0x20 /* a pipeline wait inside a kernel gave up (result invalid)     */

/* Human-readable name of a status code (static string, never NULL). */
const char *lsa_status_string(lsa_status s);

/* Library version as major*10000 + minor*100 + patch. */
int lsa_version(void);

/*
 * lsa_launch_count -- number of GPU kernels this library has launched since it was loaded, over
 * all devices, streams and threads (counted on the host when each launch is issued; a launch
 * captured into a CUDA graph is counted once, at capture, not at each replay).  Memory sets and
 * copies issued by the library are not kernels and are not counted.  No counterpart in the
 * paper: it lets a caller state how many kernels one call of the path costs.
 */
uint64_t lsa_launch_count(void);

/*
 * lsa_index_workspace_bytes -- bytes of workspace lsa_index needs for these sizes (0 if the
 * sizes are invalid).  Arguments as for lsa_index.
 */
size_t lsa_index_workspace_bytes(int B, int T, int H_I, int D_I, int64_t L_max, int K_sparse,
                                 int page, int sub_block, int M);

/*
 * lsa_index -- Lightning Indexer + Streaming-aware Indexing + (optionally) Hierarchical
 * Indexing for B sequences with T queries each.
 *   Paper: Sec. 2.2 Eq. 1 (score), Eq. 2 (arg topK), Sec. 3.1 (S_sparse over the middle region,
 *   K_sparse = K - K_sink - K_swa), Sec. 3.3 Eq. 9-11 (HI), Sec. 4.1.2 (HI operator).
 *
 *   q_I      bf16 [B, T, H_I, D_I]   indexer queries
 *   w_I      bf16 [B, T, H_I]        indexer head weights (any sign)
 *   k_I      bf16 [B, L_max, D_I]    indexer key cache (one key per token, shared by all heads)
 *   k_mean   bf16 [B, ceil(L_max/sub_block), D_I]  sub-block-mean keys as written by
 *            lsa_kv_append; read only when M > 0 (may be NULL when M == 0)
 *   kv_len   int32 [B] device        tokens present in each sequence (<= L_max)
 *   q_pos    int32 [B, T] device     position t of each query (0 <= t < kv_len[b])
 *   H_I      1..128, multiple of 8;  D_I in {64, 128}
 *   K_sparse 1..4096                 dynamic budget (e.g. 2048 - 16 - 1024 = 1008)
 *   sink, swa >= 0                   fixed budgets (16 and 1024 in the paper; 0/0 = DSA)
 *   page, sub_block                  HI page size P and sub-block size B (P % B == 0,
 *                                    P in {32,64,128,256}); ignored when M == 0
 *   M        0 = flat indexer over dyn; > 0 = HI with M recalled pages (1..4096)
 *   indices  int32 [B, T, K_sparse] out: selected dynamic positions, ranked by
 *            (score desc, position asc), written sorted ascending, -1 in unused slots
 *            (a query whose dyn region holds fewer than K_sparse tokens).
 *   scores_dbg      float [B, T, L_max] or NULL: the fp32 score of every scored token at its
 *                   position (flat: all of dyn; HI: recalled pages within dyn); other entries
 *                   are left unspecified.
 *   page_scores_dbg float [B, T, ceil(L_max/page)] or NULL (HI only): fp32 page score of every
 *                   page that intersects dyn, at its page id.
 *   ws, ws_bytes    workspace of at least lsa_index_workspace_bytes(...) bytes.
 *   stream          cudaStream_t.
 * The caller applies the paper's HI gates (length >= 256K, shallow layers off) by passing M.
 */
lsa_status lsa_index(const void *q_I, const void *w_I, const void *k_I, const void *k_mean,
                     const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H_I, int D_I,
                     int64_t L_max, int K_sparse, int sink, int swa, int page, int sub_block,
                     int M, int32_t *indices, float *scores_dbg, float *page_scores_dbg,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * lsa_attend_workspace_bytes -- bytes of workspace lsa_attend needs (0 if invalid sizes).
 */
size_t lsa_attend_workspace_bytes(int B, int T, int H, int D_v, int K_sparse, int sink, int swa);

/*
 * lsa_attend -- Hybrid Sparse Attention (HFA) forward over absorbed-MLA latent rows.
 *   Paper: Sec. 2.2 (u_t = Attn(h_t, {c_s : s in S_t})), Sec. 3.1 (S_t = S_sink U S_swa U
 *   S_sparse; sink and window tokens still take part in the normalisation, Fig. 1),
 *   Sec. 4.1.1 (contiguous and gathered branches merged by online-softmax rescaling),
 *   Sec. 3.2 (a Cross-Layer-Indexing reuse layer passes its owner's `indices` unchanged).
 *   For each head h of each query t:
 *     z_s = scale * q[h] . c[s]  (all D_qk dims)   for s in S_t,
 *     lse[h] = ln sum_s exp(z_s),   out[h] = sum_s exp(z_s - lse[h]) * c[s][0:D_v].
 *
 *   q        bf16 [B, T, H, D_qk]   absorbed MLA queries
 *   c_kv     bf16 [B, L_max, D_qk]  latent cache rows (D_qk = 576 = 512 + 64, 1152 B per row)
 *   indices  int32 [B, T, K_sparse] dynamic positions (ascending, -1 padded), e.g. from
 *            lsa_index of this layer or of the CLI owner layer; never modified.
 *   kv_len, q_pos as for lsa_index.
 *   H        1..128, multiple of 8;  D_qk == 576, D_v == 512
 *   scale    softmax scale, positive and finite (e.g. 1/sqrt(576)); otherwise
 *            LSA_ERR_INVALID_ARG
 *   out      bf16 [B, T, H, D_v] out;  lse  float [B, T, H] out (natural log).
 * A query whose S_t is empty cannot occur (t itself is always in sink or window when
 * sink + swa > 0, and in dyn otherwise).
 */
lsa_status lsa_attend(const void *q, const void *c_kv, const int32_t *indices,
                      const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H, int D_qk,
                      int D_v, int64_t L_max, int K_sparse, int sink, int swa, float scale,
                      void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * lsa_attend_bwd -- backward of lsa_attend: gradients of sum(out * dout) with respect to q and
 * the latent rows (the paper's training path).
 *   Paper: Sec. 4.1.1 (HFA backward: dQ through the gathered rows, scatter-add of the row
 *   gradients, whose set the window halves), Table 2 (training setting), over the S_t of
 *   Sec. 3.1.  With z_s = scale q.c_s, p_s = exp(z_s - lse), dp_s = dout . c_s[0:D_v],
 *   D = sum_s p_s dp_s, dz_s = p_s (dp_s - D):
 *     dq = scale sum_s dz_s c_s;   dc_s += scale dz_s q + p_s dout (first D_v dims).
 *   The products run on bf16 operands with fp32 accumulation: p_s and scale dz_s are rounded
 *   to bf16 before the dq and dc_kv products (relative error 2^-8 per term).
 *   out, lse  the forward's outputs for the same inputs (as lsa_attend writes them: bf16
 *          [B, T, H, 512], 16-byte aligned, and fp32 [B, T, H], natural log), or both NULL.
 *          Given, lse is used as is and D = sum_d dout_d out_d (fp32 over the bf16 output), the
 *          usual training path, which skips a pass over the keys; NULL, both are recomputed in
 *          fp32 from the inputs in a first pass (exact up to fp32 rounding).  D from the bf16
 *          output carries its rounding: where dq nearly cancels (attention flat over identical
 *          rows) the relative error of dq grows accordingly, while the recomputed D keeps it at
 *          the bf16-operand level.
 *   q, c_kv, indices, kv_len, q_pos, sizes, sink, swa, scale: as lsa_attend (indices as lsa_index
 *   writes them); H a multiple of 32.
 *   dout   bf16 [B, T, H, 512]    gradient of the output (16-byte aligned)
 *   dq     fp32 [B, T, H, 576]    out: written (8-byte aligned); a query flagged
 *          LSA_DEVERR_QPOS gets a zero dq
 *   dc_kv  fp32 [B, L_max, 576]   in/out (16-byte aligned): every row of every S_t gets its
 *          gradient added (atomically; rows selected by several queries or head groups
 *          accumulate).  The caller zeroes it first.  Summation order is not fixed, so results
 *          vary in the last bits.
 *   device_error  int32 device word or NULL: LSA_DEVERR_QPOS / INDEX / NONFINITE bits, and
 *          LSA_DEVERR_TIMEOUT if a pipeline wait inside the kernel gave up (the results are then
 *          invalid).
 *   Kernels: with out / lse given and H a multiple of 64, one CTA per (query, 64 heads) on
 *   the tcgen05 tensor cores (LSA_NO_TCGEN05=1 selects the warp-level MMA kernel instead);
 *   otherwise the warp-level MMA kernel, one CTA per (query, 32 heads).  Same roundings.
 *   Asynchronous on `stream`; host-side errors as lsa_attend.
 */
lsa_status lsa_attend_bwd(const void *q, const void *c_kv, const int32_t *indices,
                          const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H,
                          int D_qk, int D_v, int64_t L_max, int K_sparse, int sink, int swa,
                          float scale, const void *out, const float *lse, const void *dout,
                          float *dq, float *dc_kv, int32_t *device_error, void *stream);

/*
 * lsa_kv_append -- append n_new tokens per sequence to the indexer key cache and/or the
 * latent cache, and refresh the sub-block-mean cache that Hierarchical Indexing reads.
 *   Paper: Sec. 3.3 (Hierarchical Indexing reads the sub-block means from a per-sequence
 *   cache; Sec. 3.3 and Table 4 count its upkeep among the overheads).
 *   Token i of sequence b goes to position kv_len_old[b] + i.  Every sub-block touched by the
 *   append is recomputed from the key cache: k_mean[b][n] = bf16(fp32 mean of the present
 *   tokens of [n*sub_block, (n+1)*sub_block)), so a partial last block holds the mean of the
 *   tokens present so far.
 *
 *   k_I_new  bf16 [B, n_new, D_I] or NULL (skip the indexer part)
 *   k_I      bf16 [B, L_max, D_I] (required when k_I_new != NULL)
 *   k_mean   bf16 [B, ceil(L_max/sub_block), D_I] or NULL (no mean upkeep)
 *   c_new    bf16 [B, n_new, D_qk] or NULL (skip the latent part)
 *   c_kv     bf16 [B, L_max, D_qk] (required when c_new != NULL)
 *   kv_len_old int32 [B] device: lengths before the append (not modified; the caller keeps
 *            its own lengths)
 *   device_error int32 device word or NULL: LSA_DEVERR_APPEND is OR-ed in for a sequence that
 *            would overflow L_max (that sequence is then left untouched).
 */
lsa_status lsa_kv_append(const void *k_I_new, void *k_I, void *k_mean, const void *c_new,
                         void *c_kv, const int32_t *kv_len_old, int B, int n_new, int D_I,
                         int D_qk, int64_t L_max, int sub_block, int32_t *device_error,
                         void *stream);

/*
 * lsa_kv_minmax -- refresh the MinMax pooling rows that lsa_index_minmax reads, for the
 * sub-blocks touched by tokens [kv_len_old[b], kv_len_old[b] + n_new) of each sequence.
 *   Paper: Sec. 5.3.5, pooling ablation (Table 11): instead of the mean key, a sub-block keeps
 *   the element-wise maximum and minimum of its keys.  Row n of a sequence holds
 *   (k_max[n, 0..D_I), k_min[n, 0..D_I)) over the tokens of [n*sub_block, (n+1)*sub_block)
 *   present so far; both are exact bf16 values of the cache.
 *   Call it after lsa_kv_append has written those tokens' keys into k_I.
 *   k_I       bf16 [B, L_max, D_I]                       key cache (read)
 *   k_minmax  bf16 [B, ceil(L_max/sub_block), 2 * D_I]   MinMax rows (touched rows rewritten)
 *   kv_len_old int32 [B] device: lengths before the append; D_I in {64, 128}; sub_block 1..4096
 *   device_error int32 device word or NULL: LSA_DEVERR_APPEND for a sequence whose range
 *            passes L_max (its rows are then left untouched).
 *   Asynchronous on `stream`; pointers 16-byte aligned; host errors as lsa_kv_append.
 */
lsa_status lsa_kv_minmax(const void *k_I, void *k_minmax, const int32_t *kv_len_old, int B,
                         int n_new, int D_I, int64_t L_max, int sub_block, int32_t *device_error,
                         void *stream);

/*
 * lsa_index_minmax -- lsa_index with Hierarchical Indexing whose stage 1 uses MinMax pooling.
 *   Paper: Sec. 3.3 Eq. 9-11 (HI), with the sub-block term of the Sec. 5.3.5 pooling ablation:
 *     s~[t,n,j] = sum_d max(q[t,j,d] * k_max[n,d], q[t,j,d] * k_min[n,d])
 *   in place of q[t,j] . k_mean[n] inside Eq. 9 (this library's reading; the paper prints only
 *   the term):  I_page[t,p] = sum_j w[t,j] * sum_{n in page p} ReLU(s~[t,n,j]).  Computed as one
 *   contraction of depth 2 D_I: (max(q,0) | min(q,0)) . (k_max | k_min).  Stage 2, selection,
 *   outputs and errors are those of lsa_index.  The paper finds mean pooling better (Table 11);
 *   this entry point exists for that comparison.
 *   k_minmax  bf16 [B, ceil(L_max/sub_block), 2 * D_I] as lsa_kv_minmax writes it.
 *   Other arguments as lsa_index; M >= 1 (otherwise LSA_ERR_INVALID_ARG).  The MinMax page score
 *   runs on the tensor cores only: H_I in {64, 128}, D_I in {64, 128}, B*T <= 65535, and
 *   LSA_ERR_UNSUPPORTED otherwise (or when LSA_NO_TCGEN05=1 disables those kernels).
 *   Workspace: lsa_index_workspace_bytes with the same sizes.
 */
lsa_status lsa_index_minmax(const void *q_I, const void *w_I, const void *k_I,
                            const void *k_minmax, const int32_t *kv_len, const int32_t *q_pos,
                            int B, int T, int H_I, int D_I, int64_t L_max, int K_sparse, int sink,
                            int swa, int page, int sub_block, int M, int32_t *indices,
                            float *scores_dbg, float *page_scores_dbg, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * lsa_index_noalloc -- lsa_index for callers that cannot allocate device memory.  (The paper has
 * no counterpart: this is a deployment convenience of this library.)
 *   Some callers cannot provide a workspace: a plug-in inside a host application whose memory
 *   pool owns the whole GPU and is not shared with the plug-in, or a serving loop that forbids
 *   cudaMalloc on its hot path because an allocation can synchronise the device and take
 *   unbounded time.  This entry point takes its scratch from a fixed array inside the library,
 *   LSA_NOALLOC_SCRATCH_BYTES (64 MiB) of device memory that every GPU loading the library holds
 *   until the process exits.  It calls no cudaMalloc, cudaFree or allocating library routine.
 *   Arguments, results and errors are those of lsa_index without ws / ws_bytes and without the
 *   debug score exports; the caller still owns every input and output.
 *   device_error  int32 device word or NULL: receives (asynchronously, on `stream`) the device
 *                 error word of this call (LSA_DEVERR_* bits).
 *   Returns LSA_ERR_WORKSPACE when the sizes need more scratch than LSA_NOALLOC_SCRATCH_BYTES
 *   (lsa_index_workspace_bytes tells how much they need; e.g. 32 sequences x 128K tokens of
 *   flat indexing need about 34 MB).
 *   The first call on a device looks up the scratch array's device address for that device
 *   (cudaGetSymbolAddress, with the device current) and keeps it for the life of the process;
 *   make that first call before any stream capture, and do not call this entry point after a
 *   cudaDeviceReset of that device (the array may then sit at another address).  All calls on a device share the array and it keeps the previous call's contents;
 *   each call clears what must start at zero.  Calls whose work overlaps on the GPU (several
 *   streams or host threads at once) race on the array: serialise them.
 */
#define LSA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
lsa_status lsa_index_noalloc(const void *q_I, const void *w_I, const void *k_I, const void *k_mean,
                             const int32_t *kv_len, const int32_t *q_pos, int B, int T, int H_I,
                             int D_I, int64_t L_max, int K_sparse, int sink, int swa, int page,
                             int sub_block, int M, int32_t *indices, int32_t *device_error,
                             void *stream);

/*
 * lsa_quantize_fp8 -- per-row FP8 (E4M3) quantisation for the FP8 indexer.
 *   Paper: Sec. 2.2 ("Why Lightning": the indexer may compute in FP8) and Sec. 1 (DSA
 *   lowers the indexer's cost by FP8 quantisation).  The pages fix no scheme; this library's:
 *   for each row of D values, scale = max|x| / 448 (fp32) and code = E4M3(x / scale), rounded to
 *   the nearest even code and saturated to +-448 (OCP E4M3: bias 7, 3 mantissa bits, no
 *   infinities), both quotients in IEEE fp32; an all-zero row gets scale 0 and zero codes.
 *   Use it on key rows (one token's d_I values: the FP8 key cache) and on query rows (one
 *   (token, head) vector).
 *   x       bf16 device             input rows: row r at x + r * x_stride (elements)
 *   codes   uint8 device            out: E4M3 codes, row r at codes + r * codes_stride (bytes;
 *                                   pointer and stride even)
 *   scales  fp32 device             out: per-row scales at scales[r * scales_stride]
 *   D       even, 2..4096; x_stride >= D, codes_stride >= D, scales_stride >= 1 (strides let a
 *           caller write a new token's key straight into its slot of a [B, L_max, D] cache)
 *   device_error  int32 device word or NULL: LSA_DEVERR_NONFINITE is OR-ed in if an input is
 *                 NaN or infinite (its row's codes are then meaningless).
 *   Asynchronous on `stream`; rows == 0 does nothing.  LSA_ERR_INVALID_ARG on a NULL pointer or
 *   a bad size, LSA_ERR_CUDA if the launch fails.
 */
lsa_status lsa_quantize_fp8(const void *x, int64_t x_stride, int64_t rows, int D, uint8_t *codes,
                            int64_t codes_stride, float *scales, int64_t scales_stride,
                            int32_t *device_error, void *stream);

/*
 * lsa_index_fp8 -- lsa_index (flat indexer, M = 0) on FP8 queries and keys.
 *   Paper: Sec. 2.2 Eq. 1-2 and Sec. 3.1 as lsa_index, with the FP8 computation the pages name
 *   as the indexer's low-cost option.  The score of key s for query t is Eq. 1 on the decoded
 *   rows:  I[t,s] = sum_j w[t,j] * max(0, qs[t,j] * ks[s] * (q8[t,j] . k8[s])),
 *   accumulated in fp32 on the tensor cores (kind::f8f6f4); selection, output and errors are
 *   those of lsa_index.
 *   q8       uint8 [B, T, H_I, D_I]  E4M3 query codes (lsa_quantize_fp8 over B*T*H_I rows)
 *   q_scale  fp32 [B, T, H_I]        their scales
 *   w_I      bf16 [B, T, H_I]        head weights
 *   k8       uint8 [B, L_max, D_I]   E4M3 key cache (lsa_quantize_fp8 over the key rows)
 *   k_scale  fp32 [B, L_max]         its per-token scales
 *   H_I in {64, 128}, D_I = 128, B*T <= 65535; q8, k8 and ws 16-byte aligned.  Other sizes
 *   return LSA_ERR_UNSUPPORTED (the FP8 scorer exists only on the tensor cores).
 *   The workspace is lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, 128, 8, 0).
 */
lsa_status lsa_index_fp8(const uint8_t *q8, const float *q_scale, const void *w_I,
                         const uint8_t *k8, const float *k_scale, const int32_t *kv_len,
                         const int32_t *q_pos, int B, int T, int H_I, int D_I, int64_t L_max,
                         int K_sparse, int sink, int swa, int32_t *indices, float *scores_dbg,
                         void *ws, size_t ws_bytes, void *stream);

/*
 * lsa_get_error -- wait for `stream`, then read the device error word of the workspace used by
 * the last lsa_index / lsa_attend call on it (each of those calls clears the word when it
 * starts).  *device_code receives the OR of LSA_DEVERR_* bits (0 = clean).  Returns LSA_OK,
 * LSA_ERR_DEVICE when the word is non-zero, or LSA_ERR_CUDA if the stream reports a fault.
 */
lsa_status lsa_get_error(const void *ws, int32_t *device_code, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
