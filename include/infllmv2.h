/*
 * infllmv2.h -- C ABI of the InfLLM-V2 dense-sparse switchable attention
 * hot path for NVIDIA B200 (sm_100a).
 *
 * The method (InfLLM-V2: Dense-Sparse Switchable Attention for Seamless
 * Short-to-Long Adaptation; abstract on the cochat.ai paper page) reuses the
 * dense attention's parameters.  For a long input it works in two steps: it
 * picks the key blocks that matter for each query, then runs attention over
 * those blocks alone (reportify digest, Technical Mechanism).  A short input
 * gets plain dense attention (InfLLM-V2 skill write-up, Architecture
 * Overview, the dense pathway bullet).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent),
 *   16-byte aligned, densely packed in the stated row-major layout.
 * - bf16 = IEEE bfloat16 stored as uint16; fp32 = float.
 * - Layouts (BSHD):  Q, O  [B, T, Hq,  d] bf16
 *                    K, V  [B, T, Hkv, d] bf16
 *                    Kc    [B, n_c, Hkv, 2, d] bf16, n_c = (T-32)/16 + 1 (0 if T < 32):
 *                          each compressed key as the pair (hi, lo), value hi + lo
 *                    idx   [B, Hkv, T, topk] int32
 *                    lse   [B, Hq, T] fp32 (natural log)
 * - GQA: query head h belongs to KV head g = h / (Hq/Hkv).
 * - `stream` is a cudaStream_t passed as void*; NULL = legacy default stream.
 *   Every call only ENQUEUES work on `stream` and returns; nothing
 *   synchronises except infllmv2_get_status.
 * - Ownership: the caller allocates and frees every buffer, workspace
 *   included.  The library allocates no device memory; its only global state
 *   is one status word per device in a static __device__ variable.  Inputs
 *   are read-only; outputs are fully overwritten.
 * - Return value: INFLLMV2_OK or a negative error code.  On a host-side error
 *   nothing is enqueued.  Device-side conditions (a bounded wait that expired,
 *   a decode sequence at capacity) set bits in the device status word, read
 *   with infllmv2_get_status.
 * - Built and supported: head_dim == 128, block_size == 64, cmp_kernel == 32,
 *   cmp_stride == 16, causal == 1, Hq/Hkv in {1,2,4,8,16}, T <= 2^22 tokens;
 *   block selection (select_blocks and the sparse branches of forward and
 *   prefill_chunk) up to INFLLMV2_MAX_SELECT_T tokens per sequence, decode up
 *   to INFLLMV2_MAX_DECODE_T.  Other values return INFLLMV2_ERR_UNSUPPORTED
 *   before anything is enqueued.
 */
#ifndef INFLLMV2_H_
#define INFLLMV2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define INFLLMV2_MAX_SELECT_T   262144  /* 4096 key blocks */
#define INFLLMV2_MAX_DECODE_T   524288  /* 8192 key blocks */

#define INFLLMV2_OK                    0
#define INFLLMV2_ERR_INVALID_ARG      -1  /* null pointer, bad shape, topk < forced count */
#define INFLLMV2_ERR_UNSUPPORTED      -2  /* a value outside the built configuration, misaligned pointer */
#define INFLLMV2_ERR_CUDA             -3  /* a CUDA runtime/driver call failed (launch, tensor map) */
#define INFLLMV2_ERR_TIMEOUT          -4  /* a device-side bounded wait expired (reported by get_status) */
#define INFLLMV2_ERR_WORKSPACE        -5  /* ws_bytes smaller than infllmv2_workspace_bytes() */
#define INFLLMV2_ERR_DEVICE_CHECK     -6  /* a device-side argument check failed (reported by get_status) */

/* Device status bits (infllmv2_get_status). */
#define INFLLMV2_STATUS_TIMEOUT        0x1
#define INFLLMV2_STATUS_SEQ_FULL       0x2  /* decode: seqlens[b] reached the cache capacity */
#define INFLLMV2_STATUS_CHECK          0x4  /* bounds-checked build only: an index check failed
                                               and its access was skipped */

/* The method's knobs.  Source of each: the sequence-length switch and the
 * block size (skill write-up, Implementation Steps 2-3); compressed keys that
 * aggregate tokens hierarchically, here by mean-pooling with window 32 and
 * stride 16 (skill write-up, Core Concept); blocks kept for local context
 * (the sliding pattern, ibid.) and the initial block; top-k block selection
 * (reportify digest, Technical Mechanism). */
typedef struct infllmv2_params {
  int32_t B;                /* batch (sequences) */
  int32_t T;                /* tokens per sequence; for decode: cache capacity Lmax */
  int32_t Hq;               /* query heads */
  int32_t Hkv;              /* key/value heads (GQA groups) */
  int32_t head_dim;         /* d; must be 128 */
  int32_t block_size;       /* key block size; must be 64 */
  int32_t cmp_kernel;       /* compression window; must be 32 */
  int32_t cmp_stride;       /* compression stride; must be 16 */
  int32_t topk;             /* blocks attended per query row, forced ones included; 1..256 */
  int32_t n_init;           /* always-kept initial blocks 0..n_init-1 */
  int32_t n_local;          /* always-kept most recent blocks cur-n_local+1..cur */
  int32_t switch_threshold; /* forward(): dense iff T <= switch_threshold */
  float   scale;            /* softmax scale; 0 => 1/sqrt(head_dim) */
  int32_t causal;           /* must be 1 */
} infllmv2_params;

/* Operations for infllmv2_workspace_bytes. */
#define INFLLMV2_OP_SELECT   1
#define INFLLMV2_OP_FORWARD  2
#define INFLLMV2_OP_DECODE   3
#define INFLLMV2_OP_ATTN     4  /* sparse_attn: union lists (groups of 4+ heads) or packed K/V */
#define INFLLMV2_OP_ATTN_PER_TOKEN 5  /* sparse_attn_per_token: packed K and V */
#define INFLLMV2_OP_FORWARD_FP32   6  /* forward_fp32: block scores (0 when dense) */
#define INFLLMV2_OP_BACKWARD       7  /* sparse_attn_backward */

/* Path reported by infllmv2_forward. */
#define INFLLMV2_PATH_DENSE  1
#define INFLLMV2_PATH_SPARSE 2

/*
 * Compressed keys: Kc[b, j, g, :] = (1/32) * sum_{i=16j}^{16j+31} K[b, i, g, :]
 * for j < n_c (the compressed pattern's token aggregation, skill write-up,
 * Core Concept; mean-pooling with window 32, stride 16).  Sums in fp32 in
 * token order and stores the mean m as two bf16 planes, hi = RNE(m) and
 * lo = RNE(m - hi) (about 17 significant bits: a single bf16 rounding moves
 * block scores by up to ~1e-2 relative, more than selection can absorb).
 *   K  [B, T, Hkv, d] bf16 (in);  Kc [B, n_c, Hkv, 2, d] bf16 (out).
 */
int infllmv2_compress_keys(const infllmv2_params* p, const void* K, void* Kc,
                           void* stream);

/*
 * Block selection (reportify digest, Technical Mechanism: the first of the
 * two steps picks the relevant key/value blocks; scores are summed over the
 * heads of a group, skill write-up, Architecture Overview, Hardware Kernel
 * bullet).  For every
 * (b, g, t):
 *   s[h, j] = scale * Q[b,t,h,:] . Kc[b,j,g,:]   for the visible windows
 *             j < v(t) = #{j : 16j + 31 <= t},  h in group g;
 *   p[h, :] = softmax_j s[h, :];   S[j] = sum_{h in g} p[h, j];
 *   bs[blk] = max { S[j] : window j overlaps block blk's tokens } (-inf if none);
 *   forced  = {0..n_init-1} U {cur-n_local+1..cur}, cur = t / 64;
 *   the other topk-|forced| slots take the blocks blk <= cur with the largest
 *   bs, equal scores to the lower block.
 *   idx[b, g, t, :] = selected blocks ascending, padded with -1.
 *   Q  [B, T, Hq, d] bf16 (in);  Kc from infllmv2_compress_keys (in);
 *   idx [B, Hkv, T, topk] int32 (out);
 *   ws: device workspace of at least infllmv2_workspace_bytes(p, INFLLMV2_OP_SELECT)
 *   bytes (block scores of every row; contents on return unspecified).
 */
int infllmv2_select_blocks(const infllmv2_params* p, const void* Q, const void* Kc,
                           int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Block-sparse causal attention (reportify digest, Technical Mechanism: the
 * second step attends only to the picked blocks):
 *   keys(t) = union over blk in idx[b, g, t, :] (blk >= 0) of [64 blk, 64 blk + 63],
 *             clipped to [0, t];
 *   O[b,t,h,:] = sum_{i in keys(t)} softmax_i(scale * q.K_i) V_i;
 *   lse[b,h,t] = log sum_{i in keys(t)} exp(scale * q.K_i).
 *   idx rows must be ascending with valid entries first (as select_blocks
 *   writes them); entries > t/64 are ignored.
 * Schedule: with Hq/Hkv in {4, 8, 16} and ws of at least
 * infllmv2_workspace_bytes(p, INFLLMV2_OP_ATTN) bytes, query tiles of 128
 * rows (128/G tokens x G heads) run over the union of their tokens' selected
 * blocks, each row masked to its own token's blocks, so a block that several
 * tokens of a tile selected is loaded and multiplied once (ws holds the
 * union lists and K and V repacked into 16 KB block tiles, each block then
 * gathered by one bulk copy; contents on return unspecified).  Otherwise (smaller groups, or
 * ws NULL / too small) the call runs infllmv2_sparse_attn_per_token's
 * schedule.  Results agree within rounding.
 */
int infllmv2_sparse_attn(const infllmv2_params* p, const void* Q, const void* K,
                         const void* V, const int32_t* idx, void* O, float* lse, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * infllmv2_sparse_attn with one work item per query token: the token's G
 * heads against its own selected blocks only, two blocks per tensor-core
 * product with keys on the 128-row side.  ws: optional, at least
 * infllmv2_workspace_bytes(p, INFLLMV2_OP_ATTN_PER_TOKEN) bytes: K and V are
 * first repacked into block-contiguous tiles (one 16 KB chunk per 64-key
 * block and kv head) so that every selected block is gathered by one bulk
 * copy; with ws NULL (or too small) blocks are gathered from K and V by
 * tensor-map copies.  Same arguments and results as infllmv2_sparse_attn.
 */
int infllmv2_sparse_attn_per_token(const infllmv2_params* p, const void* Q, const void* K,
                                   const void* V, const int32_t* idx, void* O, float* lse,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * Gradients of infllmv2_sparse_attn with the block selection held fixed (the
 * method is a trainable sparse attention: paper page, Abstract; the selection
 * is a discrete choice, so training propagates through the attention over the
 * chosen blocks).  For every query row over keys(t) as in infllmv2_sparse_attn,
 * with P = softmax(scale q K^T) recomputed from lse and D = rowsum(dO * O):
 *   dP = dO V^T,  dS = P * (dP - D),
 *   dQ[row] = scale dS K,  dK += scale dS^T q,  dV += P^T dO,
 * dK and dV summing over every row that selected a key's block.
 *   Q, K, V, idx as given to infllmv2_sparse_attn; O, lse its outputs;
 *   dO [B, T, Hq, d] bf16 (in);
 *   dQ [B, T, Hq, d], dK, dV [B, T, Hkv, d] fp32 (out);
 *   ws: at least infllmv2_workspace_bytes(p, INFLLMV2_OP_BACKWARD) bytes.
 * Built for Hq/Hkv in {4, 8, 16} (other groups: INFLLMV2_ERR_UNSUPPORTED).
 * dK and dV are summed in a fixed order (the rows of each block ascending),
 * so repeated calls give identical results.  For the dense path's gradients
 * pass an idx that lists every block (topk >= number of blocks).
 */
int infllmv2_sparse_attn_backward(const infllmv2_params* p, const void* Q, const void* K,
                                  const void* V, const int32_t* idx, const void* O,
                                  const float* lse, const void* dO, float* dQ, float* dK,
                                  float* dV, void* ws, size_t ws_bytes, void* stream);

/*
 * Exact dense causal attention (skill write-up, Architecture Overview, the
 * dense pathway bullet): keys(t) = [0, t], same O and lse definitions as
 * infllmv2_sparse_attn.  Query tiles of 128 rows against 128-key tiles on the
 * tensor cores.  ws and ws_bytes are unused (may be NULL / 0).
 */
int infllmv2_dense_attn(const infllmv2_params* p, const void* Q, const void* K,
                        const void* V, void* O, float* lse, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * The compressed-attention branch (skill write-up, Core Concept: the
 * compressed pattern aggregates tokens hierarchically into representatives
 * that every query can attend to): each query row attends over the compressed
 * windows it can see,
 *   keys(t) = { j : 16 j + 31 <= t, j < n_c },
 *   O[b,t,h,:] = sum_{j in keys(t)} softmax_j(scale * q . Kc[j]) Vc[j],
 *   lse[b,h,t] = log sum_{j in keys(t)} exp(scale * q . Kc[j]);
 * a row with no visible window (t < 31) gets O = 0 and lse = -inf.
 *   Q [B, T, Hq, d] bf16 (in);
 *   Kc = infllmv2_compress_keys of K, Vc = infllmv2_compress_keys of V
 *     ([B, n_c, Hkv, 2, d] bf16, in; scores use both planes of Kc, the values
 *     the high plane of Vc);
 *   O [B, T, Hq, d] bf16, lse [B, Hq, T] fp32 (out).
 */
int infllmv2_compressed_attn(const infllmv2_params* p, const void* Q, const void* Kc,
                             const void* Vc, void* O, float* lse, void* stream);

/*
 * The switchable attention (skill write-up, Implementation Step 3: dense when
 * seq_len <= threshold, else sparse).  Sparse: compress_keys into Kc_ws, then
 * select_blocks into idx_ws, then sparse_attn.  Dense: dense_attn; Kc_ws and
 * idx_ws may be NULL.  *path_used (host pointer, may be NULL) receives
 * INFLLMV2_PATH_DENSE or INFLLMV2_PATH_SPARSE.
 *   Kc_ws: [B, n_c, Hkv, 2, d] bf16; idx_ws: [B, Hkv, T, topk] int32 (both out);
 *   ws: at least infllmv2_workspace_bytes(p, INFLLMV2_OP_FORWARD) bytes (0 when
 *   dense): the selection's block scores, then infllmv2_sparse_attn's.
 */
int infllmv2_forward(const infllmv2_params* p, const void* Q, const void* K,
                     const void* V, void* O, float* lse, void* Kc_ws, int32_t* idx_ws,
                     int32_t* path_used, void* ws, size_t ws_bytes, void* stream);

/*
 * The fp32 validation build of infllmv2_forward: the same switch and the same
 * steps (compressed keys, per-head softmax scores summed over the group and
 * max-pooled to blocks, top-k with the forced blocks, block-sparse or dense
 * causal attention), with every product and sum in fp32 on the CUDA cores:
 * compressed keys stored in fp32, scores and softmax in fp32, P and O never
 * rounded to bf16.  For checking the method's arithmetic to ~1e-6 (the
 * tensor-core path's error is set by bf16 rounding); not tuned for speed.
 *   Q, K, V as for infllmv2_forward (bf16, in);
 *   O [B, T, Hq, d] fp32, lse [B, Hq, T] fp32 (out);
 *   Kc32_ws [B, n_c, Hkv, d] fp32 and idx_ws [B, Hkv, T, topk] int32 (out;
 *     unused and may be NULL when dense);
 *   ws: at least infllmv2_workspace_bytes(p, INFLLMV2_OP_FORWARD_FP32) bytes.
 */
int infllmv2_forward_fp32(const infllmv2_params* p, const void* Q, const void* K,
                          const void* V, float* O, float* lse, float* Kc32_ws, int32_t* idx_ws,
                          int32_t* path_used, void* ws, size_t ws_bytes, void* stream);

/*
 * Chunked prefill: queries for the tokens q_offset .. q_offset+q_len-1 of a
 * sequence whose keys, values and compressed keys are already in the caches
 * (the chunk's own tokens included).  Each query row t gets exactly what
 * infllmv2_forward gives row t of the whole sequence: the same switch (dense
 * iff p->T <= p->switch_threshold), selection over the compressed keys
 * visible at t and the blocks <= t/64, attention over keys <= t.  Serving
 * splits a long prompt into such chunks (reportify digest, Performance
 * Evaluation: prefill and decode over a growing cache).
 *   p->T = q_offset + q_len: the tokens in the caches (INVALID_ARG otherwise);
 *   Q [B, q_len, Hq, d] bf16 (in); K, V [B, T, Hkv, d] bf16 (in);
 *   Kc [B, n_c(T), Hkv, 2, d] bf16 (in: compressed keys of the caches, e.g. from
 *     infllmv2_compress_keys or the decode steps' appends; unused when dense);
 *   O [B, q_len, Hq, d] bf16, lse [B, Hq, q_len] fp32 (out);
 *   idx [B, Hkv, q_len, topk] int32 (out; unused and may be NULL when dense);
 *   path_used: host int32 (may be NULL);
 *   ws: at least infllmv2_prefill_chunk_workspace_bytes(p, q_offset, q_len)
 *     bytes (0 when dense).
 */
size_t infllmv2_prefill_chunk_workspace_bytes(const infllmv2_params* p, int32_t q_offset,
                                              int32_t q_len);
int infllmv2_prefill_chunk(const infllmv2_params* p, int32_t q_offset, int32_t q_len,
                           const void* Q, const void* K, const void* V, const void* Kc,
                           void* O, float* lse, int32_t* idx, int32_t* path_used, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Variable-length prefill: n_seqs sequences of different lengths packed
 * together, each a query chunk over its own caches (the last q_len_i of its
 * k_len_i tokens: q_len_i = k_len_i is an ordinary prefill), so that serving
 * can prefill a batch of ragged prompts with one call (reportify digest,
 * Performance Evaluation: prefill speed-up on long inputs).  Every row gets
 * exactly what infllmv2_prefill_chunk gives it, with the switch taken per
 * sequence (dense iff k_len_i <= p->switch_threshold).  p->B and p->T are
 * ignored.  The sequences run one after another on `stream` and share ws.
 *   cu_seqlens_q, cu_seqlens_k: HOST int32 arrays of n_seqs + 1 ascending
 *     offsets from 0; q_len_i = cu_seqlens_q[i+1] - cu_seqlens_q[i] <= k_len_i;
 *   Q, O [total_q, Hq, d] bf16; K, V [total_k, Hkv, d] bf16;
 *   Kc: the sequences' compressed keys one after another, sequence i's
 *     n_c(k_len_i) rows [n_c_i, Hkv, 2, d] (as infllmv2_compress_keys writes
 *     them for B = 1); unused and may be NULL when no sequence is sparse;
 *   lse: sequence i's [Hq, q_len_i] fp32 block at element Hq * cu_seqlens_q[i];
 *   idx: sequence i's [Hkv, q_len_i, topk] int32 block at element
 *     Hkv * topk * cu_seqlens_q[i] (unused, may be NULL, when all are dense);
 *   path_used: host int32[n_seqs] (may be NULL);
 *   ws: at least infllmv2_prefill_varlen_workspace_bytes(...) bytes.
 */
size_t infllmv2_prefill_varlen_workspace_bytes(const infllmv2_params* p, int32_t n_seqs,
                                               const int32_t* cu_seqlens_q,
                                               const int32_t* cu_seqlens_k);
int infllmv2_prefill_varlen(const infllmv2_params* p, int32_t n_seqs,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            const void* Q, const void* K, const void* V, const void* Kc,
                            void* O, float* lse, int32_t* idx, int32_t* path_used, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * One decode step for B sequences (reportify digest, Performance Evaluation:
 * the operator speed-up is reported for both prefill and decode).  p->T is the cache
 * capacity Lmax in tokens; the compressed-key cache holds n_c(Lmax) rows.
 * For every sequence b, with pos = seqlens[b] (device int32, pos < Lmax):
 *   1. K_cache[b,pos] = k_new[b]; V_cache[b,pos] = v_new[b];
 *   2. if pos >= 31 and (pos-31) % 16 == 0: Kc_cache[b,(pos-31)/16] = mean of
 *      K_cache[b, pos-31 .. pos]  (incremental compressed-key cache);
 *   3. the new token attends as query row t = pos exactly as select_blocks +
 *      sparse_attn define it over the caches;
 *   4. seqlens[b] = pos + 1.
 *   q [B, Hq, d], k_new/v_new [B, Hkv, d] bf16 (in);
 *   K_cache/V_cache [B, Lmax, Hkv, d] bf16, Kc_cache [B, n_c(Lmax), Hkv, 2, d] bf16,
 *   seqlens [B] int32 (in/out);  O [B, Hq, d] bf16, lse [B, Hq] fp32 (out);
 *   idx_out [B, Hkv, topk] int32 (out, may be NULL);
 *   ws: at least infllmv2_workspace_bytes(p, INFLLMV2_OP_DECODE) bytes.
 * A sequence with seqlens[b] >= Lmax is left untouched, its O/lse rows are
 * zero and INFLLMV2_STATUS_SEQ_FULL is set.
 */
int infllmv2_decode_step(const infllmv2_params* p, const void* q, const void* k_new,
                         const void* v_new, void* K_cache, void* V_cache, void* Kc_cache,
                         int32_t* seqlens, void* O, float* lse, int32_t* idx_out,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * infllmv2_decode_step without a workspace argument: nothing is allocated,
 * by the caller or by the library.  The paper has no counterpart; this entry
 * point exists for callers that cannot allocate device memory.  A host
 * runtime that embeds the library often hands it only the step's inputs and
 * outputs: its own allocator already owns the rest of the GPU's memory (a
 * pool reserved up front), its plugin interface has no way to pass scratch
 * space, and a cudaMalloc of its own from inside the decode loop would fail
 * or fragment that pool.
 *
 * Arguments and results are those of infllmv2_decode_step.  The scratch is
 * one file-scope static __device__ array of INFLLMV2_NOALLOC_SCRATCH_BYTES
 * bytes inside the library, so every GPU that loads the library holds that
 * memory until the process exits.
 * - If infllmv2_workspace_bytes(p, INFLLMV2_OP_DECODE) exceeds the array, the
 *   call returns INFLLMV2_ERR_WORKSPACE and enqueues nothing.  (The B=16,
 *   131072-token, Hq=32, Hkv=2 decode needs about 19 MiB.)
 * - The first call on a device looks up the array's device address with
 *   that device current (cudaGetSymbolAddress); make this first call before
 *   any stream capture on that device.
 * - All calls share the one array, which keeps the last call's contents.
 *   Calls whose kernels can overlap on the GPU (different streams with no
 *   ordering between them) race on it and corrupt each other's results;
 *   calls issued on one stream are ordered and safe.  Nothing in the array
 *   needs clearing between calls: every kernel of a step writes the scratch
 *   it reads later in the same step.
 */
#define INFLLMV2_NOALLOC_SCRATCH_BYTES (32u << 20)
int infllmv2_decode_step_noalloc(const infllmv2_params* p, const void* q, const void* k_new,
                                 const void* v_new, void* K_cache, void* V_cache,
                                 void* Kc_cache, int32_t* seqlens, void* O, float* lse,
                                 int32_t* idx_out, void* stream);

/* Device workspace bytes needed by an operation (0 if none; SIZE_MAX on bad params). */
size_t infllmv2_workspace_bytes(const infllmv2_params* p, int32_t op);

/* Number of compressed-key rows for T tokens: (T-32)/16 + 1, or 0 if T < 32. */
int32_t infllmv2_num_compressed(int32_t T);

/*
 * Synchronises `stream`, returns the current device's status bits in
 * *status_out (host pointer) and clears them.  Returns INFLLMV2_OK, or
 * INFLLMV2_ERR_CUDA if the synchronisation itself failed (for example after
 * an earlier kernel fault).
 */
int infllmv2_get_status(void* stream, int32_t* status_out);

/*
 * Time limit, in nanoseconds, of every device-side bounded wait (mbarrier
 * polls; default 2e9 = 2 s).  A wait that runs out sets
 * INFLLMV2_STATUS_TIMEOUT, abandons its loop and the kernel returns after
 * releasing its tensor memory.  Takes effect for calls enqueued afterwards.
 */
void infllmv2_set_wait_limit(int64_t ns);

/*
 * Self-test of the timeout path: one CTA waits, with the current wait limit,
 * on an mbarrier that nothing ever arrives on.  The wait expires, the kernel
 * sets INFLLMV2_STATUS_TIMEOUT and returns; infllmv2_get_status then reports
 * the bit and the context stays usable.
 */
int infllmv2_selftest_timeout(void* stream);

/*
 * Measuring aid for the block-sparse attention's roofline: the rate at which
 * this GPU moves 16 KB key/value tiles from L2 into shared memory, the
 * movement that bounds the attention when tokens share few blocks
 * (reportify digest, Model Advantages: the method's kernels are designed to
 * cut HBM traffic, so the gathered blocks are served from L2).  One CTA per
 * SM issues `rounds` x 12 bulk copies of 16 KB (three 64 KB stages per round)
 * from pseudo-random 16 KB-aligned offsets of `src` (a device buffer of
 * src_bytes >= 16 KB; keep it smaller than L2 so that the copies hit L2)
 * into shared memory, and nothing else.  The caller times the launch on
 * `stream`; it moves *ctas_out x rounds x 196608 bytes.  *ctas_out (host
 * pointer, may be NULL) receives the number of CTAs.
 */
int infllmv2_gather_peak(const void* src, size_t src_bytes, int32_t rounds, int32_t* ctas_out,
                         void* stream);

/* Human-readable text of an error code. */
const char* infllmv2_strerror(int code);

/* Library version, e.g. 100 for 0.1.0. */
int infllmv2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INFLLMV2_H_ */
