/*
 * msa.h -- C ABI of the MiniMax Sparse Attention (MSA) hot path on NVIDIA
 * B200 (sm_100a).  Library: libmsa.so (long_context_index_b200/).
 *
 * The method (titansim.online summary of "MiniMax Sparse Attention"):
 *   * Index branch, eq. (6) (section 4.2): per GQA group r and query i,
 *       S_ij = <Q_idx_i^(r), K_idx_j> / sqrt(d_idx),
 *       M_ib = max_{j in block b, j <= i} S_ij          (causal block max-pool),
 *     then the top-k blocks by M, the local block always included, form
 *     I_i^(r).  Selection ranks raw scores; nothing is exponentiated
 *     (section 4.4.1).  One index query per group and one index key shared by
 *     all groups (m.163.com post, "Step 1 Index Attention":
 *     Q_idx in R^{n x h x d}, K_idx in R^{n x 1 x d}).
 *   * Main branch, eq. (8) (section 4.3): every query head h of group r runs
 *     exact, causally masked softmax attention over K^(r), V^(r) gathered at
 *     the selected blocks.  Dense attention is eq. (1) (section 2.2).
 *
 * Conventions shared by every entry point:
 *   * Tensors are caller-owned DEVICE memory, contiguous, row-major with the
 *     last dimension innermost, base addresses 16-byte aligned.  bf16 values
 *     are passed as raw 16-bit patterns (void*).  The library never allocates
 *     device memory: callers query msa_workspace_size() and pass a device
 *     workspace of at least that many bytes (256-byte aligned).
 *   * Head h of the main branch belongs to group r = h / (h_q / h_kv).
 *   * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  They are stateless: concurrent calls on different
 *     streams with different workspaces are safe.
 *   * Return value: MSA_OK, or a negative MSA_ERR_* code.  Argument errors are
 *     detected on the host before anything is launched.  Kernels bound every
 *     wait instead of hanging; a wait that gave up is recorded in the status
 *     word at the start of the call's workspace, which msa_device_status()
 *     reads (MSA_ERR_TIMEOUT).
 *   * block_ids: int32 [rows, h_kv, topk], ascending, padded with -1 when a
 *     row has fewer than topk eligible blocks.
 *   * Positions: query row i of a prefill sits at absolute position
 *     q_pos0 + i (q_pos0 = 0 for a full prefill, n_kv - n_q for the final
 *     chunk of a chunked prefill).  A decode query sits at position L_b - 1 of
 *     its sequence, whose cache already holds that position.
 *   * Supported shapes: d in {64, 128}; d_idx in {32, 64, 128};
 *     block_k in {64, 128}; 1 <= topk <= 32; h_q % h_kv == 0 and the group
 *     size h_q / h_kv divides 128; n_q, n_kv <= 2^24 (MSA_ERR_UNSUPPORTED
 *     otherwise).
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define MSA_OK 0
#define MSA_ERR_INVALID (-1)     /* null pointer, negative or inconsistent size */
#define MSA_ERR_UNSUPPORTED (-2) /* shape outside the supported set above */
#define MSA_ERR_MISALIGNED (-3)  /* a base address is not 16-byte aligned */
#define MSA_ERR_WORKSPACE (-4)   /* workspace smaller than msa_workspace_size() */
#define MSA_ERR_CUDA (-5)        /* a CUDA call or launch failed */
#define MSA_ERR_TIMEOUT (-6)     /* a kernel gave up a bounded wait */

/* Operation ids for msa_workspace_size(). */
#define MSA_OP_INDEX_TOPK 0
#define MSA_OP_PREFILL 1
#define MSA_OP_DECODE 2
#define MSA_OP_INDEX_TOPK_VARLEN 3 /* n_q = total rows, batch = sequences */
#define MSA_OP_PREFILL_VARLEN 4    /* n_q = total rows, batch = sequences */
#define MSA_OP_INDEX_PROJECT 5     /* n_q = rows */

/* Problem parameters (the pages' notation: H_q, H_kv, d_h, d_idx, B_k, k). */
typedef struct {
  int h_q;         /* query heads of the main branch */
  int h_kv;        /* KV heads = GQA groups = index queries per token */
  int d;           /* head dimension d_h of Q, K, V */
  int d_idx;       /* index dimension of Q_idx, K_idx */
  int block_k;     /* KV block size B_k */
  int topk;        /* selected blocks per (query, group), local block included */
  int causal;      /* 1: key j visible from position p iff j <= p; 0: all keys */
  int force_local; /* 1: the block holding the query position is always selected */
  float scale;     /* main-branch softmax scale; <= 0 means 1/sqrt(d) */
  int pool;        /* block pooling of the index scores: 0 = max (eq. (6)); 1 = mean over the block's visible
                      keys (the MoBA-style mean pooling the m.163.com post compares max-pooling with), ranked
                      by the fp32 quotient of the exact score sum and the key count */
} msa_params;

/*
 * Workspace bytes needed by one call of `op` with these sizes (batch and
 * max_kv are used by MSA_OP_DECODE only; n_q/n_kv by the prefill ops).
 * Returns 0 for invalid arguments.  Host-only; never touches the GPU.
 */
MSA_API size_t msa_workspace_size(int op, const msa_params* p, int n_q, int n_kv, int batch, int max_kv);

/*
 * Index projections ahead of the index branch (titansim.online section 4.2:
 * an index-query projection per GQA group and one index-key projection
 * shared by all groups):
 *   Q_idx[i, r, :] = x[i, :] W_q^idx(r)^T,   K_idx[i, 0, :] = x[i, :] W_k^idx^T
 * computed as one GEMM on the tensor cores with fp32 accumulation, rounded
 * to bf16 (nearest even).
 *   x      bf16 [n, d_model]                 hidden states (d_model % 8 == 0)
 *   w_idx  bf16 [(h_kv + 1) * d_idx, d_model] stacked weights, nn.Linear
 *          layout: rows r*d_idx .. (r+1)*d_idx - 1 are W_q^idx(r), the last
 *          d_idx rows W_k^idx
 *   q_idx  bf16 [n, h_kv, d_idx] output;  k_idx bf16 [n, 1, d_idx] output
 * Uses p->h_kv and p->d_idx; the workspace is msa_workspace_size
 * (MSA_OP_INDEX_PROJECT, p, n, 0, 0, 0) bytes (the status word).
 */
MSA_API int msa_index_project(const msa_params* p, const void* x, const void* w_idx, int n, int d_model,
                              void* q_idx, void* k_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Index branch of a (chunked) prefill: eq. (6) scores, causal block
 * max-pool and top-k with the local block (titansim.online section 4.2).
 *   q_idx     bf16 [n_q, h_kv, d_idx]  index queries, one per group
 *   k_idx     bf16 [n_kv, 1, d_idx]    index keys, shared by all groups
 *   block_ids int32 [n_q, h_kv, topk]  output
 * Ranking is by raw dot product (the 1/sqrt(d_idx) factor is positive and
 * does not change order); ties go to the lower block index.  With integer-
 * valued index inputs the scores are exact, and the ids are exactly those of
 * the definition.  Requires q_pos0 >= 0 and q_pos0 + n_q <= n_kv.
 */
MSA_API int msa_index_topk(const msa_params* p, const void* q_idx, const void* k_idx, int n_q, int n_kv,
                   int q_pos0, int32_t* block_ids, void* ws, size_t ws_bytes, void* stream);

/*
 * Main branch of a (chunked) prefill, eq. (8) (titansim.online section 4.3):
 *   q         bf16 [n_q, h_q, d]
 *   k, v      bf16 [n_kv, h_kv, d]
 *   block_ids int32 [n_q, h_kv, topk] from msa_index_topk, or NULL for the
 *             dense run (every causal block: eq. (1))
 *   o         bf16 [n_q, h_q, d] output (fp32 accumulation, rounded to
 *             nearest even)
 * Ids must be valid: each -1 or a block holding a visible key of the row,
 * and the non-negative ids of a (row, group) pairwise distinct (a repeated id
 * would be attended twice; msa_index_topk never emits one).
 * The sparse run indexes its schedule with 32-bit integers: n_q * h_kv * topk,
 * the (query wave of 4096 rows, group, block) lists, and the partial rows
 * (about 128 * n_q * h_kv * topk * h_kv / h_q) must each stay below 2^31
 * (MSA_ERR_UNSUPPORTED otherwise; far beyond what one GPU's memory holds at
 * the model shapes).
 */
MSA_API int msa_sparse_attn_prefill(const msa_params* p, const void* q, const void* k, const void* v,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * One batched decode step: for every sequence b the query at position
 * L_b - 1 runs the index branch over its whole index-key cache, then the main
 * branch over the selected blocks.  The sparse step is persistent: the index
 * scan splits the blocks of all sequences into equal ranges per CTA, the
 * attention splits the (sequence, group, slot) list the same way, and partial
 * results of a sequence or group split between CTAs are merged by the last
 * CTA to finish it.  The step runs as two launches (index scan, then
 * attention); with MSA_OPT_DECODE_FUSED set (msa_set_option) a step that fits
 * one co-resident wave of CTAs runs as one cooperative launch whose attention
 * CTAs start as soon as the ids of their own sequences are merged.
 *   q            bf16 [batch, h_q, d]
 *   q_idx        bf16 [batch, h_kv, d_idx]
 *   k_cache,
 *   v_cache      bf16 [sum L_b, h_kv, d]   sequences stored back to back
 *   k_idx_cache  bf16 [sum L_b, 1, d_idx]
 *   cu_kv        int64 [batch + 1] DEVICE prefix sums of L_b (cu_kv[0] = 0)
 *   max_kv       host upper bound on every L_b (sizes the launch grid)
 *   dense        1: attend to every causal block (the index branch is skipped
 *                and block_ids is not written)
 *   block_ids    int32 [batch, h_kv, topk] output (may be NULL when dense)
 *   o            bf16 [batch, h_q, d] output
 * Every L_b must be in [1, max_kv].  h_kv <= 8; with dense = 0 also
 * batch <= 4096 and batch * max_kv < 2^31 (MSA_ERR_UNSUPPORTED otherwise).
 */
MSA_API int msa_sparse_attn_decode(const msa_params* p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Packed batches of independent prefills (the serving form: many sequences
 * of different lengths in one call).  Sequence s owns rows
 * [cu_seqlens[s], cu_seqlens[s + 1]) of every tensor below; its query i sits
 * at position i of the sequence (a full causal prefill of each sequence), it
 * sees only its own keys, and its block ids are local to it.  Per sequence
 * the result is exactly that of msa_index_topk / msa_sparse_attn_prefill on
 * its rows (titansim.online section 4.2 and eq. (8), section 4.3).
 *   cu_seqlens    int32 [batch + 1] DEVICE prefix of the sequence lengths:
 *                 cu_seqlens[0] = 0, non-decreasing, cu_seqlens[batch] = total.
 *                 A violation is found on the device: nothing is computed and
 *                 msa_device_status() reports MSA_ERR_INVALID.
 *   topk_per_seq  int32 [batch] DEVICE, or NULL: the number of blocks kept
 *                 for each sequence (adaptive k; the future-work direction of
 *                 titansim.online section 5.3), clamped to [1, p->topk]; the
 *                 ids beyond it are -1.  NULL keeps p->topk for every sequence.
 *   q_idx [total, h_kv, d_idx], k_idx [total, 1, d_idx], block_ids
 *   [total, h_kv, topk], q [total, h_q, d], k, v [total, h_kv, d],
 *   o [total, h_q, d]; layouts and types as for the single-sequence calls.
 * The prefill runs the sparse (block-major) path only: block_ids must not be
 * NULL.  batch >= 1; total <= 2^24.  Workspace: msa_workspace_size with
 * MSA_OP_INDEX_TOPK_VARLEN / MSA_OP_PREFILL_VARLEN, n_q = total and
 * batch = the number of sequences.
 */
MSA_API int msa_index_topk_varlen(const msa_params* p, const void* q_idx, const void* k_idx,
                                  const int32_t* cu_seqlens, int batch, int total, const int32_t* topk_per_seq,
                                  int32_t* block_ids, void* ws, size_t ws_bytes, void* stream);
MSA_API int msa_sparse_attn_prefill_varlen(const msa_params* p, const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens, int batch, int total,
                                           const int32_t* block_ids, void* o, void* ws, size_t ws_bytes,
                                           void* stream);

/*
 * msa_sparse_attn_decode with adaptive k: sequence b keeps
 * min(max(topk_per_seq[b], 1), p->topk) blocks (its local block included when
 * force_local), its remaining ids being -1 -- the per-sequence choice of k
 * that titansim.online section 5.3 names as future work.  topk_per_seq is
 * int32 [batch] DEVICE memory, or NULL (every sequence keeps p->topk: exactly
 * msa_sparse_attn_decode).  Ignored when dense.  Everything else as for
 * msa_sparse_attn_decode; the workspace is the same.
 */
MSA_API int msa_sparse_attn_decode_adaptive_k(const msa_params* p, const void* q, const void* q_idx,
                                              const void* k_cache, const void* v_cache, const void* k_idx_cache,
                                              const int64_t* cu_kv, const int32_t* topk_per_seq, int batch,
                                              int max_kv, int dense, int32_t* block_ids, void* o, void* ws,
                                              size_t ws_bytes, void* stream);

/*
 * Device status recorded by the last call that used workspace `ws`: MSA_OK,
 * MSA_ERR_TIMEOUT when one of its kernels gave up a bounded wait, or
 * MSA_ERR_INVALID when a varlen call found cu_seqlens invalid.  Every
 * call clears the status word (the first 4 bytes of its workspace) before
 * launching.  Synchronises `stream` first; returns MSA_ERR_CUDA if that or the
 * 4-byte read fails.
 */
MSA_API int msa_device_status(const void* ws, void* stream);

/*
 * Allocation-free variant of msa_sparse_attn_decode, for callers that cannot
 * allocate device memory (no workspace argument).  The paper has no
 * counterpart: this is a deployment convenience.  Arguments and results are
 * exactly those of msa_sparse_attn_decode.
 *   * Scratch: a file-scope device array of MSA_NOALLOC_SCRATCH_BYTES that
 *     every GPU which loads the library holds until process exit.  A problem
 *     whose scratch would not fit is rejected with MSA_ERR_WORKSPACE before
 *     anything is launched.  The scratch is that of the run requested: the
 *     sparse run needs completion counters, top-k candidates and one partial
 *     per (attention CTA, group) share (64 q heads, 4 KV heads, d = 128,
 *     k = 16: about 10 MB at 64 sequences); the dense run needs 32 split
 *     partials per head.  msa_workspace_size(MSA_OP_DECODE, ...) reports the
 *     larger of the two, an upper bound.
 *   * The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   * Every call on a device shares the one array: calls that overlap on the
 *     GPU (different streams, no ordering between them) race and may return
 *     wrong results.  Serialise them, e.g. on one stream.
 *   * The array keeps the last call's contents; the call itself clears what
 *     must start at zero.  msa_device_status() does not apply to it.
 */
#define MSA_NOALLOC_SCRATCH_BYTES (16u << 20)
MSA_API int msa_sparse_attn_decode_noalloc(const msa_params* p, const void* q, const void* q_idx,
                                           const void* k_cache, const void* v_cache, const void* k_idx_cache,
                                           const int64_t* cu_kv, int batch, int max_kv, int dense,
                                           int32_t* block_ids, void* o, void* stream);

/*
 * MXFP8 quantisation of a bf16 tensor (the MXFP8 KV cache of the zhichai.net
 * summary; format: OCP Microscaling formats v1.0, E4M3 elements with an E8M0
 * scale per 32 consecutive elements of the last dimension).  Per block:
 * e = floor(log2 max|x|) - 8 clamped to [-127, 127] (-127 for an all-zero
 * block), elements x / 2^e rounded to the E4M3 grid (nearest even, saturated
 * at +-448), scale byte e + 127.
 *   x       bf16  [rows, cols], cols % 32 == 0 (16-byte aligned)
 *   q       uint8 [rows, cols] E4M3 codes (16-byte aligned), output
 *   scales  uint8 [rows, cols / 32] E8M0 codes, output
 * Element i of x dequantises to E4M3(q_i) * 2^(scales[i / 32] - 127).
 * Asynchronous on `stream`; no workspace.
 */
MSA_API int msa_quantize_mxfp8(const void* x, long long rows, int cols, void* q, void* scales, void* stream);

/*
 * One batched decode step over MXFP8 caches (codes and scales as produced by
 * msa_quantize_mxfp8): K, V and the index keys are stored as E4M3 with an
 * E8M0 scale per 32 elements, about half the bytes of bf16 caches; the query,
 * the index query and the output stay bf16.  The kernels dequantise exactly
 * (E4M3 code * 2^(scale - 127) is exact in bf16), so the result is the bf16
 * decode step of the dequantised caches: the ids those caches select and
 * attention over their values.  Sparse run only; d = 128.
 *   k8, v8         uint8 [sum L_b, h_kv, d]   E4M3 codes (16-byte aligned)
 *   k_scale,
 *   v_scale        uint8 [sum L_b, h_kv, d / 32] E8M0 codes (4-byte aligned)
 *   k_idx8         uint8 [sum L_b, 1, d_idx]  E4M3 codes (16-byte aligned)
 *   k_idx_scale    uint8 [sum L_b, 1, d_idx / 32]
 *   topk_per_seq   as for msa_sparse_attn_decode_adaptive_k (NULL: topk)
 * Other arguments, limits and the workspace as for msa_sparse_attn_decode.
 */
MSA_API int msa_sparse_attn_decode_mxfp8(const msa_params* p, const void* q, const void* q_idx, const void* k8,
                                         const void* k_scale, const void* v8, const void* v_scale,
                                         const void* k_idx8, const void* k_idx_scale, const int64_t* cu_kv,
                                         const int32_t* topk_per_seq, int batch, int max_kv, int32_t* block_ids,
                                         void* o, void* ws, size_t ws_bytes, void* stream);

/* Human-readable text of a status code (static storage). */
/*
 * Process-wide options (host only; take effect at the next call).
 *   MSA_OPT_DECODE_FUSED  the form of a sparse decode step: 1 = one
 *       cooperative launch (index scan and attention in every CTA, the ids
 *       handed over through the L2) whenever the step fits one co-resident
 *       wave, else the two launches; 0 = always the two persistent launches
 *       (index scan, then streaming attention).  Both forms compute the same
 *       ids and outputs bit for bit.
 * msa_set_option returns MSA_OK, or MSA_ERR_INVALID for an unknown option or
 * value; msa_get_option returns the value, or MSA_ERR_INVALID.
 */
#define MSA_OPT_DECODE_FUSED 0
MSA_API int msa_set_option(int option, int value);
MSA_API int msa_get_option(int option);

MSA_API const char* msa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
