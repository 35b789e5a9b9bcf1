// msa_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/msa.h"

namespace msa {

// Device status word values written by kernels.
constexpr int kDevOk = 0;
constexpr int kDevTimeout = 1;

// Bytes reserved at the start of every workspace: the device status word
// (int at offset 0) and padding to keep what follows 256-byte aligned.
constexpr size_t kWsHeader = 256;

// Encodes a tiled TMA descriptor for a bf16 tensor of rank 2..5.
// dims[0] is innermost; strides[] are the byte strides of dims 1..rank-1.
bool encode_tma_bf16(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle);
// The same for a uint8 tensor (MXFP8 codes).
bool encode_tma_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                   const uint32_t* box, CUtensorMapSwizzle swizzle);

// A packed batch of independent causal prefills (the varlen entry points):
// sequence s owns rows [cu_seqlens[s], cu_seqlens[s + 1]) of every tensor.
// The prefixes are built on the device by run_varlen_prep.
struct Varlen {
  const int* cu_seqlens;   // device [batch + 1]
  const int* tile_pfx;     // device [batch + 1]: prefix of ceil(L_s / 128) (index query tiles)
  const int* blk_pfx;      // device [batch + 1]: prefix of ceil(L_s / B_k) (KV blocks)
  const int* topk_seq;     // device [batch] per-sequence k (index branch only), or null
  int batch;
};

// Device status word value for a packed batch whose cu_seqlens is not a
// valid prefix (cu[0] = 0, non-decreasing, cu[batch] = total rows).
constexpr int kDevBadInput = 2;

// Builds tile_pfx and blk_pfx from cu_seqlens (one CTA); an invalid
// cu_seqlens sets the status word and zero prefixes, so no sequence has work.
int run_varlen_prep(const int* cu_seqlens, int batch, int total, int block_k, int* tile_pfx, int* blk_pfx,
                    int* status, cudaStream_t stream);

int run_index_topk_prefill(const msa_params& p, const void* q_idx, const void* k_idx, int n_q, int n_kv,
                           int q_pos0, int32_t* block_ids, int* status, cudaStream_t stream,
                           const Varlen* vl = nullptr);

// Index projections (index_project.cu): q_idx [n, h_kv, d_idx] and
// k_idx [n, 1, d_idx] from x [n, d_model] and the stacked weight
// [(h_kv + 1) d_idx, d_model].
int run_index_project(const msa_params& p, const void* x, const void* w_idx, int n, int d_model, void* q_idx,
                      void* k_idx, int* status, cudaStream_t stream);

// The varlen entry points (varlen.cu): workspace bytes (header included) and
// the run of MSA_OP_INDEX_TOPK_VARLEN (a0, a1 = q_idx, k_idx; ids_out) or
// MSA_OP_PREFILL_VARLEN (a0, a1, a2 = q, k, v; ids_in; o).
size_t varlen_workspace_bytes(int op, const msa_params& p, int batch, int total);
int run_varlen(int op, const msa_params& p, const void* a0, const void* a1, const void* a2, const int32_t* cu,
               int batch, int total, const int32_t* topk_seq, const int32_t* ids_in, int32_t* ids_out, void* o,
               void* ws, size_t ws_bytes, cudaStream_t stream);

// Prefill main branch.  ws/ws_bytes: the op's workspace after the header.
// batch > 0: a packed batch of that many sequences (n_q = n_kv = total rows).
size_t prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv, int batch = 0);
int run_sparse_attn_prefill(const msa_params& p, const void* q, const void* k, const void* v,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream, const Varlen* vl = nullptr);

// Block-major sparse prefill (attn_sparse.cu).
size_t sparse_prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv, int batch);
// False when the block-major schedule's 32-bit list, entry or partial-row
// indices would overflow (huge n_q * h_kv * topk or lists).
bool sparse_sizes_supported(const msa_params& p, int n_q, int n_kv, int batch);
int run_sparse_attn_kvouter(const msa_params& p, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream, const Varlen* vl);

// Decode step.
// Limits of the decode kernels (checked on the host before any launch).
constexpr int kDecodeMaxGroups = 8;     // h_kv: one index-scan warp per group
constexpr int kDecodeMaxBatch = 4096;   // sparse: the block prefix of every sequence in shared memory
size_t decode_counter_bytes(const msa_params& p, int batch);
// MXFP8 decode caches (E4M3 codes with E8M0 scales per 32 elements), or null
// in run_sparse_attn_decode for the bf16 caches.
struct DecodeMx8 {
  const void *k8, *k_sc, *v8, *v_sc;        // [sum L, h_kv, d] codes, [sum L, h_kv, d / 32] scales
  const void *k_idx8, *k_idx_sc;            // [sum L, 1, d_idx] codes, [sum L, 1, d_idx / 32] scales
};
// dense: 1 = the dense run, 0 = the sparse run, -1 = the larger of the two.
size_t decode_workspace_bytes(const msa_params& p, int batch, int max_kv, int dense);
int run_sparse_attn_decode(const msa_params& p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t ws_bytes,
                           int* status, cudaStream_t stream, const int32_t* topk_seq = nullptr,
                           const DecodeMx8* mx8 = nullptr);

// MSA_OPT_DECODE_FUSED (msa_set_option).
extern std::atomic<int> g_decode_fused;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace msa
