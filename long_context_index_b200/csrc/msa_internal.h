// msa_internal.h -- declarations shared by the library's translation units.
#pragma once
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

int run_index_topk_prefill(const msa_params& p, const void* q_idx, const void* k_idx, int n_q, int n_kv,
                           int q_pos0, int32_t* block_ids, int* status, cudaStream_t stream);

// Prefill main branch.  ws/ws_bytes: the op's workspace after the header.
size_t prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv);
int run_sparse_attn_prefill(const msa_params& p, const void* q, const void* k, const void* v,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream);

// Block-major sparse prefill (attn_sparse.cu).
size_t sparse_prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv);
int run_sparse_attn_kvouter(const msa_params& p, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream);

// Decode step.
// Limits of the decode kernels (checked on the host before any launch).
constexpr int kDecodeMaxGroups = 8;     // h_kv: one index-scan warp per group
constexpr int kDecodeMaxBatch = 4096;   // sparse: the block prefix of every sequence in shared memory
size_t decode_counter_bytes(const msa_params& p, int batch);
// dense: 1 = the dense run, 0 = the sparse run, -1 = the larger of the two.
size_t decode_workspace_bytes(const msa_params& p, int batch, int max_kv, int dense);
int run_sparse_attn_decode(const msa_params& p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t ws_bytes,
                           int* status, cudaStream_t stream);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace msa
