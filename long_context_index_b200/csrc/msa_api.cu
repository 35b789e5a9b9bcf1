// msa_api.cu -- host side of the C ABI declared in include/msa.h: argument
// validation, workspace sizing and layout, the device status word, TMA
// descriptor encoding, and dispatch to the kernels.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"

namespace msa {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxRows = 1 << 24;

int check_params(const msa_params* p) {
  if (!p) return MSA_ERR_INVALID;
  if (p->h_q <= 0 || p->h_kv <= 0 || p->d <= 0 || p->d_idx <= 0 || p->block_k <= 0 || p->topk <= 0)
    return MSA_ERR_INVALID;
  if ((p->causal != 0 && p->causal != 1) || (p->force_local != 0 && p->force_local != 1)) return MSA_ERR_INVALID;
  if (p->pool != 0 && p->pool != 1) return MSA_ERR_INVALID;
  if (p->h_q % p->h_kv != 0) return MSA_ERR_UNSUPPORTED;
  const int g = p->h_q / p->h_kv;
  if (g > 128 || 128 % g != 0) return MSA_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return MSA_ERR_UNSUPPORTED;
  if (p->d_idx != 32 && p->d_idx != 64 && p->d_idx != 128) return MSA_ERR_UNSUPPORTED;
  if (p->block_k != 64 && p->block_k != 128) return MSA_ERR_UNSUPPORTED;
  if (p->topk > 32) return MSA_ERR_UNSUPPORTED;
  if (!(p->scale <= 0.0f || std::isfinite(p->scale))) return MSA_ERR_INVALID;
  return MSA_OK;
}

int check_rows(int n_q, int n_kv, int q_pos0) {
  if (n_q < 0 || n_kv <= 0 || q_pos0 < 0) return MSA_ERR_INVALID;
  if (n_q > kMaxRows || n_kv > kMaxRows) return MSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(q_pos0) + n_q > n_kv) return MSA_ERR_INVALID;
  return MSA_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return MSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MSA_ERR_MISALIGNED;
  if (ws_bytes < need) return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

int clear_status(void* ws, cudaStream_t st) {
  return cudaMemsetAsync(ws, 0, sizeof(int), st) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

}  // namespace

static bool encode_tma(CUtensorMapDataType type, CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides[i];
  CUresult r = fn(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d,
                  s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tma_bf16(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                     const uint32_t* box, CUtensorMapSwizzle swizzle) {
  return encode_tma(CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, map, rank, base, dims, strides, box, swizzle);
}

bool encode_tma_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                   const uint32_t* box, CUtensorMapSwizzle swizzle) {
  return encode_tma(CU_TENSOR_MAP_DATA_TYPE_UINT8, map, rank, base, dims, strides, box, swizzle);
}

// The decode step's form; the two launches measured faster on the bench
// decode (64 sequences of 64K-128K tokens) than the one fused launch.
std::atomic<int> g_decode_fused{0};

}  // namespace msa

using namespace msa;

extern "C" {

size_t msa_workspace_size(int op, const msa_params* p, int n_q, int n_kv, int batch, int max_kv) {
  if (check_params(p) != MSA_OK) return 0;
  switch (op) {
    case MSA_OP_INDEX_TOPK:
      if (check_rows(n_q, n_kv, 0) != MSA_OK) return 0;
      return kWsHeader;
    case MSA_OP_PREFILL:
      if (check_rows(n_q, n_kv, 0) != MSA_OK) return 0;
      return kWsHeader + align_up(prefill_workspace_bytes(*p, n_q, n_kv), 256);
    case MSA_OP_DECODE:
      if (batch <= 0 || max_kv <= 0 || max_kv > kMaxRows) return 0;
      return kWsHeader + align_up(decode_workspace_bytes(*p, batch, max_kv, -1), 256);
    case MSA_OP_INDEX_PROJECT:
      if (n_q < 0 || n_q > kMaxRows) return 0;
      return kWsHeader;
    case MSA_OP_INDEX_TOPK_VARLEN:
    case MSA_OP_PREFILL_VARLEN:
      if (batch <= 0 || check_rows(n_q, n_q > 0 ? n_q : 1, 0) != MSA_OK) return 0;
      return varlen_workspace_bytes(op, *p, batch, n_q);
    default:
      return 0;
  }
}

int msa_index_project(const msa_params* p, const void* x, const void* w_idx, int n, int d_model, void* q_idx,
                      void* k_idx, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if (n < 0 || d_model <= 0) return MSA_ERR_INVALID;
  if (n > kMaxRows || d_model % 8 != 0 || d_model > (1 << 20)) return MSA_ERR_UNSUPPORTED;
  if ((rc = check_ws(ws, ws_bytes, kWsHeader))) return rc;
  if (n > 0 && (!x || !w_idx || !q_idx || !k_idx)) return MSA_ERR_INVALID;
  if (n > 0 && (!aligned16(x) || !aligned16(w_idx) || !aligned16(q_idx) || !aligned16(k_idx)))
    return MSA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(ws, st))) return rc;
  return run_index_project(*p, x, w_idx, n, d_model, q_idx, k_idx, static_cast<int*>(ws), st);
}

int msa_index_topk(const msa_params* p, const void* q_idx, const void* k_idx, int n_q, int n_kv, int q_pos0,
                   int32_t* block_ids, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_rows(n_q, n_kv, q_pos0))) return rc;
  if ((rc = check_ws(ws, ws_bytes, kWsHeader))) return rc;
  if (n_q > 0 && (!q_idx || !k_idx || !block_ids)) return MSA_ERR_INVALID;
  if (n_q > 0 && (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(block_ids))) return MSA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(ws, st))) return rc;
  return run_index_topk_prefill(*p, q_idx, k_idx, n_q, n_kv, q_pos0, block_ids, static_cast<int*>(ws), st);
}

int msa_sparse_attn_prefill(const msa_params* p, const void* q, const void* k, const void* v,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_rows(n_q, n_kv, q_pos0))) return rc;
  const size_t need = kWsHeader + align_up(prefill_workspace_bytes(*p, n_q, n_kv), 256);
  if ((rc = check_ws(ws, ws_bytes, need))) return rc;
  if (n_q > 0 && (!q || !k || !v || !o)) return MSA_ERR_INVALID;
  if (n_q > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))) return MSA_ERR_MISALIGNED;
  if (block_ids && !aligned16(block_ids)) return MSA_ERR_MISALIGNED;
  if (block_ids && n_q > 0 && !sparse_sizes_supported(*p, n_q, n_kv, 0)) return MSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(ws, st))) return rc;
  return run_sparse_attn_prefill(*p, q, k, v, block_ids, n_q, n_kv, q_pos0, o,
                                 static_cast<uint8_t*>(ws) + kWsHeader, ws_bytes - kWsHeader,
                                 static_cast<int*>(ws), st);
}

static int decode_call(const msa_params* p, const void* q, const void* q_idx, const void* k_cache, const void* v_cache,
                       const void* k_idx_cache, const int64_t* cu_kv, const int32_t* topk_per_seq, int batch,
                       int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t ws_bytes, void* stream,
                       const DecodeMx8* mx8) {
  int rc = check_params(p);
  if (rc) return rc;
  if (batch <= 0 || max_kv <= 0 || (dense != 0 && dense != 1)) return MSA_ERR_INVALID;
  if (max_kv > kMaxRows) return MSA_ERR_UNSUPPORTED;
  if (p->h_kv > kDecodeMaxGroups) return MSA_ERR_UNSUPPORTED;
  // Sparse: the block prefix of every sequence sits in shared memory, and TMA
  // row coordinates of the caches are 32-bit.
  if (!dense && (batch > kDecodeMaxBatch || static_cast<long long>(batch) * max_kv > 0x7fffffffLL))
    return MSA_ERR_UNSUPPORTED;
  // The call needs only the scratch of the run it makes (sparse or dense).
  const size_t need = kWsHeader + align_up(decode_workspace_bytes(*p, batch, max_kv, dense), 256);
  if ((rc = check_ws(ws, ws_bytes, need))) return rc;
  if (!q || !k_cache || !v_cache || !cu_kv || !o) return MSA_ERR_INVALID;
  if (!dense && (!q_idx || !k_idx_cache || !block_ids)) return MSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return MSA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(cu_kv) & 7u) != 0) return MSA_ERR_MISALIGNED;
  if (topk_per_seq && (reinterpret_cast<uintptr_t>(topk_per_seq) & 3u) != 0) return MSA_ERR_MISALIGNED;
  if (!dense && (!aligned16(q_idx) || !aligned16(k_idx_cache) || !aligned16(block_ids))) return MSA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // One memset clears the status word and the decode completion counters.
  if (cudaMemsetAsync(ws, 0, kWsHeader + decode_counter_bytes(*p, batch), st) != cudaSuccess) return MSA_ERR_CUDA;
  return run_sparse_attn_decode(*p, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, batch, max_kv, dense,
                                block_ids, o, static_cast<uint8_t*>(ws) + kWsHeader, ws_bytes - kWsHeader,
                                static_cast<int*>(ws), st, dense ? nullptr : topk_per_seq, mx8);
}

int msa_sparse_attn_decode_adaptive_k(const msa_params* p, const void* q, const void* q_idx, const void* k_cache,
                                      const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv,
                                      const int32_t* topk_per_seq, int batch, int max_kv, int dense,
                                      int32_t* block_ids, void* o, void* ws, size_t ws_bytes, void* stream) {
  return decode_call(p, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, topk_per_seq, batch, max_kv, dense,
                     block_ids, o, ws, ws_bytes, stream, nullptr);
}

int msa_sparse_attn_decode_mxfp8(const msa_params* p, const void* q, const void* q_idx, const void* k8,
                                 const void* k_scale, const void* v8, const void* v_scale, const void* k_idx8,
                                 const void* k_idx_scale, const int64_t* cu_kv, const int32_t* topk_per_seq, int batch,
                                 int max_kv, int32_t* block_ids, void* o, void* ws, size_t ws_bytes, void* stream) {
  const int rc = check_params(p);
  if (rc) return rc;
  if (p->d != 128) return MSA_ERR_UNSUPPORTED;
  if (!k8 || !k_scale || !v8 || !v_scale || !k_idx8 || !k_idx_scale) return MSA_ERR_INVALID;
  if (!aligned16(k8) || !aligned16(v8) || !aligned16(k_idx8)) return MSA_ERR_MISALIGNED;
  if (((reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale)) & 3u) != 0)
    return MSA_ERR_MISALIGNED;
  DecodeMx8 mx{k8, k_scale, v8, v_scale, k_idx8, k_idx_scale};
  // The bf16 cache arguments are unused: the MXFP8 codes stand in for them
  // (non-null placeholders for the shared validation).
  return decode_call(p, q, q_idx, k8, v8, k_idx8, cu_kv, topk_per_seq, batch, max_kv, 0, block_ids, o, ws,
                     ws_bytes, stream, &mx);
}


int msa_sparse_attn_decode(const msa_params* p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t ws_bytes,
                           void* stream) {
  return msa_sparse_attn_decode_adaptive_k(p, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, nullptr, batch, max_kv,
                                           dense, block_ids, o, ws, ws_bytes, stream);
}

namespace {
int varlen_call(int op, const msa_params* p, const void* a0, const void* a1, const void* a2, const int32_t* cu,
                int batch, int total, const int32_t* topk_seq, const int32_t* ids_in, int32_t* ids_out, void* o,
                void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if (batch <= 0 || total < 0 || !cu) return MSA_ERR_INVALID;
  if (total > kMaxRows || batch > kMaxRows) return MSA_ERR_UNSUPPORTED;
  if (op == MSA_OP_PREFILL_VARLEN && total > 0 && !sparse_sizes_supported(*p, total, total, batch))
    return MSA_ERR_UNSUPPORTED;
  if ((rc = check_ws(ws, ws_bytes, varlen_workspace_bytes(op, *p, batch, total)))) return rc;
  if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return MSA_ERR_MISALIGNED;
  if (topk_seq && (reinterpret_cast<uintptr_t>(topk_seq) & 3u) != 0) return MSA_ERR_MISALIGNED;
  if (total > 0) {
    if (!a0 || !a1 || (op == MSA_OP_PREFILL_VARLEN && (!a2 || !ids_in || !o)) ||
        (op == MSA_OP_INDEX_TOPK_VARLEN && !ids_out))
      return MSA_ERR_INVALID;
    if (!aligned16(a0) || !aligned16(a1) || (a2 && !aligned16(a2)) || (o && !aligned16(o)) ||
        (ids_in && !aligned16(ids_in)) || (ids_out && !aligned16(ids_out)))
      return MSA_ERR_MISALIGNED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(ws, st))) return rc;
  return run_varlen(op, *p, a0, a1, a2, cu, batch, total, topk_seq, ids_in, ids_out, o, ws, ws_bytes, st);
}
}  // namespace

int msa_index_topk_varlen(const msa_params* p, const void* q_idx, const void* k_idx, const int32_t* cu_seqlens,
                          int batch, int total, const int32_t* topk_per_seq, int32_t* block_ids, void* ws,
                          size_t ws_bytes, void* stream) {
  return varlen_call(MSA_OP_INDEX_TOPK_VARLEN, p, q_idx, k_idx, nullptr, cu_seqlens, batch, total, topk_per_seq,
                     nullptr, block_ids, nullptr, ws, ws_bytes, stream);
}

int msa_sparse_attn_prefill_varlen(const msa_params* p, const void* q, const void* k, const void* v,
                                   const int32_t* cu_seqlens, int batch, int total, const int32_t* block_ids,
                                   void* o, void* ws, size_t ws_bytes, void* stream) {
  return varlen_call(MSA_OP_PREFILL_VARLEN, p, q, k, v, cu_seqlens, batch, total, nullptr, block_ids, nullptr, o, ws,
                     ws_bytes, stream);
}

int msa_device_status(const void* ws, void* stream) {
  if (!ws) return MSA_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSA_ERR_CUDA;
  int s = 0;
  if (cudaMemcpy(&s, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MSA_ERR_CUDA;
  return s == kDevOk ? MSA_OK : (s == kDevBadInput ? MSA_ERR_INVALID : MSA_ERR_TIMEOUT);
}

int msa_set_option(int option, int value) {
  if (option != MSA_OPT_DECODE_FUSED || (value != 0 && value != 1)) return MSA_ERR_INVALID;
  msa::g_decode_fused.store(value);
  return MSA_OK;
}

int msa_get_option(int option) {
  if (option != MSA_OPT_DECODE_FUSED) return MSA_ERR_INVALID;
  return msa::g_decode_fused.load();
}

const char* msa_status_string(int status) {
  switch (status) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape";
    case MSA_ERR_MISALIGNED: return "misaligned pointer";
    case MSA_ERR_WORKSPACE: return "workspace too small";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
