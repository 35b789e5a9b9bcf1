// varlen.cu -- packed batches of independent prefills (cu_seqlens): the
// serving-shaped form of the prefill, many sequences of different lengths in
// one call.  Every kernel of the single-sequence path runs unchanged in
// structure; this file builds the per-sequence prefixes they read and holds
// the two entry points.
//
// Sequence s owns rows [cu_seqlens[s], cu_seqlens[s + 1]) of Q_idx, K_idx, Q,
// K, V, O and the block ids; its positions restart at 0, and its block ids
// are local to it (block b holds its keys [b B_k, (b + 1) B_k)).  Each
// sequence is the problem of the titansim.online summary of "MiniMax Sparse
// Attention" (eq. (6) and the top-k rule of section 4.2, eq. (8) of section
// 4.3) on its own rows.
#include <cstdint>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kPrepThreads = 1024;

// One CTA: exclusive prefixes of ceil(L_s / 128) (query tiles of the index
// kernel) and ceil(L_s / B_k) (KV blocks), and a validity check of cu_seqlens.
__global__ void __launch_bounds__(kPrepThreads) varlen_prep_kernel(const int* cu, int batch, int total, int block_k,
                                                                   int* tile_pfx, int* blk_pfx, int* status) {
  __shared__ int bad;
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    bad = (cu[0] != 0 || cu[batch] != total) ? 1 : 0;
    carry[0] = carry[1] = 0;
  }
  __syncthreads();
  for (int base = 0; base < batch; base += kPrepThreads) {
    const int s = base + threadIdx.x;
    int nt = 0, nbk = 0;
    if (s < batch) {
      const int L = cu[s + 1] - cu[s];
      if (L < 0) {
        bad = 1;
      } else {
        nt = (L + 127) / 128;
        nbk = (L + block_k - 1) / block_k;
      }
    }
    int a = nt, b = nbk;   // inclusive warp scans
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int xa = __shfl_up_sync(0xffffffffu, a, off), xb = __shfl_up_sync(0xffffffffu, b, off);
      if (lane >= off) {
        a += xa;
        b += xb;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = a;
      wsum[1][warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
      int x = wsum[0][lane], y = wsum[1][lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int xa = __shfl_up_sync(0xffffffffu, x, off), xb = __shfl_up_sync(0xffffffffu, y, off);
        if (lane >= off) {
          x += xa;
          y += xb;
        }
      }
      wsum[0][lane] = x;
      wsum[1][lane] = y;
    }
    __syncthreads();
    if (s < batch) {
      tile_pfx[s] = carry[0] + (warp ? wsum[0][warp - 1] : 0) + a - nt;
      blk_pfx[s] = carry[1] + (warp ? wsum[1][warp - 1] : 0) + b - nbk;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry[0] += wsum[0][31];
      carry[1] += wsum[1][31];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    tile_pfx[batch] = carry[0];
    blk_pfx[batch] = carry[1];
  }
  __syncthreads();
  if (bad) {   // no sequence gets any work; the caller learns it from the status word
    for (int s = threadIdx.x; s <= batch; s += kPrepThreads) {
      tile_pfx[s] = 0;
      blk_pfx[s] = 0;
    }
    if (threadIdx.x == 0) atomicExch(status, kDevBadInput);
  }
}

// Workspace after the header: tile_pfx, blk_pfx, then (prefill) the
// block-major schedule and partials.
size_t prefix_bytes(int batch) { return 2 * align_up(static_cast<size_t>(batch + 1) * 4, 256); }

}  // namespace

int run_varlen_prep(const int* cu_seqlens, int batch, int total, int block_k, int* tile_pfx, int* blk_pfx,
                    int* status, cudaStream_t stream) {
  varlen_prep_kernel<<<1, kPrepThreads, 0, stream>>>(cu_seqlens, batch, total, block_k, tile_pfx, blk_pfx, status);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

size_t varlen_workspace_bytes(int op, const msa_params& p, int batch, int total) {
  if (op == MSA_OP_INDEX_TOPK_VARLEN) return kWsHeader + prefix_bytes(batch);
  return kWsHeader + prefix_bytes(batch) + align_up(prefill_workspace_bytes(p, total, total, batch), 256);
}

int run_varlen(int op, const msa_params& p, const void* a0, const void* a1, const void* a2, const int32_t* cu,
               int batch, int total, const int32_t* topk_seq, const int32_t* ids_in, int32_t* ids_out, void* o,
               void* ws, size_t ws_bytes, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  Varlen vl;
  vl.cu_seqlens = cu;
  vl.tile_pfx = reinterpret_cast<int*>(w + kWsHeader);
  vl.blk_pfx = reinterpret_cast<int*>(w + kWsHeader + prefix_bytes(batch) / 2);
  vl.topk_seq = topk_seq;
  vl.batch = batch;
  int* status = static_cast<int*>(ws);
  int rc = run_varlen_prep(cu, batch, total, p.block_k, const_cast<int*>(vl.tile_pfx), const_cast<int*>(vl.blk_pfx),
                           status, stream);
  if (rc || total == 0) return rc;
  if (op == MSA_OP_INDEX_TOPK_VARLEN)
    return run_index_topk_prefill(p, a0, a1, total, total, 0, ids_out, status, stream, &vl);
  const size_t off = kWsHeader + prefix_bytes(batch);
  return run_sparse_attn_prefill(p, a0, a1, a2, ids_in, total, total, 0, o, w + off, ws_bytes - off, status, stream,
                                 &vl);
}

}  // namespace msa
