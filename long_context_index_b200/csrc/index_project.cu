// index_project.cu -- the index projections ahead of the index branch, on
// sm_100a tensor cores.
//
// The titansim.online summary of "MiniMax Sparse Attention" (section 4.2)
// gives the index branch its own index-query projection per GQA group and one
// index-key projection shared by all groups; the m.163.com post ("Step 1 Index
// Attention") gives the shapes Q_idx in R^{n x h x d}, K_idx in R^{n x 1 x d}.
// With the stacked weight W = [W_q^idx(0); ...; W_q^idx(h_kv - 1); W_k^idx]
// ((h_kv + 1) d_idx rows of d_model, nn.Linear layout) both are one GEMM:
//   Y[i, c] = sum_t x[i, t] W[c, t],   c < h_kv d_idx -> Q_idx[i, c / d_idx, c % d_idx],
//                                      c >= h_kv d_idx -> K_idx[i, 0, c - h_kv d_idx].
// fp32 accumulation in TMEM, rounded to bf16 (nearest even) on the way out.
//
// Design: persistent grid over 128-row tiles of x; each tile's output columns
// (at most 512 per pass, all of them for h_kv = 4, d_idx = 64) accumulate in
// TMEM as two N = NH halves, so x is read from HBM once per pass while the
// stacked weight (a few MB) stays in L2.  warp 0 streams 64-column K-slices
// of x and W by TMA through a shared-memory ring; warp 1 issues the two
// 128 x NH x 16 tcgen05.mma per 16 columns of K; warps 4..7 (one TMEM lane
// quarter each, one row per thread) convert and store a finished tile while
// the next tile's K-slices are already loading.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kThreads = 256;     // 8 warps
constexpr int kEpiW0 = 4;         // epilogue warps 4..7
constexpr int kKSlice = 64;       // K columns per stage (one 128-byte swizzle atom)
constexpr int kABytes = 128 * 128;   // 128 rows x 128 bytes
constexpr int kSmemBudget = 200 * 1024;

struct ProjArgs {
  uint16_t* q_idx;   // [n, h_kv * d_idx]
  uint16_t* k_idx;   // [n, d_idx]
  int* status;
  int n, d_model, nq_cols, d_idx;   // nq_cols = h_kv * d_idx
  int col0, nh;                     // this pass: output columns [col0, col0 + 2 nh)
  int stages, n_tiles;
};

__global__ void __launch_bounds__(kThreads, 1)
    index_project_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const ProjArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b_bytes = 2 * a.nh * 128;                 // both halves of the weight slice
  const int stage_bytes = kABytes + b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.stages * stage_bytes);
  uint64_t* full = bars;                              // [stages]
  uint64_t* empty = full + a.stages;                  // [stages]
  uint64_t* acc_full = empty + a.stages;              // [1]
  uint64_t* acc_empty = acc_full + 1;                 // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status};
  const int n_k = (a.d_model + kKSlice - 1) / kKSlice;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
      int it = 0;
      for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
        for (int kk = 0; kk < n_k; ++kk, ++it) {
          const int s = it % a.stages;
          if (!mbar_wait(&empty[s], ((it / a.stages) & 1) ^ 1, wc)) goto done;
          uint8_t* st = smem + s * stage_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          tma_load_2d(st, &tm_x, &full[s], kk * kKSlice, tile * 128);
          tma_load_2d(st + kABytes, &tm_w, &full[s], kk * kKSlice, a.col0);
          tma_load_2d(st + kABytes + a.nh * 128, &tm_w, &full[s], kk * kKSlice, a.col0 + a.nh);
        }
      }
    }
  done:;
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (whole warp, elected lane)
    const uint32_t idesc = idesc_bf16_f32(128, a.nh, false, false);
    const uint64_t desc0 = smem_desc(smem_u32(smem), 16, 1024, kSwizzle128B);
    int it = 0, ti = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++ti) {
      // The single accumulator is free once the epilogue has read the previous tile.
      if (!__all_sync(0xffffffffu, mbar_wait(acc_empty, (ti & 1) ^ 1, wc))) break;
      tc_fence_after();
      for (int kk = 0; kk < n_k; ++kk, ++it) {
        const int s = it % a.stages;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / a.stages) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = desc0 + ((s * stage_bytes) >> 4);
        const uint64_t bd = ad + (kABytes >> 4);
#pragma unroll
        for (int ks = 0; ks < kKSlice / 16; ++ks) {
          const uint32_t acc = (kk > 0 || ks > 0) ? 1u : 0u;
          umma_ss_elect(tmem, ad + ks * 2, bd + ks * 2, idesc, acc);
          umma_ss_elect(tmem + a.nh, ad + ks * 2, bd + ((a.nh * 128) >> 4) + ks * 2, idesc, acc);
        }
        umma_commit_elect(&empty[s]);   // the stage is free once these MMAs have read it
      }
      if (ok) umma_commit_elect(acc_full);
      __syncwarp();
    }
  } else if (warp >= kEpiW0) {
    // ---------------------------------------------------------------- epilogue: TMEM -> bf16 -> Q_idx / K_idx
    const int quarter = warp & 3;
    const int row_in = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int ti = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++ti) {
      if (!mbar_wait(acc_full, ti & 1, wc)) break;
      tc_fence_after();
      const int row = tile * 128 + row_in;
      for (int c0 = 0; c0 < 2 * a.nh; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_base + c0, v);
        tmem_ld_wait();
        if (row < a.n) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          // 32 columns never straddle the Q_idx / K_idx boundary (both are
          // multiples of 32 columns).
          const int c = a.col0 + c0;
          uint16_t* dst = c < a.nq_cols ? a.q_idx + static_cast<size_t>(row) * a.nq_cols + c
                                        : a.k_idx + static_cast<size_t>(row) * a.d_idx + (c - a.nq_cols);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) __nanosleep(1000000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int run_index_project(const msa_params& p, const void* x, const void* w_idx, int n, int d_model, void* q_idx,
                      void* k_idx, int* status, cudaStream_t stream) {
  if (n == 0) return MSA_OK;
  const int n_cols = (p.h_kv + 1) * p.d_idx;
  CUtensorMap tx;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(d_model), static_cast<uint64_t>(n)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d_model) * 2};
    const uint32_t box[2] = {kKSlice, 128};
    if (!encode_tma_bf16(&tx, 2, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ProjArgs a;
  a.q_idx = static_cast<uint16_t*>(q_idx);
  a.k_idx = static_cast<uint16_t*>(k_idx);
  a.status = status;
  a.n = n;
  a.d_model = d_model;
  a.nq_cols = p.h_kv * p.d_idx;
  a.d_idx = p.d_idx;
  a.n_tiles = (n + 127) / 128;
  const int grid = a.n_tiles < sms ? a.n_tiles : sms;
  // Passes of at most 512 output columns (the TMEM width), split into two
  // equal MMA halves (each a multiple of 16 columns, at most 256).
  for (int col0 = 0; col0 < n_cols; col0 += 512) {
    const int np = n_cols - col0 < 512 ? n_cols - col0 : 512;
    a.col0 = col0;
    a.nh = np / 2;
    CUtensorMap tw;
    const uint64_t dims[2] = {static_cast<uint64_t>(d_model), static_cast<uint64_t>(n_cols)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d_model) * 2};
    const uint32_t box[2] = {kKSlice, static_cast<uint32_t>(a.nh)};
    if (!encode_tma_bf16(&tw, 2, w_idx, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
    const int stage_bytes = kABytes + 2 * a.nh * 128;
    a.stages = kSmemBudget / stage_bytes;
    if (a.stages > 6) a.stages = 6;
    const int smem = a.stages * stage_bytes + 256 + 1024;
    if (cudaFuncSetAttribute(index_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return MSA_ERR_CUDA;
    index_project_kernel<<<grid, kThreads, smem, stream>>>(tx, tw, a);
    if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;
  }
  return MSA_OK;
}

}  // namespace msa
