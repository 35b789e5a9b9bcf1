// attn_prefill.cu -- main branch of a (chunked) prefill on sm_100a: the
// dispatch between the sparse (block-major, attn_sparse.cu) and the dense
// path, and the dense kernel itself.
//
// The dense run computes eq. (1) of the titansim.online summary of "MiniMax
// Sparse Attention" (section 2.2) for GQA: for every query row i and head h of
// group r = h / G,
//   O_i^(h) = softmax( Q_i^(h) K^(r)[0..p_i]^T / sqrt(d) ) V^(r)[0..p_i],
// i.e. eq. (8) with every causal block selected.  It is the baseline the
// sparse path is measured against.  A block-major (KV-outer) pass over every
// block would write one partial per (query, block) -- at 128K that is 2 TB --
// so the dense run keeps the query as the outer loop.
//
// Kernel design (query-outer, GQA-packed):
//   * One CTA owns a 128-row tile = QT = 128/G consecutive queries x the G
//     heads of one group.  All rows share each K/V block, so one 128-key block
//     staged by TMA feeds a full M = 128 UMMA (the heads of a group share the
//     block selection: "同一 GQA 分组内的所有 Query 头共享相同的检索结果",
//     titansim.online section 1.2).
//   * warp 0: TMA producer (Q tile once; K and V blocks through a 2-deep ring).
//   * warp 1: UMMA issuer.  S_j = Q K_j^T (SS form) into one of two TMEM S
//     buffers; O += P_j V_j with P_j read from TMEM (TS form) and V_j as an
//     MN-major shared-memory operand.
//   * warps 4..7: softmax + epilogue, one thread per TMEM lane (= row).  Online
//     softmax in fp32 with base-2 exponentials; O is rescaled in TMEM only when
//     the running max grows by more than 2^8 (otherwise P may exceed 1 by at
//     most 256, which fp32 accumulation absorbs).  P is written back to TMEM as
//     bf16 over the S buffer it came from.
//   * A tile walks every block up to its last query's position; a row masks
//     the keys after its own position.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kThreads = 256;   // 8 warps
constexpr int kSoftWarp0 = 4;   // softmax warps 4..7
constexpr int kStages = 2;      // K/V ring depth
constexpr float kRescaleLog2 = 8.0f;

template <int D, int BK>
struct AttnCfg {
  static constexpr int kAtoms = D / 64;                    // 128-byte swizzle atoms along d
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = BK * D * 2;
  static constexpr int kSmemData = kQBytes + kStages * 2 * kKVBytes;
  static constexpr int kSmemBytes = kSmemData + 4096 + 1024;
  static constexpr int kTmemCols = (2 * BK + D) <= 256 ? 256 : 512;
  static constexpr int kColS0 = 0;
  static constexpr int kColS1 = BK;
  static constexpr int kColO = 2 * BK;
};

struct AttnArgs {
  uint16_t* o;               // [n_q, h_q, d]
  int* status;
  int n_q, n_kv, q_pos0, h_q, h_kv, causal;
  int n_qtiles;
  float scale_log2;          // softmax scale * log2(e)
};

template <int D, int BK, int G>
__global__ void __launch_bounds__(kThreads, 1)
    attn_qouter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
  using Cfg = AttnCfg<D, BK>;
  constexpr int QT = 128 / G;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;                                   // [atoms][128 rows][128 B]
  uint8_t* skv = smem + Cfg::kQBytes;                   // [stage][K|V][atoms][BK rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kSmemData);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                         // [kStages]
  uint64_t* kv_empty = kv_full + kStages;               // [kStages]
  uint64_t* s_full = kv_empty + kStages;                // [2]
  uint64_t* s_free = s_full + 2;                        // [2]
  uint64_t* p_full = s_free + 2;                        // [2]
  uint64_t* o_done = p_full + 2;                        // one phase per PV
  uint64_t* o_final = o_done + 1;                       // the last PV only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int qtile = args.n_qtiles - 1 - static_cast<int>(blockIdx.x) / args.h_kv;  // heavy tiles first
  const int r = static_cast<int>(blockIdx.x) % args.h_kv;
  const int i0 = qtile * QT;
  const int q_here = min(QT, args.n_q - i0);

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 1);
      mbar_init(&p_full[b], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  // Blocks of the tile: every block up to its last query's position.
  const int p_last = args.q_pos0 + i0 + q_here - 1;
  const int nb_total = (args.n_kv + BK - 1) / BK;
  const int nblk = args.causal ? min(p_last / BK + 1, nb_total) : nb_total;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, args.status};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
      for (int a = 0; a < Cfg::kAtoms; ++a) tma_load_3d(sq + a * 128 * 128, &tm_q, q_full, a * 64, r * G, i0);
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kStages;
        const int b = j;
        if (!mbar_wait(&kv_empty[s], ((j / kStages) & 1) ^ 1, wc)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * Cfg::kKVBytes);
        uint8_t* sk = skv + s * 2 * Cfg::kKVBytes;
        uint8_t* sv = sk + Cfg::kKVBytes;
        for (int a = 0; a < Cfg::kAtoms; ++a) {
          tma_load_3d(sk + a * BK * 128, &tm_k, &kv_full[s], a * 64, r, b * BK);
          tma_load_3d(sv + a * BK * 128, &tm_v, &kv_full[s], a * 64, r, b * BK);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA
    // The whole warp runs the loop (warp-uniform waits and descriptor math)
    // and one elected lane issues: a divergent single-lane issue loop loses
    // most of its issue slots to the softmax warps sharing this SMSP.
    if (nblk > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BK, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      // Descriptors differ only in their start-address field (address >> 4,
      // bits 0-13): a base plus an offset.
      const uint64_t q_desc0 = smem_desc(smem_u32(sq), 16, 1024, kSwizzle128B);
      const uint64_t k_desc0 = smem_desc(smem_u32(skv), 16, 1024, kSwizzle128B);
      const uint64_t v_desc0 = smem_desc(smem_u32(skv) + Cfg::kKVBytes, BK * 128, 1024, kSwizzle128B);
      bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, wc));
      auto issue_pv = [&](int j) -> bool {
        const int s = j % kStages;
        const int sb = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&p_full[sb], (j >> 1) & 1, wc))) return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + ((s * 2 * Cfg::kKVBytes) >> 4);
        const uint32_t p_tmem = tmem + (sb ? Cfg::kColS1 : Cfg::kColS0);
        const bool leader = elect_one();
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // B = V block, MN-major: 16 keys per step = 2048 bytes; d atoms are BK*128 bytes apart.
          if (leader)
            umma_ts(tmem + Cfg::kColO, p_tmem + kk * 8, vd + ((kk * 2048) >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (leader) {
          umma_commit(&kv_empty[s]);
          umma_commit(&s_free[sb]);
          umma_commit(o_done);
        }
        __syncwarp();
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % kStages;
        const int sb = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&kv_full[s], (j / kStages) & 1, wc))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_free[sb], ((j >> 1) & 1) ^ 1, wc))) break;
        tc_fence_after();
        const uint64_t kd = k_desc0 + ((s * 2 * Cfg::kKVBytes) >> 4);
        const bool leader = elect_one();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t aoff = ((ks / 4) * 128 * 128 + (ks % 4) * 32) >> 4;
          const uint32_t boff = ((ks / 4) * BK * 128 + (ks % 4) * 32) >> 4;
          if (leader)
            umma_ss(tmem + (sb ? Cfg::kColS1 : Cfg::kColS0), q_desc0 + aoff, kd + boff, idesc_s, ks > 0 ? 1u : 0u);
        }
        if (leader) umma_commit(&s_full[sb]);
        __syncwarp();
        if (j > 0 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) {
        const bool done = issue_pv(nblk - 1);
        const bool leader = elect_one();   // the same lane that issued the MMAs
        if (done && leader) umma_commit(o_final);
        __syncwarp();
      }
    }
  } else if (warp >= kSoftWarp0) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qi = row / G;
    const int hh = row % G;
    const bool row_ok = qi < q_here;
    const int p = args.q_pos0 + i0 + qi;
    const int kv_lim = row_ok ? (args.causal ? min(p + 1, args.n_kv) : args.n_kv) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = args.scale_log2;
    float m_run = __int_as_float(0xff800000);  // running max of raw scores (-inf)
    float l_run = 0.f;

    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      const int kb0 = j * BK;
      const int lim = row_ok ? min(BK, kv_lim - kb0) : 0;   // valid keys of this block for the row
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, wc)) break;
      tc_fence_after();
      uint32_t sv[BK];
      const uint32_t s_tmem = lane_base + (sb ? Cfg::kColS1 : Cfg::kColS0);
#pragma unroll
      for (int cch = 0; cch < BK / 32; ++cch)
        tmem_ld32(s_tmem + cch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[cch * 32]));
      tmem_ld_wait();
      float mx = __int_as_float(0xff800000);
      if (lim >= BK) {
#pragma unroll
        for (int e = 0; e + 2 < BK; e += 3)
          mx = max3f(mx, __uint_as_float(sv[e]), fmaxf(__uint_as_float(sv[e + 1]), __uint_as_float(sv[e + 2])));
        if (BK % 3 != 0) {
#pragma unroll
          for (int e = (BK / 3) * 3; e < BK; ++e) mx = fmaxf(mx, __uint_as_float(sv[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < BK; ++e) {
          const float v = e < lim ? __uint_as_float(sv[e]) : __int_as_float(0xff800000);
          sv[e] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      // Lazy rescale: only when the max grows by more than 2^kRescaleLog2.
      const bool grow = m_run != __int_as_float(0xff800000) && (m_new - m_run) * c > kRescaleLog2;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2_approx((m_run - m_new) * c);
        l_run *= alpha;
        m_run = m_new;
      } else if (m_run == __int_as_float(0xff800000)) {
        m_run = m_new;   // first visible keys: O and l are still exactly zero
      }
      if (__any_sync(0xffffffffu, grow)) {
        // O must hold every PV up to block j-1 before it is rescaled.  Here
        // PV_{j-2} is complete (it was issued before S_j) and PV_j is not yet
        // issued, so the PV barrier is at most one phase from phase j-1.
        if (!mbar_wait(o_done, (j - 1) & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int cch = 0; cch < D / 32; ++cch) {
          uint32_t ov[32];
          tmem_ld32(lane_base + Cfg::kColO + cch * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(lane_base + Cfg::kColO + cch * 32, ov);
        }
        tmem_st_wait();
      }
      const float bias = m_run == __int_as_float(0xff800000) ? 0.f : m_run * c;
      float lsum = 0.f;
      uint32_t pk[BK / 2];
#pragma unroll
      for (int e = 0; e < BK; e += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c, -bias));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c, -bias));
        lsum += p0 + p1;
        pk[e / 2] = pack_bf16x2(p0, p1);
      }
      l_run += lsum;
#pragma unroll
      for (int cch = 0; cch < BK / 64; ++cch)
        tmem_st32(s_tmem + cch * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[cch * 32]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }

    // Epilogue: O / l -> bf16.  (The PV barrier may run up to two phases
    // ahead of this point, so the last PV signals a barrier of its own.)
    bool ok = !*abort_flag && nblk > 0;
    if (ok) ok = mbar_wait(o_final, 0, wc);
    if (ok) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint16_t* orow = args.o + (static_cast<size_t>(i0 + qi) * args.h_q + r * G + hh) * D;
#pragma unroll
      for (int cch = 0; cch < D / 32; ++cch) {
        uint32_t ov[32];
        tmem_ld32(lane_base + Cfg::kColO + cch * 32, ov);
        tmem_ld_wait();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[v4 * 8 + 0]) * inv, __uint_as_float(ov[v4 * 8 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ov[v4 * 8 + 2]) * inv, __uint_as_float(ov[v4 * 8 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ov[v4 * 8 + 4]) * inv, __uint_as_float(ov[v4 * 8 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ov[v4 * 8 + 6]) * inv, __uint_as_float(ov[v4 * 8 + 7]) * inv);
            dst[v4] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) __nanosleep(1000000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

template <int D, int BK, int G>
cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                        cudaStream_t st) {
  auto kern = attn_qouter_kernel<D, BK, G>;
  const int smem = AttnCfg<D, BK>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<a.n_qtiles * a.h_kv, kThreads, smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_g(int G, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                     cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn<D, BK, 1>(tq, tk, tv, a, st);
    case 2: return launch_attn<D, BK, 2>(tq, tk, tv, a, st);
    case 4: return launch_attn<D, BK, 4>(tq, tk, tv, a, st);
    case 8: return launch_attn<D, BK, 8>(tq, tk, tv, a, st);
    case 16: return launch_attn<D, BK, 16>(tq, tk, tv, a, st);
    case 32: return launch_attn<D, BK, 32>(tq, tk, tv, a, st);
    case 64: return launch_attn<D, BK, 64>(tq, tk, tv, a, st);
    default: return launch_attn<D, BK, 128>(tq, tk, tv, a, st);
  }
}

}  // namespace

size_t prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv, int batch) {
  return sparse_prefill_workspace_bytes(p, n_q, n_kv, batch);
}

int run_sparse_attn_prefill(const msa_params& p, const void* q, const void* k, const void* v,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream, const Varlen* vl) {
  if (n_q == 0) return MSA_OK;
  const int G = p.h_q / p.h_kv;
  const int QT = 128 / G;
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.h_q), static_cast<uint64_t>(n_q)};
    const uint64_t strides[2] = {static_cast<uint64_t>(p.d) * 2, static_cast<uint64_t>(p.h_q) * p.d * 2};
    const uint32_t box[3] = {64, static_cast<uint32_t>(G), static_cast<uint32_t>(QT)};
    if (!encode_tma_bf16(&tq, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.h_kv),
                              static_cast<uint64_t>(n_kv)};
    const uint64_t strides[2] = {static_cast<uint64_t>(p.d) * 2, static_cast<uint64_t>(p.h_kv) * p.d * 2};
    const uint32_t box[3] = {64, 1, static_cast<uint32_t>(p.block_k)};
    if (!encode_tma_bf16(&tk, 3, k, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
    if (!encode_tma_bf16(&tv, 3, v, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  if (block_ids)   // sparse: block-major schedule (attn_sparse.cu)
    return run_sparse_attn_kvouter(p, q, tk, tv, block_ids, n_q, n_kv, q_pos0, o, ws, ws_bytes, status, stream, vl);
  if (vl) return MSA_ERR_INVALID;   // packed batches run sparse only
  AttnArgs a;
  a.o = static_cast<uint16_t*>(o);
  a.status = status;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.q_pos0 = q_pos0;
  a.h_q = p.h_q;
  a.h_kv = p.h_kv;
  a.causal = p.causal;
  a.n_qtiles = (n_q + QT - 1) / QT;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf(static_cast<float>(p.d));
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e;
  if (p.d == 64) {
    e = p.block_k == 64 ? launch_g<64, 64>(G, tq, tk, tv, a, stream) : launch_g<64, 128>(G, tq, tk, tv, a, stream);
  } else {
    e = p.block_k == 64 ? launch_g<128, 64>(G, tq, tk, tv, a, stream) : launch_g<128, 128>(G, tq, tk, tv, a, stream);
  }
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace msa
