// index_prefill.cu -- index branch of a (chunked) prefill on sm_100a.
//
// Computes, per query row i and GQA group r (titansim.online summary of
// "MiniMax Sparse Attention", eq. (6), section 4.2):
//   S_ij = <Q_idx_i^(r), K_idx_j>                  (the 1/sqrt(d_idx) factor is
//                                                   positive: order-preserving)
//   M_ib = max over visible j in block b of S_ij   (causal block max-pool;
//          with pool = mean, the mean over the visible keys of the block,
//          the MoBA-style pooling the m.163.com post compares it with)
//   I_i^(r) = local block + the best (topk - 1) other eligible blocks by M,
//             ties to the lower block index, emitted ascending, -1 padded.
// Selection compares raw scores and never exponentiates (section 4.4.1).
//
// Design (one CTA = 128 query rows x one group):
//   * warp 0, one lane: TMA producer.  Loads the Q_idx tile (A operand,
//     resident for the CTA) and streams 256-key K_idx tiles (B operand)
//     through an NST-deep shared-memory ring.
//   * warp 1, one lane: UMMA issuer.  Per key tile, one 128x256xd_idx
//     tcgen05.mma chain into one of two TMEM accumulator stages (2 x 256 fp32
//     columns = all 512 columns), so the MMA of tile t+1 overlaps the
//     epilogue of tile t.  N = 256 halves the MMA instructions per flop: the
//     issuing thread shares its SMSP's issue port with two epilogue warps,
//     and a contended issue slot costs more than the MMA itself.
//   * warps 4..11: epilogue.  Thread = (TMEM lane = query row, half of the
//     tile's 256 columns).  Reads its 128 columns of S from TMEM, masks
//     invisible keys, max-pools per block with 3-input max, and keeps a
//     register top-k list of the blocks in its halves (insertion only when
//     the candidate beats the current k-th score, so ties keep the earlier,
//     lower block).  At the end the two half-lists of a row are merged by
//     (score desc, block asc).  M is never written to memory.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;      // query rows per CTA (UMMA M)
constexpr int kKeys = 256;      // keys per tile (UMMA N)
constexpr int kThreads = 384;   // 12 warps
constexpr int kEpiWarp0 = 4;    // first epilogue warp
constexpr int kPoolMax = 0;     // msa_params.pool: block max-pool (eq. (6))
constexpr int kPoolMean = 1;    //                  block mean-pool (MoBA-style ablation)

template <int DIDX>
struct IdxCfg {
  static constexpr int kSwB = DIDX * 2 >= 128 ? 128 : DIDX * 2;   // swizzle span (bytes)
  static constexpr int kAtoms = DIDX * 2 / kSwB;                  // swizzle atoms along K
  static constexpr uint32_t kSwz = kSwB == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int kQBytes = kRows * DIDX * 2;                // the 128 x DIDX Q_idx tile
  static constexpr int kTileBytes = kKeys * DIDX * 2;             // one 256 x DIDX K_idx tile
  static constexpr int kStages = DIDX == 128 ? 2 : (DIDX == 64 ? 5 : 8);
  static constexpr int kSmemQ = kQBytes;
  static constexpr int kSmemK = kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemQ + kSmemK + 1024 /*barriers etc.*/ + 1024 /*align*/;
};

struct IdxArgs {
  int32_t* block_ids;
  int* status;
  int n_q, n_kv, q_pos0, h_kv, topk, causal, force_local, pool;
  int n_tiles;
  // Packed batch of independent causal prefills (varlen), or null: sequence
  // s owns rows [cu_seqlens[s], cu_seqlens[s + 1]) of Q_idx, K_idx and the
  // ids, positions restart at 0, and block ids are local to the sequence.
  const int* cu_seqlens;   // [batch + 1]
  const int* tile_pfx;     // [batch + 1] prefix of ceil(L_s / 128) (query tiles per sequence)
  const int* topk_seq;     // [batch] selected blocks of each sequence (adaptive k), or null: topk
  int batch;
};

// Sorted-descending register list of KMAX (score, block) pairs.  Slots
// [0, KMAX - k_free) hold +inf sentinels that never move; the live part is
// the last k_free slots.
template <int KMAX>
struct TopK {
  float sc[KMAX];
  int id[KMAX];

  __device__ __forceinline__ void init(int k_free) {
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      const bool dead = i < KMAX - k_free;
      sc[i] = dead ? __int_as_float(0x7f800000) : __int_as_float(0xff800000);
      id[i] = -1;
    }
  }
  __device__ __forceinline__ float threshold() const { return sc[KMAX - 1]; }

  // Insert (x, b); caller guarantees x > threshold().  An equal score already
  // in the list stays ahead of x (it has a lower block index).
  __device__ __forceinline__ void insert(float x, int b) {
#pragma unroll
    for (int i = KMAX - 1; i > 0; --i) {
      const bool down = x > sc[i - 1];          // element i-1 moves down to i
      const bool here = !down && (x > sc[i]);   // x lands at i
      sc[i] = down ? sc[i - 1] : (here ? x : sc[i]);
      id[i] = down ? id[i - 1] : (here ? b : id[i]);
    }
    if (x > sc[0]) {
      sc[0] = x;
      id[0] = b;
    }
  }
};

template <int DIDX, int BK, int KMAX, int POOL>
__global__ void __launch_bounds__(kThreads, 1)
    index_topk_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const IdxArgs args) {
  using Cfg = IdxCfg<DIDX>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;                       // [atoms][128 rows][kSwB]
  uint8_t* sk = smem + Cfg::kSmemQ;         // [stages][atoms][128 keys][kSwB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sk + Cfg::kSmemK);
  uint64_t* full = bars;                    // [kStages]
  uint64_t* empty = bars + Cfg::kStages;    // [kStages]
  uint64_t* acc_full = empty + Cfg::kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* q_full = acc_empty + 2;         // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int grp = static_cast<int>(blockIdx.x) % args.h_kv;
  // The problem this CTA belongs to: the whole call, or one sequence of a
  // packed batch (row_base = its first row; local positions from 0).
  int tile, n_q = args.n_q, n_kv = args.n_kv, q_pos0 = args.q_pos0, row_base = 0, k_sel = args.topk;
  if (args.cu_seqlens) {
    const int tl = static_cast<int>(blockIdx.x) / args.h_kv;
    if (tl >= args.tile_pfx[args.batch]) return;   // CTA-uniform, before any barrier or TMEM use
    int lo = 0, hi = args.batch - 1;               // sequence: largest s with tile_pfx[s] <= tl
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (args.tile_pfx[mid] <= tl) lo = mid; else hi = mid - 1;
    }
    row_base = args.cu_seqlens[lo];
    n_q = n_kv = args.cu_seqlens[lo + 1] - row_base;
    q_pos0 = 0;
    tile = args.tile_pfx[lo + 1] - 1 - tl;         // a sequence's heavy (late) tiles first
    if (args.topk_seq) k_sel = min(max(args.topk_seq[lo], 1), args.topk);
  } else {
    tile = args.n_tiles - 1 - static_cast<int>(blockIdx.x) / args.h_kv;  // heavy tiles first
  }
  const int i0 = tile * kRows;
  const int rows_here = min(kRows, n_q - i0);

  // Key range this CTA must score.  A row at position p needs keys < kv_lim(p)
  // where kv_lim = p + 1 (causal) or n_kv; with force_local its own block is
  // not scored, so it needs only keys below the start of that block.
  const int p_last = q_pos0 + i0 + rows_here - 1;
  int kv_end;
  if (!args.causal) {
    kv_end = n_kv;
  } else if (args.force_local) {
    kv_end = (p_last / BK) * BK;
  } else {
    kv_end = p_last + 1;
  }
  const int n_ktiles = (kv_end + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(q_full, 1);
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
  const WaitCtx wc{abort_flag, args.status};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0 && n_ktiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
      for (int a = 0; a < Cfg::kAtoms; ++a)
        tma_load_3d(sq + a * kRows * Cfg::kSwB, &tm_q, q_full, a * (Cfg::kSwB / 2), grp, row_base + i0);
      for (int t = 0; t < n_ktiles; ++t) {
        const int s = t % Cfg::kStages;
        const uint32_t ph = (t / Cfg::kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, wc)) break;
        mbar_arrive_expect_tx(&full[s], Cfg::kTileBytes);
        for (int a = 0; a < Cfg::kAtoms; ++a)
          tma_load_2d(sk + (s * Cfg::kAtoms + a) * kKeys * Cfg::kSwB, &tm_k, &full[s], a * (Cfg::kSwB / 2),
                      row_base + t * kKeys);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA
    // The whole warp runs the loop (warp-uniform waits and descriptor math)
    // and each MMA is predicated on an elected lane: a single-lane divergent
    // issue loop loses most of its issue slots to the two epilogue warps on
    // this SMSP (measured: 108 against 272 cycles per MMA with three busy
    // warps).
    if (n_ktiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kKeys, false, false);
      constexpr uint32_t sbo = 8 * Cfg::kSwB;   // 8-row core-matrix group stride
      // Descriptors differ only in the start-address field (address >> 4 in
      // bits 0-13, no carry for shared-memory addresses): base + offset.
      const uint64_t q_desc0 = smem_desc(smem_u32(sq), 16, sbo, Cfg::kSwz);
      const uint64_t k_desc0 = smem_desc(smem_u32(sk), 16, sbo, Cfg::kSwz);
      bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, wc));
      for (int t = 0; ok && t < n_ktiles; ++t) {
        const int s = t % Cfg::kStages;
        const int acc = t & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&acc_empty[acc], ((t >> 1) & 1) ^ 1, wc))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (t / Cfg::kStages) & 1, wc))) break;
        tc_fence_after();
        const uint64_t kd = k_desc0 + ((s * Cfg::kAtoms * kKeys * Cfg::kSwB) >> 4);
        const uint32_t d_tmem = tmem + acc * kKeys;
#pragma unroll
        for (int ks = 0; ks < DIDX / 16; ++ks) {
          constexpr int kPerAtom = Cfg::kSwB / 32;
          const uint32_t aoff = ((ks / kPerAtom) * kRows * Cfg::kSwB + (ks % kPerAtom) * 32) >> 4;
          const uint32_t boff = ((ks / kPerAtom) * kKeys * Cfg::kSwB + (ks % kPerAtom) * 32) >> 4;
          umma_ss_elect(d_tmem, q_desc0 + aoff, kd + boff, idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit_elect(&empty[s]);       // smem stage free once these MMAs finish
        umma_commit_elect(&acc_full[acc]);  // accumulator ready for the epilogue
        __syncwarp();
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - kEpiWarp0) >> 2;   // columns [128 half, 128 half + 128) of each tile
    const int row = quarter * 32 + lane;
    const bool row_ok = row < rows_here;
    const int p = q_pos0 + i0 + row;
    const int kv_lim = args.causal ? min(p + 1, n_kv) : n_kv;
    const int b_loc = p / BK;
    const int k_free = k_sel - (args.force_local ? 1 : 0);
    TopK<KMAX> tk;
    tk.init(k_free);
    const uint32_t taddr_row = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 128;

    for (int t = 0; t < n_ktiles; ++t) {
      const int acc = t & 1;
      if (!mbar_wait(&acc_full[acc], (t >> 1) & 1, wc)) break;
      tc_fence_after();
      constexpr int kBlocksPerHalf = 128 / BK;
      float bmax[kBlocksPerHalf];
#pragma unroll
      for (int bb = 0; bb < kBlocksPerHalf; ++bb) bmax[bb] = __int_as_float(0xff800000);
      const int j0 = t * kKeys + half * 128;
      if (j0 < kv_end) {
        // 128 columns in two 64-column pieces (two TMEM loads in flight per
        // wait); per block, four independent 3-input max chains (max-pool)
        // or add chains (mean-pool: masked keys add 0, and the sum of
        // integer-valued scores is exact in fp32 below 2^24).
        constexpr uint32_t kMasked = POOL == kPoolMax ? 0xff800000u : 0u;   // -inf / 0
        float m4[kBlocksPerHalf][4];
#pragma unroll
        for (int bb = 0; bb < kBlocksPerHalf; ++bb)
          m4[bb][0] = m4[bb][1] = m4[bb][2] = m4[bb][3] = __uint_as_float(kMasked);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[64];
          tmem_ld32(taddr_row + acc * kKeys + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld32(taddr_row + acc * kKeys + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_ld_wait();
          const int jh = j0 + h * 64;
          if (jh + 64 > kv_lim) {   // keys this row must not see
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (jh + e >= kv_lim) v[e] = kMasked;
          }
#pragma unroll
          for (int e = 0; e < 64; e += 8) {
            const int bb = (h * 64 + e) / BK;
            const int k = (e / 8) & 3;
            if (POOL == kPoolMax) {
              m4[bb][k] = max3f(m4[bb][k], fmaxf(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                                max3f(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]), __uint_as_float(v[e + 4])));
              m4[bb][k] = max3f(m4[bb][k], __uint_as_float(v[e + 5]),
                                fmaxf(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
            } else {
              float a0, a1, b0, b1;
              fadd2(a0, a1, __uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                    __uint_as_float(v[e + 3]));
              fadd2(b0, b1, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]), __uint_as_float(v[e + 6]),
                    __uint_as_float(v[e + 7]));
              fadd2(a0, a1, a0, a1, b0, b1);
              m4[bb][k] += a0 + a1;
            }
          }
        }
#pragma unroll
        for (int bb = 0; bb < kBlocksPerHalf; ++bb) {
          if (POOL == kPoolMax) {
            bmax[bb] = fmaxf(fmaxf(m4[bb][0], m4[bb][1]), fmaxf(m4[bb][2], m4[bb][3]));
          } else {
            // Mean over the visible keys of the block, ranked in fp32: a full
            // block divides by B_k exactly, a partial one rounds the quotient.
            const float sum = (m4[bb][0] + m4[bb][1]) + (m4[bb][2] + m4[bb][3]);
            const int cnt = min(BK, kv_lim - (j0 + bb * BK));
            bmax[bb] = cnt >= BK ? sum * (1.0f / BK)
                                 : (cnt > 0 ? __fdiv_rn(sum, static_cast<float>(cnt)) : __int_as_float(0xff800000));
          }
        }
      }
      // Release the accumulator stage to the MMA warp.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (row_ok && j0 < kv_end) {
#pragma unroll
        for (int bb = 0; bb < kBlocksPerHalf; ++bb) {
          const int b = (j0 / BK) + bb;
          const bool eligible = static_cast<long long>(b) * BK < kv_lim && !(args.force_local && b == b_loc);
          const float x = bmax[bb];
          if (eligible && x > tk.threshold()) tk.insert(x, b);
        }
      }
    }

    // Merge the two half-lists of each row: both go to shared memory (the K
    // ring is idle once every tile has been consumed), then the half-0 thread
    // takes the top k_free by (score desc, block asc), adds the local block
    // and writes the ids ascending, -1 padded.
    named_bar(1, 256);   // every epilogue thread is past its last accumulator read
    float* msc = reinterpret_cast<float*>(sk) + (half * kRows + row) * KMAX;
    int* mid = reinterpret_cast<int*>(sk + 2 * kRows * KMAX * 4) + (half * kRows + row) * KMAX;
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      msc[i] = tk.sc[i];
      mid[i] = tk.id[i];
    }
    named_bar(1, 256);
    if (half == 0 && row_ok) {
      const float* asc = msc;
      const int* aid = mid;
      const float* bsc = msc + kRows * KMAX;
      const int* bid = mid + kRows * KMAX;
      int ia = KMAX - k_free, ib = KMAX - k_free;   // live parts, each sorted (score desc, block asc)
      int ids[KMAX + 1];
#pragma unroll
      for (int i = 0; i < KMAX + 1; ++i) ids[i] = 0x7fffffff;
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        if (k < k_free) {
          const bool a_ok = ia < KMAX && aid[ia] >= 0;
          const bool b_ok = ib < KMAX && bid[ib] >= 0;
          if (a_ok || b_ok) {
            const bool take_a =
                a_ok && (!b_ok || asc[ia] > bsc[ib] || (asc[ia] == bsc[ib] && aid[ia] < bid[ib]));
            ids[k] = take_a ? aid[ia] : bid[ib];
            ia += take_a ? 1 : 0;
            ib += take_a ? 0 : 1;
          }
        }
      }
      ids[KMAX] = args.force_local ? b_loc : 0x7fffffff;
      // Odd-even transposition sort on static indices (stays in registers).
#pragma unroll
      for (int pass = 0; pass < KMAX + 1; ++pass) {
#pragma unroll
        for (int i = pass & 1; i + 1 < KMAX + 1; i += 2) {
          const int lo = min(ids[i], ids[i + 1]);
          const int hi = max(ids[i], ids[i + 1]);
          ids[i] = lo;
          ids[i + 1] = hi;
        }
      }
      int32_t* out = args.block_ids + (static_cast<size_t>(row_base + i0 + row) * args.h_kv + grp) * args.topk;
#pragma unroll
      for (int i = 0; i < KMAX + 1; ++i)
        if (i < args.topk) out[i] = ids[i] == 0x7fffffff ? -1 : ids[i];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) __nanosleep(1000000);  // let in-flight async copies/MMAs land
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DIDX, int BK, int KMAX, int POOL>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const IdxArgs& a, cudaStream_t st) {
  auto kern = index_topk_prefill_kernel<DIDX, BK, KMAX, POOL>;
  const int smem = IdxCfg<DIDX>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_tiles * a.h_kv);
  kern<<<grid, kThreads, smem, st>>>(tq, tk, a);
  return cudaGetLastError();
}

template <int DIDX, int BK>
cudaError_t launch_k(const CUtensorMap& tq, const CUtensorMap& tk, const IdxArgs& a, cudaStream_t st) {
  if (a.pool == kPoolMean)
    return a.topk <= 16 ? launch_t<DIDX, BK, 16, kPoolMean>(tq, tk, a, st) : launch_t<DIDX, BK, 32, kPoolMean>(tq, tk, a, st);
  return a.topk <= 16 ? launch_t<DIDX, BK, 16, kPoolMax>(tq, tk, a, st) : launch_t<DIDX, BK, 32, kPoolMax>(tq, tk, a, st);
}

template <int DIDX>
cudaError_t launch_b(int bk, const CUtensorMap& tq, const CUtensorMap& tk, const IdxArgs& a, cudaStream_t st) {
  if (bk == 64) return launch_k<DIDX, 64>(tq, tk, a, st);
  return launch_k<DIDX, 128>(tq, tk, a, st);
}

}  // namespace

int run_index_topk_prefill(const msa_params& p, const void* q_idx, const void* k_idx, int n_q, int n_kv,
                           int q_pos0, int32_t* block_ids, int* status, cudaStream_t stream, const Varlen* vl) {
  if (n_q == 0) return MSA_OK;
  const int sw_elems = p.d_idx >= 64 ? 64 : p.d_idx;    // TMA box inner extent (elements)
  const CUtensorMapSwizzle swz = p.d_idx >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.d_idx), static_cast<uint64_t>(p.h_kv),
                              static_cast<uint64_t>(n_q)};
    const uint64_t strides[2] = {static_cast<uint64_t>(p.d_idx) * 2, static_cast<uint64_t>(p.h_kv) * p.d_idx * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(sw_elems), 1, 128};
    if (!encode_tma_bf16(&tq, 3, q_idx, dims, strides, box, swz)) return MSA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(p.d_idx), static_cast<uint64_t>(n_kv)};
    const uint64_t strides[1] = {static_cast<uint64_t>(p.d_idx) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(sw_elems), static_cast<uint32_t>(kKeys)};
    if (!encode_tma_bf16(&tk, 2, k_idx, dims, strides, box, swz)) return MSA_ERR_CUDA;
  }
  IdxArgs a;
  a.block_ids = block_ids;
  a.status = status;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.q_pos0 = q_pos0;
  a.h_kv = p.h_kv;
  a.topk = p.topk;
  a.causal = p.causal;
  a.force_local = p.force_local;
  a.pool = p.pool;
  a.n_tiles = (n_q + kRows - 1) / kRows;
  a.cu_seqlens = vl ? vl->cu_seqlens : nullptr;
  a.tile_pfx = vl ? vl->tile_pfx : nullptr;
  a.topk_seq = vl ? vl->topk_seq : nullptr;
  a.batch = vl ? vl->batch : 0;
  // A packed batch has at most n_tiles + batch query tiles (each sequence adds
  // at most one partial tile); CTAs past the last tile exit at once.
  if (vl) a.n_tiles += vl->batch;
  cudaError_t e;
  switch (p.d_idx) {
    case 32: e = launch_b<32>(p.block_k, tq, tk, a, stream); break;
    case 64: e = launch_b<64>(p.block_k, tq, tk, a, stream); break;
    default: e = launch_b<128>(p.block_k, tq, tk, a, stream); break;
  }
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace msa
