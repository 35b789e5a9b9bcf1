// attn_sparse.cu -- block-major (KV-outer) main branch of a sparse prefill.
//
// Computes eq. (8) of the titansim.online summary of "MiniMax Sparse
// Attention" (section 4.3) for every selected block, with the block as the
// outer loop ("KV-Outer", section 4.4.2): the queries that selected a KV block
// are gathered so one block load feeds full 128-row tensor-core tiles, and
// the per-block results are merged afterwards (the pages' "two-stage merge",
// with no atomics on the outputs).
//
//   1. sched_count / sched_tile_sums + sched_scan_tiles / sched_fill: invert
//      block_ids [n_q, h_kv, k] into one list per (query wave, group r,
//      block b) of the (query, slot)
//      pairs that selected it (counting sort; slot = position of b in the
//      query's ids).  Lists are handed out in (wave, group, block) order, so
//      at any moment the CTAs gather the queries of one wave of kWave rows,
//      whose Q rows (kWave x h_q x d x 2 bytes) stay resident in L2.
//   2. attn_kvouter_kernel (persistent, warp-specialised, tcgen05):
//      * warp 0 grabs the next (r, b) list with an atomic counter, loads K_b
//        by TMA, then streams chunks of 128/G queries of the list (each
//        query's G head rows of group r are one 3-D TMA box, gathered with an
//        L2 evict-last policy into a 3-stage ring) and publishes a descriptor
//        per chunk in an 8-deep ring; V_b follows the list's first chunk.  K
//        and V have their own barriers, so the next list's K lands once the
//        last S has read K while the last PV still reads V.
//      * warp 1 issues S = Q K_b^T into the TMEM S buffer; warp 14 issues
//        O = P V_b (P read from one of two TMEM P buffers) into one of two
//        TMEM O buffers.  Both run their loops with the whole warp and issue
//        from one elected lane with precomputed descriptors: a tcgen05.mma
//        issuing thread slows with every busy warp on its SMSP.  S is
//        released as soon as the softmax has loaded it.
//      * warps 2..9 (softmax): two threads per row, each owning 64 of the 128
//        columns; the exact softmax of the row over the block's visible keys
//        (causal only in the local block); the two halves exchange only their
//        max through shared memory; P (bf16) goes to a P buffer; (m, l_lo,
//        l_hi) go to the epilogue.  (The exponentials are MUFU-bound: 16 per
//        clock per SM, so one 128x128 tile costs as many cycles as its two
//        MMAs; two warps per SM sub-partition keep the MUFU pipe fed.)
//      * warps 10..13 (epilogue): o = O / l in bf16 staged in shared memory and
//        written by TMA (L2 evict-first) as one contiguous 128-row tile per
//        chunk (chunk-major partials), lse2 = m c + log2 l beside it.
//   3. merge_partials_kernel: per (query, group), O = sum_s 2^(lse2_s - L) o_s
//      over the valid slots, L = log2 sum 2^lse2_s; rounded to bf16.  The
//      schedule records, per (query, group, slot), the partial row it wrote.
//
// A packed batch of sequences (varlen) runs the same kernels: a selection
// (query q, block b of q's sequence) goes to global block blk_pfx[s] + b, so
// lists never mix sequences, and the softmax masks with positions local to
// the sequence.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kThreads = 480;   // 15 warps
constexpr int kSoftW0 = 2;      // softmax warps 2..9: two per TMEM lane quarter, 64 columns each
constexpr int kEpiW0 = 10;      // epilogue warps 10..13
constexpr int kPvW = 14;        // PV issuer (S is issued by warp 1): each SMSP's issue port is shared
                                // with two softmax warps, so one thread issuing both would cap the rate
// One K/V stage suffices because a CTA switches blocks only once per
// (group, block) list (hundreds of chunks); the partial tile is staged in
// two shared-memory buffers for the TMA stores.
constexpr int kQStages = 3;
constexpr int kKVStages = 1;
constexpr int kOStages = 1;
constexpr int kDesc = 8;        // descriptor ring depth (a slot is held until the epilogue is done)
constexpr int kCtrlBytes = 20480;   // descriptors, softmax stats, staged entries, barriers
constexpr int kSchedThreads = 256;
constexpr int kStageEntries = 256;   // list entries staged in shared memory at a time
constexpr int kWave = 4096;          // query rows per wave (L2-resident Q working set)

template <int D, int BK>
struct KvoCfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = BK * D * 2;          // one of K or V
  static constexpr int kOBytes = 128 * D * 2;          // staged bf16 partial tile
  static constexpr int kSmemData = kQStages * kQBytes + kKVStages * 2 * kKVBytes + kOStages * kOBytes;
  static constexpr int kSmemBytes = kSmemData + kCtrlBytes + 1024;
  // TMEM: one S buffer (freed as soon as the softmax has loaded it), two P
  // buffers (bf16 pairs, BK/2 columns each), two O buffers.
  static constexpr int kColS = 0;        // S: [0, BK)
  static constexpr int kColP = BK;       // P: [BK, BK + BK/2), [BK + BK/2, 2BK)
  static constexpr int kColO = 2 * BK;   // O: [2BK, 2BK + D), [2BK + D, 2BK + 2D)
  static constexpr int kTmemCols = (2 * BK + 2 * D) <= 256 ? 256 : 512;
};

// One chunk of gathered queries of a (group, block) list.  (Declared before
// KvoCfg's users; the shared-memory budget check follows it.)
struct Desc {
  int entry[128];   // (query << 5) | slot, for the first `count` rows' queries
  int r, b, count, kvs;                      // b: block index within its sequence
  int first_of_kv, last_of_kv, end, chunk;   // chunk: global chunk id (partial tile index)
  int seq_row0, seq_len;                     // the block's sequence: first row, length
};

static_assert(kDesc * (sizeof(Desc) + 128 * 12) + 4 * 128 * 4 + kStageEntries * 4 + 64 * 8 + 16 <= kCtrlBytes,
              "control block of attn_kvouter_kernel exceeds its shared-memory reservation");

struct KvoArgs {
  const int* offs;       // [n_waves * h_kv * nb + 1] list offsets
  const int* chunk_off;  // [n_waves * h_kv * nb] first global chunk id of each list
  const int* entries;    // (query << 5) | slot, grouped by list
  const int* lists;      // non-empty list ids ((wave * h_kv + r) * nb + b)
  const int* wave_lo;    // the launch's lists: [wave_lo[0], wave_lo[1]) of `lists`
  int* work_counter;     // the launch's list counter
  float* part_lse;       // [chunks * 128] lse2 of each partial row
  int* status;
  int n_q, n_kv, q_pos0, h_q, h_kv, topk, causal, nb;
  float scale_log2;
  const int* cu_seqlens;   // packed batch of sequences (varlen), or null: one (chunked) prefill
  const int* blk_pfx;      // [batch + 1] prefix of ceil(L_s / B_k): global block = blk_pfx[s] + local block
  int batch;
};

// Sequence of a query row / of a global block in a packed batch: the largest
// s with pfx[s] <= x, for a non-decreasing pfx[0..batch].
__device__ __forceinline__ int seq_search(const int* pfx, int batch, int x) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pfx[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int D, int BK, int G>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kvouter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_po,
                        const KvoArgs args) {
  using Cfg = KvoCfg<D, BK>;
  constexpr int QPC = 128 / G;   // queries per chunk
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;                                        // [stage][atoms][128][128 B]
  uint8_t* skv = smem + kQStages * Cfg::kQBytes;             // [stage][K|V][atoms][BK][128 B]
  uint8_t* so = skv + kKVStages * 2 * Cfg::kKVBytes;         // [stage][atoms][128][128 B] partial tile
  Desc* desc = reinterpret_cast<Desc*>(smem + Cfg::kSmemData);
  float2* ml = reinterpret_cast<float2*>(desc + kDesc);      // [kDesc][128] (m, l of columns 0..63)
  float* lhi = reinterpret_cast<float*>(ml + kDesc * 128);   // [kDesc][128] l of columns 64..127
  float* smx = lhi + kDesc * 128;                            // [2 parity][2 halves][128] row-max exchange
  int* stage = reinterpret_cast<int*>(smx + 4 * 128);        // [kStageEntries] staged list entries
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage + kStageEntries);
  uint64_t* q_full = bars;                                   // [kQStages]
  uint64_t* q_empty = q_full + kQStages;
  // K and V of a stage have their own barriers: the next list's K can land
  // once the current list's last S has read K, while its last PV still
  // reads V.
  uint64_t* k_full = q_empty + kQStages;                     // [kKVStages]
  uint64_t* k_empty = k_full + kKVStages;
  uint64_t* v_full = k_empty + kKVStages;
  uint64_t* v_empty = v_full + kKVStages;
  uint64_t* d_full = v_empty + kKVStages;                    // [kDesc]
  uint64_t* d_empty = d_full + kDesc;
  uint64_t* s_full = d_empty + kDesc;                        // [1] S ready
  uint64_t* s_free = s_full + 1;                             // [1] S loaded by the softmax
  uint64_t* p_free = s_free + 1;                             // [2] P consumed by its PV
  uint64_t* p_full = p_free + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_free = o_full + 2;
  uint64_t* ml_full = o_free + 2;                            // [kDesc]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ml_full + kDesc);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < kDesc; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], 14);  // S and PV issuers + 8 softmax warps + 4 epilogue warps
      mbar_init(&ml_full[s], 8);   // 8 softmax warps
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);          // the 8 softmax warps, once their S loads completed
    for (int s = 0; s < 2; ++s) {
      mbar_init(&p_free[s], 1);
      mbar_init(&p_full[s], 8);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_free[s], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, args.status};
  const int list_lo = args.wave_lo[0], list_hi = args.wave_lo[1];
  // Gathered Q rows are re-read by up to k lists of their wave: keep them in
  // L2; partial tiles are read once, much later: let them leave first.
  const uint64_t q_policy = l2_evict_last();
  const uint64_t part_policy = l2_evict_first();

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (whole warp)
    // The list's (query, slot) entries are staged in shared memory 256 at a
    // time with coalesced loads, so no TMA issue waits on a dependent global
    // load; each lane issues the TMA boxes of its own queries.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    int t = 0;      // chunk counter
    int kvc = 0;    // KV stage use counter
    bool ok = true;
    while (ok) {
      int li = 0;
      if (lane == 0) li = list_lo + atomicAdd(args.work_counter, 1);
      li = __shfl_sync(0xffffffffu, li, 0);
      if (li >= list_hi) break;
      const int rb = args.lists[li];
      const int r = (rb / args.nb) % args.h_kv, gb = rb % args.nb;
      // The block's sequence: its key rows start at seq_row0 + b * BK.
      int b = gb, seq_row0 = 0, seq_len = args.n_kv;
      if (args.cu_seqlens) {
        const int sq_ = seq_search(args.blk_pfx, args.batch, gb);
        b = gb - args.blk_pfx[sq_];
        seq_row0 = args.cu_seqlens[sq_];
        seq_len = args.cu_seqlens[sq_ + 1] - seq_row0;
      }
      const int kv_row = seq_row0 + b * BK;
      const int start = args.offs[rb], cnt = args.offs[rb + 1] - start;
      const int chunk0 = args.chunk_off[rb];
      const int kvs = kvc % kKVStages;
      const uint32_t kv_ph = ((kvc / kKVStages) & 1) ^ 1;
      uint8_t* sk = skv + kvs * 2 * Cfg::kKVBytes;
      if (lane == 0) {
        ok = mbar_wait(&k_empty[kvs], kv_ph, wc);
        if (ok) {
          mbar_arrive_expect_tx(&k_full[kvs], Cfg::kKVBytes);
          for (int a = 0; a < Cfg::kAtoms; ++a)
            tma_load_3d(sk + a * BK * 128, &tm_k, &k_full[kvs], a * 64, r, kv_row);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++kvc;
      for (int c0 = 0; c0 < cnt; c0 += QPC) {
        // Refill the staging buffer every kStage entries.
        const int rel = c0 % kStageEntries;
        if (rel == 0) {
          __syncwarp();
#pragma unroll
          for (int u = 0; u < kStageEntries / 32; ++u) {
            const int k = c0 + u * 32 + lane;
            stage[u * 32 + lane] = k < cnt ? args.entries[start + k] : -1;
          }
          __syncwarp();
        }
        const int qs = t % kQStages, ds = t % kDesc;
        if (lane == 0) {
          ok = mbar_wait(&d_empty[ds], ((t / kDesc) & 1) ^ 1, wc) &&
               mbar_wait(&q_empty[qs], ((t / kQStages) & 1) ^ 1, wc);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        Desc& dd = desc[ds];
        const int n_here = min(QPC, cnt - c0);
        if (lane == 0) {
          dd.r = r;
          dd.b = b;
          dd.count = n_here;
          dd.kvs = kvs;
          dd.first_of_kv = c0 == 0;
          dd.last_of_kv = c0 + QPC >= cnt;
          dd.end = 0;
          dd.chunk = chunk0 + c0 / QPC;
          dd.seq_row0 = seq_row0;
          dd.seq_len = seq_len;
          mbar_arrive_expect_tx(&q_full[qs], Cfg::kQBytes);
        }
        __syncwarp();
        for (int qi = lane; qi < QPC; qi += 32) {
          const int e = qi < n_here ? stage[rel + qi] : -1;
          dd.entry[qi] = e;
          const int q = e >= 0 ? (e >> 5) : args.n_q;   // past the end: TMA fills zeros
          for (int a = 0; a < Cfg::kAtoms; ++a)
            tma_load_3d_hint(sq + qs * Cfg::kQBytes + a * 128 * 128 + qi * G * 128, &tm_q, &q_full[qs], a * 64,
                             r * G, q, q_policy);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_full[ds]);
        ++t;
        if (c0 == 0) {
          // V after the first chunk is out: S and the softmax of that chunk
          // run while the previous list's last PV releases the V buffer.
          if (lane == 0) {
            ok = mbar_wait(&v_empty[kvs], kv_ph, wc);
            if (ok) {
              mbar_arrive_expect_tx(&v_full[kvs], Cfg::kKVBytes);
              for (int a = 0; a < Cfg::kAtoms; ++a)
                tma_load_3d(sk + Cfg::kKVBytes + a * BK * 128, &tm_v, &v_full[kvs], a * 64, r, kv_row);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // End marker for the consumers.
    if (lane == 0 && ok && !*abort_flag) {
      const int ds = t % kDesc;
      if (mbar_wait(&d_empty[ds], ((t / kDesc) & 1) ^ 1, wc)) {
        desc[ds].end = 1;
        mbar_arrive(&d_full[ds]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA: S = Q K^T
    // Both issuers run their loops with the whole warp (warp-uniform waits
    // and descriptor math) and issue each MMA predicated on an elected lane:
    // a divergent single-lane loop loses most issue slots to the softmax and
    // epilogue warps sharing its SMSP (measured: 108 against 272 cycles per
    // MMA with three busy warps).
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, BK, false, false);
    // Descriptors differ only in their start-address field (address >> 4,
    // bits 0-13, never carrying out for shared-memory addresses), so they
    // are a base plus an offset.
    const uint64_t q_desc0 = smem_desc(smem_u32(sq), 16, 1024, kSwizzle128B);
    const uint64_t k_desc0 = smem_desc(smem_u32(skv), 16, 1024, kSwizzle128B);
    int kvc = 0;   // lists whose K was awaited
    for (int t = 0;; ++t) {
      const int ds = t % kDesc;
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[ds], (t / kDesc) & 1, wc))) break;
      const Desc& dd = desc[ds];
      const int end = dd.end, kvs = dd.kvs, first = dd.first_of_kv, last = dd.last_of_kv;
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[ds]);
      if (end) break;
      const int qs = t % kQStages;
      if (first) {
        if (!__all_sync(0xffffffffu, mbar_wait(&k_full[kvs], (kvc / kKVStages) & 1, wc))) break;
        ++kvc;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[qs], (t / kQStages) & 1, wc))) break;
      // S(t) reuses the single S buffer once the softmax has loaded S(t-1).
      if (!__all_sync(0xffffffffu, mbar_wait(s_free, (t & 1) ^ 1, wc))) break;
      tc_fence_after();
      const uint64_t qd = q_desc0 + ((qs * Cfg::kQBytes) >> 4);
      const uint64_t kd = k_desc0 + ((kvs * 2 * Cfg::kKVBytes) >> 4);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks / 4) * (128 * 128) + (ks % 4) * 32;
        const uint32_t koff = (ks / 4) * (BK * 128) + (ks % 4) * 32;
        umma_ss_elect(tmem + Cfg::kColS, qd + (off >> 4), kd + (koff >> 4), idesc_s, ks > 0 ? 1u : 0u);
      }
      umma_commit_elect(&q_empty[qs]);
      umma_commit_elect(s_full);
      if (last) umma_commit_elect(&k_empty[kvs]);   // this list's last read of K
      __syncwarp();
    }
  } else if (warp == kPvW) {
    // ---------------------------------------------------------------- UMMA: O = P V
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
    const uint64_t v_desc0 = smem_desc(smem_u32(skv) + Cfg::kKVBytes, BK * 128, 1024, kSwizzle128B);
    int vc = 0;   // lists whose V was awaited
    for (int t = 0;; ++t) {
      const int ds = t % kDesc;
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[ds], (t / kDesc) & 1, wc))) break;
      const Desc& dd = desc[ds];
      const int end = dd.end, kvs = dd.kvs, first = dd.first_of_kv, last = dd.last_of_kv;
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[ds]);
      if (end) break;
      const int sb = t & 1;
      if (first) {
        if (!__all_sync(0xffffffffu, mbar_wait(&v_full[kvs], (vc / kKVStages) & 1, wc))) break;
        ++vc;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&p_full[sb], (t >> 1) & 1, wc))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&o_free[sb], ((t >> 1) & 1) ^ 1, wc))) break;
      tc_fence_after();
      const uint64_t vd = v_desc0 + ((kvs * 2 * Cfg::kKVBytes) >> 4);
      const uint32_t p_tmem = tmem + Cfg::kColP + sb * (BK / 2);
      const uint32_t o_tmem = tmem + Cfg::kColO + sb * D;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        umma_ts_elect(o_tmem, p_tmem + kk * 8, vd + ((kk * 2048) >> 4), idesc_o, kk > 0 ? 1u : 0u);
      umma_commit_elect(&o_full[sb]);
      umma_commit_elect(&p_free[sb]);
      if (last) umma_commit_elect(&v_empty[kvs]);   // this list's last read of V
      __syncwarp();
    }
  } else if (warp >= kSoftW0 && warp < kEpiW0) {
    // ---------------------------------------------------------------- softmax
    constexpr int HC = BK / 2;                 // columns per thread
    const int quarter = warp & 3;
    const int half = (warp - kSoftW0) / 4;     // 0: columns [0, HC), 1: [HC, BK)
    const int row = quarter * 32 + lane;
    const int qi = row / G;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = args.scale_log2;
    for (int t = 0;; ++t) {
      const int ds = t % kDesc;
      if (!mbar_wait(&d_full[ds], (t / kDesc) & 1, wc)) break;
      const Desc& dd = desc[ds];
      if (dd.end) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[ds]);
        break;
      }
      const int e = qi < dd.count ? dd.entry[qi] : -1;
      const int b = dd.b, seq_row0 = dd.seq_row0, seq_len = dd.seq_len;
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[ds]);
      int lim = 0;   // visible keys of this block for the row, relative to this half
      if (e >= 0) {   // positions local to the query's sequence
        const int p = (args.cu_seqlens ? 0 : args.q_pos0) + (e >> 5) - seq_row0;
        const int kv_lim = args.causal ? min(p + 1, seq_len) : seq_len;
        lim = min(BK, kv_lim - b * BK) - half * HC;
      }
      const int sb = t & 1;   // P buffer
      if (!mbar_wait(s_full, t & 1, wc)) break;
      tc_fence_after();
      const uint32_t s_tmem = lane_base + Cfg::kColS;
      uint32_t sv[HC];
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc)
        tmem_ld32(s_tmem + half * HC + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[cc * 32]));
      tmem_ld_wait();
      // S is in registers: hand the S buffer back so the next S MMA can start.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      if (lim < HC) {
#pragma unroll
        for (int i = 0; i < HC; ++i)
          if (i >= lim) sv[i] = 0xff800000u;   // -inf: masked key
      }
      float mq[4] = {__int_as_float(0xff800000), __int_as_float(0xff800000), __int_as_float(0xff800000),
                     __int_as_float(0xff800000)};
#pragma unroll
      for (int i = 0; i < HC; i += 8) {
        const int k = (i / 8) & 3;
        mq[k] = max3f(mq[k], fmaxf(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])),
                      max3f(__uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]), __uint_as_float(sv[i + 4])));
        mq[k] = max3f(mq[k], __uint_as_float(sv[i + 5]), fmaxf(__uint_as_float(sv[i + 6]), __uint_as_float(sv[i + 7])));
      }
      // Exchange the half-row maxima with the partner warp (same lane quarter).
      // The slot alternates with the chunk parity: a warp rewrites slot
      // (t & 1) only after the next barrier, which its partner reaches only
      // after reading this chunk's value.
      float* xs = smx + (t & 1) * 256;
      xs[half * 128 + row] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      named_bar(2 + quarter, 64);
      const float mx = fmaxf(xs[row], xs[128 + row]);
      const float bias = mx == __int_as_float(0xff800000) ? 0.f : mx * c;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};   // two pairs of partial sums
      uint32_t pk[HC / 2];
#pragma unroll
      for (int i = 0; i < HC; i += 4) {
        float x0, x1, x2, x3;
        ffma2(x0, x1, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]), c, c, -bias, -bias);
        ffma2(x2, x3, __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]), c, c, -bias, -bias);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
        float s0, s1;
        fadd2(s0, s1, p0, p1, p2, p3);
        const int k = ((i / 4) & 1) * 2;
        fadd2(ls[k], ls[k + 1], ls[k], ls[k + 1], s0, s1);
        pk[i / 2] = pack_bf16x2(p0, p1);
        pk[i / 2 + 1] = pack_bf16x2(p2, p3);
      }
      // P(t) goes to P buffer t & 1 once the PV of chunk t - 2 has read it.
      if (!mbar_wait(&p_free[sb], ((t >> 1) & 1) ^ 1, wc)) break;
      tc_fence_after();
      const uint32_t p_tmem = lane_base + Cfg::kColP + sb * (BK / 2);
#pragma unroll
      for (int cc = 0; cc < HC / 64; ++cc)
        tmem_st32(p_tmem + half * (HC / 2) + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[cc * 32]));
      if (HC / 2 == 16) tmem_st16(p_tmem + half * (HC / 2), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (half == 0)
        ml[ds * 128 + row] = make_float2(mx, lsum);
      else
        lhi[ds * 128 + row] = lsum;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&p_full[sb]);
        mbar_arrive(&ml_full[ds]);
      }
    }
  } else if (warp >= kEpiW0 && warp < kEpiW0 + 4) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qi = row / G;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = args.scale_log2;
    for (int t = 0;; ++t) {
      const int ds = t % kDesc;
      if (!mbar_wait(&d_full[ds], (t / kDesc) & 1, wc)) break;
      const Desc& dd = desc[ds];
      if (dd.end) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[ds]);
        break;
      }
      const int e = qi < dd.count ? dd.entry[qi] : -1;
      const int sb = t & 1;
      if (!mbar_wait(&o_full[sb], (t >> 1) & 1, wc)) break;
      if (!mbar_wait(&ml_full[ds], (t / kDesc) & 1, wc)) break;
      tc_fence_after();
      const float2 st = ml[ds * 128 + row];
      const float lsum = st.y + lhi[ds * 128 + row];
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      const float lse2 = lsum > 0.f ? st.x * c + __log2f(lsum) : __int_as_float(0xff800000);
      const int chunk = dd.chunk;
      const int os = t % kOStages;
      // Stage the bf16 row in the swizzled tile layout (the layout TMA uses),
      // after the stores that last read this staging buffer have drained.
      if (warp == kEpiW0 && lane == 0) {
        if (kOStages == 1)
          bulk_wait_read0();
        else
          bulk_wait_read_le1();
      }
      named_bar(1, 128);
      const uint32_t so_addr = smem_u32(so + os * Cfg::kOBytes);
#pragma unroll
      for (int a = 0; a < D / 64; ++a) {
        uint32_t ov[64];
        tmem_ld32(lane_base + Cfg::kColO + sb * D + a * 64, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
        tmem_ld32(lane_base + Cfg::kColO + sb * D + a * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
        tmem_ld_wait();
        if (a == D / 64 - 1) {
          // The O buffer is free once its values are in registers.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_free[sb]);
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const float* f = reinterpret_cast<const float*>(&ov[ch * 8]);
          float g[8];
#pragma unroll
          for (int j = 0; j < 8; j += 2) fmul2(g[j], g[j + 1], f[j], f[j + 1], inv, inv);
          st_shared_v4(so_addr + a * 128 * 128 + row * 128 + ((ch ^ (row & 7)) << 4), pack_bf16x2(g[0], g[1]),
                       pack_bf16x2(g[2], g[3]), pack_bf16x2(g[4], g[5]), pack_bf16x2(g[6], g[7]));
        }
      }
      args.part_lse[static_cast<size_t>(chunk) * 128 + row] = e >= 0 ? lse2 : __int_as_float(0xff800000);
      fence_proxy_async_smem();
      named_bar(1, 128);
      // One thread issues, commits and later waits for the chunk's tile
      // stores (bulk groups are tracked per thread): one box per d atom.
      if (warp == kEpiW0 && lane == 0) {
        for (int a = 0; a < D / 64; ++a)
          tma_store_2d_hint(&tm_po, so + os * Cfg::kOBytes + a * 128 * 128, a * 64, chunk * 128, part_policy);
        bulk_commit();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[ds]);   // also releases ml[ds]
    }
    if (warp == kEpiW0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) __nanosleep(1000000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// schedule: block_ids -> per-(group, block) lists of (query, slot)
// ---------------------------------------------------------------------------
// Schedule geometry shared by the three kernels: a selection (query q, block
// b local to q's sequence) maps to global block blk_pfx[s] + b of the packed
// batch (one sequence: the block itself); -1 when b is no block of q's
// sequence.
struct SchedGeom {
  const int* cu_seqlens;   // or null: one sequence of n_kv keys
  const int* blk_pfx;
  int batch, nb_one, bk;   // nb_one: blocks of the single sequence
  int nb;                  // blocks of the schedule (bound of every global block)
  __device__ __forceinline__ int global_block(int q, int b) const {
    if (b < 0) return -1;
    if (!cu_seqlens) return b < nb_one ? b : -1;
    const int s = seq_search(cu_seqlens, batch, q);
    const int L = cu_seqlens[s + 1] - cu_seqlens[s];
    const int gb = blk_pfx[s] + b;
    return (b < (L + bk - 1) / bk && gb < nb) ? gb : -1;
  }
};

__global__ void sched_count_kernel(const int32_t* ids, long long total, int h_kv, int topk, int nb, SchedGeom geo,
                                   int* cnt) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int q = static_cast<int>(e / (static_cast<long long>(topk) * h_kv));
  const int gb = geo.global_block(q, ids[e]);
  if (gb < 0) return;
  const int r = static_cast<int>((e / topk) % h_kv);
  atomicAdd(&cnt[((q / kWave) * h_kv + r) * nb + gb], 1);
}

// The schedule's exclusive prefixes over the lists (entries, non-empty lists,
// chunks of 128 / G queries), in two multi-CTA passes over tiles of
// kScanTile lists: the tile totals, then each tile's scan on top of the sum of
// the tiles before it.  The second pass also compacts the non-empty lists
// (ascending) and, in its last thread, writes the totals and the launch's
// list range [0, n_lists).
constexpr int kScanThreads = 256;
constexpr int kScanPer = 8;
constexpr int kScanTile = kScanThreads * kScanPer;

__device__ __forceinline__ void list_totals(int v, int qpc, int& a, int& b, int& c) {
  a += v;
  b += v > 0;
  c += (v + qpc - 1) / qpc;
}

__global__ void __launch_bounds__(kScanThreads) sched_tile_sums_kernel(const int* cnt, int n, int qpc, int* tsum) {
  __shared__ int ws[3][kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i0 = blockIdx.x * kScanTile + threadIdx.x * kScanPer;
  int a = 0, b = 0, c = 0;
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) list_totals(i0 + k < n ? cnt[i0 + k] : 0, qpc, a, b, c);
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, x);
    b += __shfl_xor_sync(0xffffffffu, b, x);
    c += __shfl_xor_sync(0xffffffffu, c, x);
  }
  if (lane == 0) {
    ws[0][warp] = a;
    ws[1][warp] = b;
    ws[2][warp] = c;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kScanThreads / 32; ++w) t += ws[threadIdx.x][w];
    tsum[3 * blockIdx.x + threadIdx.x] = t;
  }
}

__global__ void __launch_bounds__(kScanThreads) sched_scan_tiles_kernel(const int* cnt, int n, int qpc,
                                                                        const int* tsum, int* offs, int* chunk_off,
                                                                        int* lists, int* n_lists, int* range) {
  constexpr int kW = kScanThreads / 32;
  __shared__ int ws[3][kW];
  __shared__ int tile_base[3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {
    // Sum of the totals of the tiles before this one.
    int a = 0, b = 0, c = 0;
    for (int t = lane; t < static_cast<int>(blockIdx.x); t += 32) {
      a += tsum[3 * t];
      b += tsum[3 * t + 1];
      c += tsum[3 * t + 2];
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, x);
      b += __shfl_xor_sync(0xffffffffu, b, x);
      c += __shfl_xor_sync(0xffffffffu, c, x);
    }
    if (lane == 0) {
      tile_base[0] = a;
      tile_base[1] = b;
      tile_base[2] = c;
    }
  }
  const int i0 = blockIdx.x * kScanTile + threadIdx.x * kScanPer;
  int v[kScanPer];
  int ta = 0, tb = 0, tc = 0;
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    v[k] = i0 + k < n ? cnt[i0 + k] : 0;
    list_totals(v[k], qpc, ta, tb, tc);
  }
  // Inclusive warp scan of the thread totals, then over the warps.
  int ia = ta, ib = tb, ic = tc;
#pragma unroll
  for (int x = 1; x < 32; x <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, ia, x);
    const int xb = __shfl_up_sync(0xffffffffu, ib, x);
    const int xc = __shfl_up_sync(0xffffffffu, ic, x);
    if (lane >= x) {
      ia += xa;
      ib += xb;
      ic += xc;
    }
  }
  if (lane == 31) {
    ws[0][warp] = ia;
    ws[1][warp] = ib;
    ws[2][warp] = ic;
  }
  __syncthreads();
  int pa = tile_base[0] + ia - ta, pb = tile_base[1] + ib - tb, pc = tile_base[2] + ic - tc;
#pragma unroll
  for (int w = 0; w < kW; ++w) {
    if (w < warp) {
      pa += ws[0][w];
      pb += ws[1][w];
      pc += ws[2][w];
    }
  }
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    const int i = i0 + k;
    if (i < n) {
      offs[i] = pa;
      chunk_off[i] = pc;
      if (v[k] > 0) lists[pb++] = i;
    }
    pa += v[k];
    pc += (v[k] + qpc - 1) / qpc;
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == kScanThreads - 1) {
    // Lists past n add nothing, so this thread's running sums are the totals.
    offs[n] = pa;
    *n_lists = pb;
    range[0] = 0;
    range[1] = pb;
  }
}

__global__ void sched_fill_kernel(const int32_t* ids, long long total, int h_kv, int topk, int nb, int G,
                                  SchedGeom geo, const int* offs, const int* chunk_off, int* fill, int* entries,
                                  int* prow_of) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int q = static_cast<int>(e / (static_cast<long long>(topk) * h_kv));
  const int gb = geo.global_block(q, ids[e]);
  if (gb < 0) {
    prow_of[e] = -1;   // padding: the merge skips it
    return;
  }
  const int slot = static_cast<int>(e % topk);
  const int r = static_cast<int>((e / topk) % h_kv);
  const int rb = ((q / kWave) * h_kv + r) * nb + gb;
  const int k = atomicAdd(&fill[rb], 1);    // position inside the list
  entries[offs[rb] + k] = (q << 5) | slot;
  const int qpc = 128 / G;
  prow_of[e] = (chunk_off[rb] + k / qpc) * 128 + (k % qpc) * G;
}

// ---------------------------------------------------------------------------
// merge: O[q, h] = sum over valid slots of 2^(lse2_s - L) o_s
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) merge_partials_kernel(const int* prow_of, const uint16_t* part_o,
                                                             const float* part_lse, uint16_t* o, int h_q, int h_kv,
                                                             int topk, int q0) {
  // One CTA per (query, group); thread = (head within group, 8-column chunk).
  // prow_of[(q, r, slot)] is the first partial row (chunk * 128 + query-in-
  // chunk * G) the block-major kernel wrote for that selection, -1 for none.
  // Slots are read 8 at a time with independent loads and folded in with an
  // online log-sum-exp, so the loads of a group are all in flight together.
  constexpr int kGrp = 8;
  const int qr = q0 * h_kv + static_cast<int>(blockIdx.x);   // this launch: queries from q0
  const int q = qr / h_kv, r = qr % h_kv;
  const int G = h_q / h_kv;
  constexpr int kChunks = D / 8;
  const int* my_rows = prow_of + static_cast<size_t>(qr) * topk;
  for (int w = threadIdx.x; w < G * kChunks; w += blockDim.x) {
    const int hh = w / kChunks, ch = w % kChunks;
    float M = __int_as_float(0xff800000), den = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < topk; s0 += kGrp) {
      float ls[kGrp];
      uint4 v[kGrp];
#pragma unroll
      for (int j = 0; j < kGrp; ++j) {
        const int s = s0 + j;
        const int pr = s < topk ? my_rows[s] : -1;   // -1: padding or no block of this sequence
        const bool ok = pr >= 0;
        const size_t prow = ok ? static_cast<size_t>(pr) + hh : 0;
        ls[j] = ok ? part_lse[prow] : __int_as_float(0xff800000);
        v[j] = ok ? *reinterpret_cast<const uint4*>(part_o + prow * D + ch * 8) : make_uint4(0, 0, 0, 0);
      }
      float gm = M;
#pragma unroll
      for (int j = 0; j < kGrp; ++j) gm = fmaxf(gm, ls[j]);
      if (gm == __int_as_float(0xff800000)) continue;
      const float alpha = ex2_approx(M - gm);   // 0 when M is still -inf
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= alpha;
      den *= alpha;
      M = gm;
#pragma unroll
      for (int j = 0; j < kGrp; ++j) {
        const float wgt = ex2_approx(ls[j] - gm);   // 0 for empty slots
        den += wgt;
        const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wgt, __uint_as_float(u[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wgt, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
        }
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint4 out;
    out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    out.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    out.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4*>(o + (static_cast<size_t>(q) * h_q + r * G + hh) * D + ch * 8) = out;
  }
}

template <int D, int BK, int G>
cudaError_t launch_kvo(const CUtensorMap* m, const KvoArgs& a, int grid, cudaStream_t st) {
  auto kern = attn_kvouter_kernel<D, BK, G>;
  const int smem = KvoCfg<D, BK>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(m[0], m[1], m[2], m[3], a);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_kvo_g(int G, const CUtensorMap* m, const KvoArgs& a, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_kvo<D, BK, 1>(m, a, grid, st);
    case 2: return launch_kvo<D, BK, 2>(m, a, grid, st);
    case 4: return launch_kvo<D, BK, 4>(m, a, grid, st);
    case 8: return launch_kvo<D, BK, 8>(m, a, grid, st);
    case 16: return launch_kvo<D, BK, 16>(m, a, grid, st);
    case 32: return launch_kvo<D, BK, 32>(m, a, grid, st);
    case 64: return launch_kvo<D, BK, 64>(m, a, grid, st);
    default: return launch_kvo<D, BK, 128>(m, a, grid, st);
  }
}

struct SparseWs {
  int *cnt, *fill, *offs, *chunk_off, *lists, *n_lists, *work, *entries, *prow_of, *wave_lo, *tsum;
  uint16_t* part_o;
  float* part_lse;
  size_t max_chunks, bytes;
};

// Blocks of the schedule: those of the one sequence, or, for a packed batch
// of `batch` sequences with n_kv rows in all, at most ceil(n_kv / B_k) +
// batch (each sequence adds at most one partial block).
int sched_blocks(const msa_params& p, int n_kv, int batch) {
  return (n_kv + p.block_k - 1) / p.block_k + (batch > 0 ? batch : 0);
}

SparseWs carve(const msa_params& p, int n_q, int n_kv, int batch, void* base) {
  const int nb = sched_blocks(p, n_kv, batch);
  const int n_waves = (n_q + kWave - 1) / kWave;
  const size_t nl = static_cast<size_t>(n_waves) * p.h_kv * nb;
  const size_t nnz = static_cast<size_t>(n_q) * p.h_kv * p.topk;
  const int qpc = 128 / (p.h_q / p.h_kv);
  uint8_t* w = static_cast<uint8_t*>(base);
  size_t off = 0;
  SparseWs s;
  auto take = [&](size_t bytes) {
    uint8_t* ptr = w ? w + off : nullptr;
    off += align_up(bytes, 256);
    return ptr;
  };
  // cnt, fill, the list count and the work counter are contiguous so one
  // memset clears them.
  s.cnt = reinterpret_cast<int*>(take((2 * nl + 2) * 4));
  s.fill = s.cnt ? s.cnt + nl : nullptr;
  s.n_lists = s.cnt ? s.cnt + 2 * nl : nullptr;
  s.work = s.cnt ? s.cnt + 2 * nl + 1 : nullptr;
  s.wave_lo = reinterpret_cast<int*>(take(2 * 4));
  s.tsum = reinterpret_cast<int*>(take(static_cast<size_t>((nl + kScanTile - 1) / kScanTile) * 3 * 4));
  s.offs = reinterpret_cast<int*>(take((nl + 1) * 4));
  s.chunk_off = reinterpret_cast<int*>(take(nl * 4));
  s.lists = reinterpret_cast<int*>(take(nl * 4));
  s.entries = reinterpret_cast<int*>(take(nnz * 4));
  s.prow_of = reinterpret_cast<int*>(take(nnz * 4));
  // Every list rounds up to whole chunks: at most nnz / qpc + nl chunks.
  s.max_chunks = (nnz + qpc - 1) / qpc + nl;
  s.part_lse = reinterpret_cast<float*>(take(s.max_chunks * 128 * 4));
  s.part_o = reinterpret_cast<uint16_t*>(take(s.max_chunks * 128 * static_cast<size_t>(p.d) * 2));
  s.bytes = off;
  return s;
}

}  // namespace

// The schedule indexes lists, entries and partial rows with 32-bit integers
// (list ids, prefix sums, TMA row coordinates of the partial tiles).
bool sparse_sizes_supported(const msa_params& p, int n_q, int n_kv, int batch) {
  const long long kMax = 0x7fffffffLL;
  const long long nb = sched_blocks(p, n_kv, batch);
  const long long nl = static_cast<long long>((n_q + kWave - 1) / kWave) * p.h_kv * nb;
  const long long nnz = static_cast<long long>(n_q) * p.h_kv * p.topk;
  const long long qpc = 128 / (p.h_q / p.h_kv);
  const long long rows = ((nnz + qpc - 1) / qpc + nl) * 128;
  return nl <= kMax && nnz <= kMax && rows <= kMax;
}

size_t sparse_prefill_workspace_bytes(const msa_params& p, int n_q, int n_kv, int batch) {
  return carve(p, n_q, n_kv, batch, nullptr).bytes;
}

int run_sparse_attn_kvouter(const msa_params& p, const void* q, const CUtensorMap& tk, const CUtensorMap& tv,
                            const int32_t* block_ids, int n_q, int n_kv, int q_pos0, void* o, void* ws,
                            size_t ws_bytes, int* status, cudaStream_t stream, const Varlen* vl) {
  const int batch = vl ? vl->batch : 0;
  if (!sparse_sizes_supported(p, n_q, n_kv, batch)) return MSA_ERR_UNSUPPORTED;
  SparseWs s = carve(p, n_q, n_kv, batch, ws);
  if (ws_bytes < s.bytes) return MSA_ERR_WORKSPACE;
  const int G = p.h_q / p.h_kv;
  CUtensorMap tq;   // one box = the G head rows of one query of one group
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.h_q), static_cast<uint64_t>(n_q)};
    const uint64_t strides[2] = {static_cast<uint64_t>(p.d) * 2, static_cast<uint64_t>(p.h_q) * p.d * 2};
    const uint32_t box[3] = {64, static_cast<uint32_t>(G), 1};
    if (!encode_tma_bf16(&tq, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  const int nb = sched_blocks(p, n_kv, batch);
  const int nl = ((n_q + kWave - 1) / kWave) * p.h_kv * nb;
  const long long total = static_cast<long long>(n_q) * p.h_kv * p.topk;
  SchedGeom geo;
  geo.cu_seqlens = vl ? vl->cu_seqlens : nullptr;
  geo.blk_pfx = vl ? vl->blk_pfx : nullptr;
  geo.batch = batch;
  geo.nb_one = (n_kv + p.block_k - 1) / p.block_k;
  geo.bk = p.block_k;
  geo.nb = nb;
  if (cudaMemsetAsync(s.cnt, 0, (2 * static_cast<size_t>(nl) + 2) * 4, stream) != cudaSuccess) return MSA_ERR_CUDA;
  const int gsz = static_cast<int>((total + kSchedThreads - 1) / kSchedThreads);
  sched_count_kernel<<<gsz, kSchedThreads, 0, stream>>>(block_ids, total, p.h_kv, p.topk, nb, geo, s.cnt);
  const int n_tiles = (nl + kScanTile - 1) / kScanTile;
  sched_tile_sums_kernel<<<n_tiles, kScanThreads, 0, stream>>>(s.cnt, nl, 128 / G, s.tsum);
  sched_scan_tiles_kernel<<<n_tiles, kScanThreads, 0, stream>>>(s.cnt, nl, 128 / G, s.tsum, s.offs, s.chunk_off,
                                                                 s.lists, s.n_lists, s.wave_lo);
  sched_fill_kernel<<<gsz, kSchedThreads, 0, stream>>>(block_ids, total, p.h_kv, p.topk, nb, G, geo, s.offs,
                                                       s.chunk_off, s.fill, s.entries, s.prow_of);
  if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;

  KvoArgs a;
  a.offs = s.offs;
  a.chunk_off = s.chunk_off;
  a.entries = s.entries;
  a.lists = s.lists;
  a.part_lse = s.part_lse;
  a.status = status;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.q_pos0 = q_pos0;
  a.h_q = p.h_q;
  a.h_kv = p.h_kv;
  a.topk = p.topk;
  a.causal = p.causal;
  a.nb = nb;
  a.cu_seqlens = geo.cu_seqlens;
  a.blk_pfx = geo.blk_pfx;
  a.batch = batch;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf(static_cast<float>(p.d));
  a.scale_log2 = scale * 1.4426950408889634f;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  CUtensorMap maps[4] = {tq, tk, tv, tq};
  {  // chunk-major partial rows [max_chunks * 128][d]: one box = 128 rows x 64 columns
    const uint64_t dims[2] = {static_cast<uint64_t>(p.d), static_cast<uint64_t>(s.max_chunks) * 128};
    const uint64_t strides[1] = {static_cast<uint64_t>(p.d) * 2};
    const uint32_t box[2] = {64, 128};
    if (!encode_tma_bf16(&maps[3], 2, s.part_o, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  auto launch_attn = [&](int w, int grid) -> cudaError_t {
    a.wave_lo = s.wave_lo + w;   // w = 0 with wave_lo[1] = n_lists: every list
    a.work_counter = s.work + w;
    if (p.d == 64)
      return p.block_k == 64 ? launch_kvo_g<64, 64>(G, maps, a, grid, stream)
                             : launch_kvo_g<64, 128>(G, maps, a, grid, stream);
    return p.block_k == 64 ? launch_kvo_g<128, 64>(G, maps, a, grid, stream)
                           : launch_kvo_g<128, 128>(G, maps, a, grid, stream);
  };
  auto launch_merge = [&](cudaStream_t st) {
    if (p.d == 64)
      merge_partials_kernel<64><<<n_q * p.h_kv, 256, 0, st>>>(s.prow_of, s.part_o, s.part_lse,
                                                              static_cast<uint16_t*>(o), p.h_q, p.h_kv, p.topk, 0);
    else
      merge_partials_kernel<128><<<n_q * p.h_kv, 256, 0, st>>>(s.prow_of, s.part_o, s.part_lse,
                                                               static_cast<uint16_t*>(o), p.h_q, p.h_kv, p.topk, 0);
  };
  // One persistent launch over every wave's lists on every SM, then the
  // merge.  (Launching each wave separately on fewer SMs, with its merge on a
  // second stream under the next wave, measured slower: ~0.2 ms of ramp and
  // tail per wave launch outweighed the overlap.)
  if (launch_attn(0, sms) != cudaSuccess) return MSA_ERR_CUDA;
  launch_merge(stream);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace msa
