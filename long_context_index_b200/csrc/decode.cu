// decode.cu -- one batched decode step of MiniMax Sparse Attention on sm_100a.
//
// For every sequence b the query sits at position p = L_b - 1 of its own
// contiguous caches.  The step is the prefill math of one row
// (titansim.online summary of "MiniMax Sparse Attention": eq. (6) and the
// local-block rule in section 4.2, eq. (8) in section 4.3), as two
// persistent HBM-streaming launches, or (process option MSA_OPT_DECODE_FUSED)
// as one fused cooperative launch when the step fits one co-resident wave.
// Both forms run the same two parts:
//
//   1. decode_index_kernel   The blocks of all sequences, end to end, are cut
//      into equal ranges, one per CTA.  Streams the index-key cache once for
//      all groups with 16-byte coalesced loads that feed mma.sync directly (a
//      fixed permutation of the d_idx axis, applied to Q_idx and K_idx alike,
//      makes each loaded 16-byte vector a fragment; the dot product does not
//      depend on the order of d_idx).  Max-pools per block and keeps, per
//      (sequence, group) share, the top (k - 1) non-local blocks.  The CTA
//      that completes a sequence's block count merges its shares (score desc,
//      block asc: exact because every global winner wins within its share),
//      adds the local block and writes the ids ascending.
//   2. decode_attn_stream_kernel  The (sequence, group, head tile, slot)
//      items are cut into equal ranges, one per CTA.  A producer warp
//      TMA-loads the Q tile and the selected K/V block per item; four consumer
//      warps run QK^T and PV on mma.sync with an fp32 online softmax.  A unit
//      split between CTAs is merged by the last of them (LSE weights).
// The fused form (decode_fused_kernel) runs 1 and 2 back to back in every CTA
// of one cooperative grid; an attention CTA waits only until the ids of its
// own sequences are published by the CTA that merged them.  With MXFP8 caches
// (E4M3 + E8M0 per 32 elements) 1 dequantises the index keys in registers and
// 2 dequantises each K/V block in shared memory before the same math.
// The dense run (every causal block) skips the index scan and uses
// decode_attn_kernel: split-KV CTAs staging K/V with cp.async, combined by
// the last split of each (sequence, group, head tile).
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kIdxThreads = 256;    // 8 warps
constexpr int kIdxCtasPerSm = 3;
constexpr int kIdxCtas = 148 * kIdxCtasPerSm;   // persistent index grid
constexpr int kIdxWCap = 1024;      // blocks per index CTA held in shared memory
constexpr int kIdxMaxBatch = kDecodeMaxBatch;   // sequences whose block prefix fits shared memory
constexpr int kAttnThreads = 128;   // 4 warps, 32 keys each
constexpr int kMergeRegCand = 8;    // per-lane register cache of the merge
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// MXFP8 (E4M3 element, E8M0 block scale) -> bf16.  Every E4M3 value is exact
// in f16, the scale is a power of two, and the product (at most 4 significant
// bits) is exact in bf16.
__device__ __forceinline__ float e8m0_scale(uint32_t e) {
  return e ? __int_as_float(static_cast<int>(e) << 23) : __int_as_float(0x00400000);   // 2^(e - 127)
}
__device__ __forceinline__ uint32_t dq_e4m3x2(uint32_t two_bytes, float sc) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(two_bytes)));
  float lo, hi;
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(static_cast<uint16_t>(h & 0xffffu)));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(static_cast<uint16_t>(h >> 16)));
  return pack_bf16x2(lo * sc, hi * sc);
}
// 8 E4M3 codes (one uint2, element 0 in the lowest byte) -> 8 bf16 (one uint4).
__device__ __forceinline__ uint4 dq_e4m3x8(uint2 v, float sc) {
  return make_uint4(dq_e4m3x2(v.x & 0xffffu, sc), dq_e4m3x2(v.x >> 16, sc), dq_e4m3x2(v.y & 0xffffu, sc),
                    dq_e4m3x2(v.y >> 16, sc));
}

// (score desc, block asc) order used for every selection.
__device__ __forceinline__ bool better(float s1, int b1, float s2, int b2) {
  return s1 > s2 || (s1 == s2 && static_cast<unsigned>(b1) < static_cast<unsigned>(b2));
}

struct DecArgs {
  const uint16_t* q;        // [B, h_q, d]
  const uint16_t* q_idx;    // [B, h_kv, d_idx]
  const uint16_t* k_cache;  // [sum L, h_kv, d]
  const uint16_t* v_cache;
  const uint16_t* k_idx;    // [sum L, 1, d_idx]
  const int64_t* cu_kv;     // [B + 1]
  int32_t* block_ids;       // [B, h_kv, topk]
  uint16_t* o;              // [B, h_q, d]
  float* cand_s;            // [idx_ctas + B, h_kv, kfree] top-k candidates per (CTA, sequence) share
  int* cand_b;
  float* part;              // dense: [B, h_q, splits, d + 4] (o[d], m, l, 2 pad); sparse: per-share rows
  int* seq_count;           // [B] index CTAs finished per sequence (zeroed per call)
  int* grp_count;           // [B, h_kv, head_tiles] attention CTAs finished (zeroed per call)
  int batch, h_q, h_kv, topk, causal, force_local, kfree, idx_ctas, idx_wmax;
  int splits, slots_per_split, dense, head_tiles, pool;
  float scale_log2;
  const int32_t* topk_seq;  // [B] blocks kept per sequence (adaptive k), or null: topk
  // MXFP8 caches (E4M3 codes + E8M0 scales per 32 elements of the last dim),
  // or null: the bf16 caches above.
  const uint8_t* k_idx8;    // [sum L, 1, d_idx] and scales [sum L, 1, d_idx / 32]
  const uint8_t* k_idx_sc;
  const uint8_t* k8;        // [sum L, h_kv, d] and scales [sum L, h_kv, d / 32]
  const uint8_t* k_sc;
  const uint8_t* v8;
  const uint8_t* v_sc;
};

// ---------------------------------------------------------------------------
// 1. index scan, persistent.  The blocks of all sequences, laid end to end
//    (sequence b owns global blocks [P_b, P_b+1) with P the prefix of
//    ceil(L_b / BK)), are split into idx_ctas equal contiguous ranges, one per
//    CTA, so every CTA streams the same number of index-key bytes whatever the
//    length mix.  A CTA scores its blocks (max-pool per block and group), then
//    keeps, per (sequence, group) it touched, the top (k - 1) non-local blocks
//    of its share as candidates in slot (CTA + sequence), a slot no other
//    (CTA, sequence) pair can take because both orders agree.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int idx_cta_of(long long gblk, long long T, int n) {
  return static_cast<int>(((gblk + 1) * n - 1) / T);
}

template <int BK>
__device__ void merge_topk_warp(const DecArgs& a, int b, int r, int lane, int* chosen, int c_lo, int nseg,
                                long long T, int n);

// The scan, as run by the persistent index kernel below and by the first
// phase of the fused decode kernel: ismem is the dynamic shared memory; with
// seq_ready non-null, the CTA that merges a sequence publishes its ids there.
// UNR: 16-key tiles whose loads a warp keeps in flight.  The index kernel runs
// three CTAs per SM (24 warps) at 2; the fused kernel has one CTA (8 warps)
// per SM and the whole register file, so it unrolls further to keep as many
// bytes in flight per SM.
template <int DIDX, int BK, int POOL, bool F8, int UNR = 2>
__device__ __forceinline__ void decode_index_body(const DecArgs& a, uint8_t* ismem, int* seq_ready) {
  constexpr int kHalves = DIDX / 32;   // 16-byte vectors per token row per thread
  constexpr int kWarps = kIdxThreads / 32;
  const int B = a.batch;
  const int wmax = a.idx_wmax;
  int* pfx = reinterpret_cast<int*>(ismem);                                       // [B + 1]
  float* smax = reinterpret_cast<float*>(ismem + ((B + 1) * 4 + 15) / 16 * 16);   // [h_kv][wmax]
  int* lastq = reinterpret_cast<int*>(smax + a.h_kv * wmax);                      // [wmax + 1]
  __shared__ int warp_tot[kWarps];
  __shared__ int chosen[kWarps][33];
  __shared__ int n_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n = a.idx_ctas, cta = blockIdx.x;

  // Block prefix over the sequences (each CTA builds its own copy).
  int running = 0;
  for (int base = 0; base < B; base += kIdxThreads) {
    const int bb = base + threadIdx.x;
    const int nb = bb < B ? static_cast<int>((a.cu_kv[bb + 1] - a.cu_kv[bb] + BK - 1) / BK) : 0;
    int v = nb;
#pragma unroll
    for (int x = 1; x < 32; x <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, x);
      if (lane >= x) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      tot += warp_tot[w];
    }
    if (bb < B) pfx[bb] = running + before + v - nb;
    running += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    pfx[B] = running;
    n_last = 0;
  }
  __syncthreads();
  const long long T = pfx[B];
  const int G0 = static_cast<int>(cta * T / n);
  const int W = min(static_cast<int>((cta + 1) * T / n) - G0, wmax);   // clamp: only a understated max_kv exceeds it
  if (W <= 0) return;
  const int G1 = G0 + W;
  auto seq_of = [&](int gb) {   // largest b with pfx[b] <= gb
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pfx[mid] <= gb) lo = mid; else hi = mid - 1;
    }
    return lo;
  };

  // Score: warp w takes blocks w, w + 8, ... of the range.
  int cur = -1, cur_end = 0, cur_p = 0, L = 0;
  const uint16_t* kbase = a.k_idx;
  const uint8_t* kbase8 = a.k_idx8;       // MXFP8: codes and scales of this sequence
  const uint8_t* sbase8 = a.k_idx_sc;
  uint4 qv[kHalves];
  for (int i = warp; i < W; i += kWarps) {
    const int gb = G0 + i;
    if (cur < 0 || gb >= cur_end) {
      cur = seq_of(gb);
      cur_p = pfx[cur];
      cur_end = pfx[cur + 1];
      const int64_t off = a.cu_kv[cur];
      L = static_cast<int>(a.cu_kv[cur + 1] - off);
      if (F8) {
        kbase8 = a.k_idx8 + static_cast<size_t>(off) * DIDX;
        sbase8 = a.k_idx_sc + static_cast<size_t>(off) * (DIDX / 32);
      } else {
        kbase = a.k_idx + static_cast<size_t>(off) * DIDX;
      }
      // Q_idx fragment (B operand): column n = group g, permuted d_idx order
      // (the order of the K_idx fragment below: thread t's h-th 8-vector is
      // d_idx positions 8t + 32h .. (bf16) or E t + 8h .. (MXFP8, E = d_idx / 4
      // contiguous codes per thread)).
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        qv[h] = make_uint4(0, 0, 0, 0);
        const int dpos = F8 ? (DIDX / 4) * t + 8 * h : 8 * t + 32 * h;
        if (g < a.h_kv)
          qv[h] = *reinterpret_cast<const uint4*>(a.q_idx + (static_cast<size_t>(cur) * a.h_kv + g) * DIDX + dpos);
      }
    }
    const int j0 = (gb - cur_p) * BK;
    // Groups 2t, 2t+1: running max (max-pool) or sum (mean-pool; the sum of
    // integer-valued scores is exact in fp32, in any order, below 2^24).
    float m0 = POOL ? 0.f : kNegInf, m1 = POOL ? 0.f : kNegInf;
#pragma unroll UNR
    for (int mt = 0; mt < BK / 16; ++mt) {
      const int ja = j0 + mt * 16 + g, jb = ja + 8;
      uint4 ra[kHalves], rb[kHalves];
      if (F8) {
        // Thread t's E = d_idx / 4 contiguous codes of rows ja and jb, all in
        // scale block (E t) / 32, dequantised into its kHalves 8-vectors.
        constexpr int E = DIDX / 4;
        uint32_t ca[E / 4], cb[E / 4];
#pragma unroll
        for (int v = 0; v < E / 16; ++v) {
          const uint4 x = ja < L ? ldg_nc_v4(kbase8 + static_cast<size_t>(ja) * DIDX + E * t + 16 * v) : make_uint4(0, 0, 0, 0);
          const uint4 y = jb < L ? ldg_nc_v4(kbase8 + static_cast<size_t>(jb) * DIDX + E * t + 16 * v) : make_uint4(0, 0, 0, 0);
          ca[4 * v] = x.x; ca[4 * v + 1] = x.y; ca[4 * v + 2] = x.z; ca[4 * v + 3] = x.w;
          cb[4 * v] = y.x; cb[4 * v + 1] = y.y; cb[4 * v + 2] = y.z; cb[4 * v + 3] = y.w;
        }
        if (E == 8) {
          const uint2 x = ja < L ? ldg_nc_v2(kbase8 + static_cast<size_t>(ja) * DIDX + E * t) : make_uint2(0, 0);
          const uint2 y = jb < L ? ldg_nc_v2(kbase8 + static_cast<size_t>(jb) * DIDX + E * t) : make_uint2(0, 0);
          ca[0] = x.x; ca[1] = x.y;
          cb[0] = y.x; cb[1] = y.y;
        }
        const float sca = ja < L ? e8m0_scale(sbase8[static_cast<size_t>(ja) * (DIDX / 32) + (E * t) / 32]) : 0.f;
        const float scb = jb < L ? e8m0_scale(sbase8[static_cast<size_t>(jb) * (DIDX / 32) + (E * t) / 32]) : 0.f;
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          ra[h] = dq_e4m3x8(make_uint2(ca[2 * h], ca[2 * h + 1]), sca);
          rb[h] = dq_e4m3x8(make_uint2(cb[2 * h], cb[2 * h + 1]), scb);
        }
      } else {
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          ra[h] = ja < L ? ldg_nc_v4(kbase + static_cast<size_t>(ja) * DIDX + 8 * t + 32 * h) : make_uint4(0, 0, 0, 0);
          rb[h] = jb < L ? ldg_nc_v4(kbase + static_cast<size_t>(jb) * DIDX + 8 * t + 32 * h) : make_uint4(0, 0, 0, 0);
        }
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        mma_bf16_16816(c, ra[h].x, rb[h].x, ra[h].y, rb[h].y, qv[h].x, qv[h].y);
        mma_bf16_16816(c, ra[h].z, rb[h].z, ra[h].w, rb[h].w, qv[h].z, qv[h].w);
      }
      if (POOL) {   // keys past L loaded zeros, so their scores add 0
        m0 += c[0] + c[2];
        m1 += c[1] + c[3];
      } else {
        if (ja < L) {
          m0 = fmaxf(m0, c[0]);
          m1 = fmaxf(m1, c[1]);
        }
        if (jb < L) {
          m0 = fmaxf(m0, c[2]);
          m1 = fmaxf(m1, c[3]);
        }
      }
    }
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
      const float o0 = __shfl_xor_sync(0xffffffffu, m0, x), o1 = __shfl_xor_sync(0xffffffffu, m1, x);
      m0 = POOL ? m0 + o0 : fmaxf(m0, o0);
      m1 = POOL ? m1 + o1 : fmaxf(m1, o1);
    }
    if (POOL) {
      // Mean over the block's keys, ranked in fp32: a full block divides by
      // B_k exactly, the partial last block rounds the quotient.
      const int cnt = min(BK, L - j0);
      m0 = cnt >= BK ? m0 * (1.0f / BK) : __fdiv_rn(m0, static_cast<float>(cnt));
      m1 = cnt >= BK ? m1 * (1.0f / BK) : __fdiv_rn(m1, static_cast<float>(cnt));
    }
    if (g == 0) {
      if (2 * t < a.h_kv) smax[(2 * t) * wmax + i] = m0;
      if (2 * t + 1 < a.h_kv) smax[(2 * t + 1) * wmax + i] = m1;
    }
  }
  __syncthreads();

  // Per (sequence, group) share: top-kfree non-local blocks by repeated warp
  // argmax with a strictly decreasing (score desc, block asc) bound.  Decode
  // sees every cached key (j <= p), so every block is eligible.
  const int b_first = seq_of(G0), b_last = seq_of(G1 - 1);
  const int nsegs = b_last - b_first + 1;
  for (int pi = warp; pi < nsegs * a.h_kv; pi += kWarps) {
    const int sb = b_first + pi / a.h_kv, r = pi % a.h_kv;
    const int p0 = pfx[sb];
    const int i_lo = max(p0, G0) - G0, i_hi = min(pfx[sb + 1], G1) - G0;
    const int i_loc = a.force_local ? pfx[sb + 1] - 1 - G0 : -1;   // the local block is the last one
    const size_t base = ((static_cast<size_t>(cta) + sb) * a.h_kv + r) * a.kfree;
    float last_s = __builtin_huge_valf();
    int last_b = -1;
    int k = 0;
    for (; k < a.kfree; ++k) {
      float bs = kNegInf;
      int bi = 0x7fffffff;
      for (int i = i_lo + lane; i < i_hi; i += 32) {
        if (i == i_loc) continue;
        const float sc = smax[r * wmax + i];
        const int blk = G0 + i - p0;
        if (k > 0 && !better(last_s, last_b, sc, blk)) continue;
        if (bi == 0x7fffffff || better(sc, blk, bs, bi)) { bs = sc; bi = blk; }
      }
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, x);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, x);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || better(os, oi, bs, bi))) { bs = os; bi = oi; }
      }
      if (bi == 0x7fffffff) break;
      if (lane == 0) {
        a.cand_s[base + k] = bs;
        a.cand_b[base + k] = bi;
      }
      last_s = bs;
      last_b = bi;
    }
    if (lane == 0)
      for (; k < a.kfree; ++k) {
        a.cand_s[base + k] = kNegInf;
        a.cand_b[base + k] = -1;
      }
  }

  // Arrive once per sequence touched, adding the blocks scored here; the CTA
  // that completes a sequence's block count merges it.  (Counting blocks,
  // not CTAs, keeps this right when the grid has more CTAs than blocks and
  // some ranges are empty.)
  __threadfence();
  __syncthreads();
  for (int sidx = threadIdx.x; sidx < nsegs; sidx += kIdxThreads) {
    const int sb = b_first + sidx;
    const int lo = max(pfx[sb], G0), hi = min(pfx[sb + 1], G1);
    if (atomicAdd(&a.seq_count[sb], hi - lo) + (hi - lo) == pfx[sb + 1] - pfx[sb]) lastq[atomicAdd(&n_last, 1)] = sb;
  }
  __syncthreads();
  if (n_last == 0) return;
  __threadfence();
  for (int pi = warp; pi < n_last * a.h_kv; pi += kWarps) {
    const int sb = lastq[pi / a.h_kv], r = pi % a.h_kv;
    const int c_lo = idx_cta_of(pfx[sb], T, n), c_hi = idx_cta_of(pfx[sb + 1] - 1, T, n);
    merge_topk_warp<BK>(a, sb, r, lane, chosen[warp], c_lo, c_hi - c_lo + 1, T, n);
  }
  if (seq_ready) {
    // Every group of the merged sequences is written: publish them.
    __threadfence();
    __syncthreads();
    for (int i = threadIdx.x; i < n_last; i += kIdxThreads) atomicExch(&seq_ready[lastq[i]], 1);
  }
}

template <int DIDX, int BK, int POOL, bool F8>
__global__ void __launch_bounds__(kIdxThreads, kIdxCtasPerSm) decode_index_kernel(const DecArgs a) {
  extern __shared__ __align__(16) uint8_t ismem[];
  decode_index_body<DIDX, BK, POOL, F8>(a, ismem, nullptr);
}

// ---------------------------------------------------------------------------
// 2. merge of the per-CTA candidate lists + local block -> block_ids
//    (ascending, -1 pad).  Exact: every global winner is a winner of the
//    share that holds it.
// ---------------------------------------------------------------------------
// Shares come from CTAs c_lo .. c_lo + nseg - 1 of an n-CTA grid over T
// blocks; a CTA whose range is empty wrote nothing and is skipped.
template <int BK>
__device__ void merge_topk_warp(const DecArgs& a, int b, int r, int lane, int* chosen, int c_lo, int nseg,
                                long long T, int n) {
  const int L = static_cast<int>(a.cu_kv[b + 1] - a.cu_kv[b]);
  const int b_loc = (L - 1) / BK;
  const int ncand = nseg * a.kfree;
  // Adaptive k: this sequence keeps its own number of blocks.  Every share
  // kept its top kfree >= kfree_b, so the global top kfree_b is among them.
  const int kb = a.topk_seq ? min(max(static_cast<int>(a.topk_seq[b]), 1), a.topk) : a.topk;
  const int kfree_b = min(a.kfree, kb - (a.force_local ? 1 : 0));
  // Ranges are empty only when the grid has more CTAs than blocks.
  const bool some_empty = T < n;
  auto cand_index = [&](int c) -> long long {   // -1: share of an empty range
    const int sg = c / a.kfree, slot = c - sg * a.kfree;
    const long long cc = c_lo + sg;
    if (some_empty && (cc + 1) * T / n == cc * T / n) return -1;
    return ((cc + b) * a.h_kv + r) * a.kfree + slot;
  };
  // Streaming merge: candidates arrive in chunks of 32 * kMergeRegCand (one
  // coalesced load per lane and slot) into a running top-kfree list, lane k
  // holding its k-th entry (block ids are unique across shares, so the order
  // (score desc, block asc) is strict).  The first chunk is selected by kfree
  // rounds of warp argmax; a later chunk only contributes the candidates that
  // beat the list's last entry -- few, since every share is itself sorted and
  // the list's threshold rises as it fills -- each inserted at its place by
  // one ballot and one shift.
  float run_s = kNegInf;
  int run_b = -1;
  // The next chunk's loads are issued before the current chunk is merged.
  auto load_chunk = [&](int c0, float (&cs)[kMergeRegCand], int (&cb)[kMergeRegCand]) {
#pragma unroll
    for (int i = 0; i < kMergeRegCand; ++i) {
      const int c = c0 + lane + 32 * i;
      cs[i] = kNegInf;
      cb[i] = -1;
      const long long idx = c < ncand ? cand_index(c) : -1;
      if (idx >= 0) {
        cb[i] = __ldcg(a.cand_b + idx);
        cs[i] = __ldcg(a.cand_s + idx);
      }
    }
  };
  float nx_s[kMergeRegCand];
  int nx_b[kMergeRegCand];
  if (ncand > 0) load_chunk(0, nx_s, nx_b);
  for (int c0 = 0; c0 < ncand; c0 += 32 * kMergeRegCand) {
    float cs[kMergeRegCand];
    int cb[kMergeRegCand];
#pragma unroll
    for (int i = 0; i < kMergeRegCand; ++i) {
      cs[i] = nx_s[i];
      cb[i] = nx_b[i];
    }
    if (c0 + 32 * kMergeRegCand < ncand) load_chunk(c0 + 32 * kMergeRegCand, nx_s, nx_b);
    if (c0 > 0) {
      if (kfree_b <= 0) break;
#pragma unroll
      for (int i = 0; i < kMergeRegCand; ++i) {
        const float ks = __shfl_sync(0xffffffffu, run_s, kfree_b - 1);
        const int kbl = __shfl_sync(0xffffffffu, run_b, kfree_b - 1);
        unsigned m = __ballot_sync(0xffffffffu, cb[i] >= 0 && (kbl < 0 || better(cs[i], cb[i], ks, kbl)));
        while (m) {
          const int src = __ffs(m) - 1;
          m &= m - 1;
          const float xs = __shfl_sync(0xffffffffu, cs[i], src);
          const int xb = __shfl_sync(0xffffffffu, cb[i], src);
          // Entries are sorted and empty ones come last, so the entries x
          // beats are a suffix; x goes to its first position.
          const unsigned bm =
              __ballot_sync(0xffffffffu, lane < kfree_b && (run_b < 0 || better(xs, xb, run_s, run_b)));
          if (bm == 0) continue;
          const int pos = __ffs(bm) - 1;
          const float up_s = __shfl_up_sync(0xffffffffu, run_s, 1);
          const int up_b = __shfl_up_sync(0xffffffffu, run_b, 1);
          if (lane == pos) {
            run_s = xs;
            run_b = xb;
          } else if (lane > pos && lane < kfree_b) {
            run_s = up_s;
            run_b = up_b;
          }
        }
      }
      continue;
    }
    float new_s = kNegInf;
    int new_b = -1;
    for (int k = 0; k < kfree_b; ++k) {
      float bs = run_s;
      int bi = run_b >= 0 ? run_b : 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kMergeRegCand; ++i)
        if (cb[i] >= 0 && (bi == 0x7fffffff || better(cs[i], cb[i], bs, bi))) { bs = cs[i]; bi = cb[i]; }
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, x);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, x);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || better(os, oi, bs, bi))) { bs = os; bi = oi; }
      }
      if (bi == 0x7fffffff) break;
      if (lane == k) {
        new_s = bs;
        new_b = bi;
      }
      if (run_b == bi) run_b = -1;
#pragma unroll
      for (int i = 0; i < kMergeRegCand; ++i)
        if (cb[i] == bi) cb[i] = -1;
    }
    run_s = new_s;
    run_b = new_b;
  }
  // The selected blocks (lanes 0 .. nsel0 - 1) plus the local block, written
  // ascending: each lane's place is the number of smaller ids (all distinct).
  const int nsel0 = __popc(__ballot_sync(0xffffffffu, run_b >= 0));
  const int nsel = nsel0 + (a.force_local ? 1 : 0);
  int v = run_b >= 0 ? run_b : 0x7fffffff;
  if (a.force_local && lane == nsel0) v = b_loc;
  int place = 0;
  for (int j = 0; j < nsel; ++j) place += __shfl_sync(0xffffffffu, v, j) < v;
  int32_t* out = a.block_ids + (static_cast<size_t>(b) * a.h_kv + r) * a.topk;
  if (lane < nsel) out[place] = v;
  for (int i = nsel + lane; i < a.topk; i += 32) out[i] = -1;
  (void)chosen;
}

// topk == 1 with the forced local block: no scan, every sequence's ids are
// its local block.
template <int BK>
__global__ void __launch_bounds__(32) decode_local_only_kernel(const DecArgs a) {
  __shared__ int chosen[33];
  merge_topk_warp<BK>(a, blockIdx.x / a.h_kv, blockIdx.x % a.h_kv, threadIdx.x, chosen, 0, 0, 1, 1);
}

// ---------------------------------------------------------------------------
// 3. split-KV attention over the selected (or all) blocks
// ---------------------------------------------------------------------------
// Shared-memory row layout: a row of D bf16 is D/8 16-byte chunks; chunk c of
// row x is stored at chunk position c ^ (x & 7) to keep ldmatrix conflict-free.
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int chunk) {
  return base + row * (D * 2) + ((chunk ^ (row & 7)) << 4);
}

template <int D, int BK>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const DecArgs a) {
  constexpr int kChunks = D / 8;
  constexpr int KPW = BK / 4;          // keys per warp
  constexpr int NT = KPW / 8;          // 8-key n-tiles per warp
  constexpr int KS = KPW / 16;         // 16-key PV steps per warp
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;                         // [BK][D]
  uint8_t* sV = smem + BK * D * 2;            // [BK][D]
  uint8_t* sQ = smem + 2 * BK * D * 2;        // [16][D]
  float* sML = reinterpret_cast<float*>(sQ + 16 * D * 2);   // [4 warps][16][2]
  const int split = blockIdx.x;
  const int r = blockIdx.y / a.head_tiles;
  const int ht = blockIdx.y % a.head_tiles;
  const int b = blockIdx.z;
  const int G = a.h_q / a.h_kv;
  const int rows = min(16, G - ht * 16);
  const int h0 = r * G + ht * 16;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t off = a.cu_kv[b];
  const int L = static_cast<int>(a.cu_kv[b + 1] - off);
  const int nb = (L + BK - 1) / BK;

  const int s_begin = split * a.slots_per_split;
  const int n_slots = a.dense ? nb : a.topk;
  const int s_end = min(n_slots, s_begin + a.slots_per_split);
  const int32_t* ids = a.block_ids + (static_cast<size_t>(b) * a.h_kv + r) * a.topk;
  // Next slot at or after s holding a block of this sequence (padding is -1).
  auto next_valid = [&](int s) {
    for (; s < s_end; ++s) {
      const int blk = a.dense ? s : ids[s];
      if (blk >= 0 && blk < nb) break;
    }
    return s;
  };
  // Two cp.async groups per block: K (with Q on the first block), then V, so
  // that Q K^T and the softmax run while V is still arriving.
  auto load_kv = [&](int blk, bool with_q) {
    const int j0 = blk * BK;
    if (with_q) {
      for (int c = tid; c < 16 * kChunks; c += kAttnThreads) {
        const int row = c / kChunks, ch = c % kChunks;
        cp_async16(swz<D>(smem_u32(sQ), row, ch),
                   a.q + (static_cast<size_t>(b) * a.h_q + h0 + min(row, rows - 1)) * D + ch * 8, row < rows);
      }
    }
    if (blk >= 0) {
      for (int c = tid; c < BK * kChunks; c += kAttnThreads) {
        const int row = c / kChunks, ch = c % kChunks;
        const bool ok = j0 + row < L;
        const size_t src = ((static_cast<size_t>(off) + (ok ? j0 + row : 0)) * a.h_kv + r) * D + ch * 8;
        cp_async16(swz<D>(smem_u32(sK), row, ch), a.k_cache + src, ok);
      }
    }
    cp_async_commit();
    if (blk >= 0) {
      for (int c = tid; c < BK * kChunks; c += kAttnThreads) {
        const int row = c / kChunks, ch = c % kChunks;
        const bool ok = j0 + row < L;
        const size_t src = ((static_cast<size_t>(off) + (ok ? j0 + row : 0)) * a.h_kv + r) * D + ch * 8;
        cp_async16(swz<D>(smem_u32(sV), row, ch), a.v_cache + src, ok);
      }
    }
    cp_async_commit();
  };

  int s = next_valid(s_begin);
  load_kv(s < s_end ? (a.dense ? s : ids[s]) : -1, true);
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int mi = lane >> 3, rr = lane & 7;
    const int row = (mi & 1) * 8 + rr, ch = 2 * ks + (mi >> 1);
    ldsm_x4(swz<D>(smem_u32(sQ), row, ch), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }

  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_lo = kNegInf, m_hi = kNegInf, l_lo = 0.f, l_hi = 0.f;   // rows g, g+8

  while (s < s_end) {
    const int blk = a.dense ? s : ids[s];
    const int j0 = blk * BK;

    // S = Q K^T for this warp's KPW keys (NT n-tiles of 8).
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ks += 2) {
        const int mi = lane >> 3, rr = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(swz<D>(smem_u32(sK), warp * KPW + nt * 8 + rr, 2 * ks + mi), b0, b1, b2, b3);
        mma_bf16_16816(sacc[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
        mma_bf16_16816(sacc[nt], qf[ks + 1][0], qf[ks + 1][1], qf[ks + 1][2], qf[ks + 1][3], b2, b3);
      }
    }
    // Mask keys past the sequence end; scale to log2 units; online softmax.
    float mx_lo = kNegInf, mx_hi = kNegInf;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int key = j0 + warp * KPW + nt * 8 + 2 * t;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = key + e < L;
        sacc[nt][e] = ok ? sacc[nt][e] * a.scale_log2 : kNegInf;
        sacc[nt][2 + e] = ok ? sacc[nt][2 + e] * a.scale_log2 : kNegInf;
        mx_lo = fmaxf(mx_lo, sacc[nt][e]);
        mx_hi = fmaxf(mx_hi, sacc[nt][2 + e]);
      }
    }
#pragma unroll
    for (int x = 1; x < 4; x <<= 1) {
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, x));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, x));
    }
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    const float al_lo = mn_lo == kNegInf ? 1.f : ex2_approx(m_lo - mn_lo);
    const float al_hi = mn_hi == kNegInf ? 1.f : ex2_approx(m_hi - mn_hi);
    const float bi_lo = mn_lo == kNegInf ? 0.f : mn_lo, bi_hi = mn_hi == kNegInf ? 0.f : mn_hi;
    m_lo = mn_lo;
    m_hi = mn_hi;
    float ps_lo = 0.f, ps_hi = 0.f;
    uint32_t pa[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p0 = ex2_approx(sacc[nt][0] - bi_lo), p1 = ex2_approx(sacc[nt][1] - bi_lo);
      const float p2 = ex2_approx(sacc[nt][2] - bi_hi), p3 = ex2_approx(sacc[nt][3] - bi_hi);
      ps_lo += p0 + p1;
      ps_hi += p2 + p3;
      pa[nt][0] = pack_bf16x2(p0, p1);
      pa[nt][1] = pack_bf16x2(p2, p3);
    }
    l_lo = l_lo * al_lo + ps_lo;
    l_hi = l_hi * al_hi + ps_hi;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      oacc[i][0] *= al_lo;
      oacc[i][1] *= al_lo;
      oacc[i][2] *= al_hi;
      oacc[i][3] *= al_hi;
    }
    cp_async_wait<0>();
    __syncthreads();   // V landed for every warp
    // O += P V (KS steps of 16 keys).
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const uint32_t a0 = pa[2 * kk][0], a1 = pa[2 * kk][1], a2 = pa[2 * kk + 1][0], a3 = pa[2 * kk + 1][1];
#pragma unroll
      for (int dt = 0; dt < D / 8; dt += 2) {
        const int mi = lane >> 3, rr = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(swz<D>(smem_u32(sV), warp * KPW + kk * 16 + (mi & 1) * 8 + rr, dt + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16_16816(oacc[dt], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(oacc[dt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    s = next_valid(s + 1);
    if (s < s_end) {
      __syncthreads();   // this block's K and V fully consumed
      load_kv(a.dense ? s : ids[s], false);
      cp_async_wait<1>();
      __syncthreads();
    }
  }
  cp_async_wait<0>();

  // Row sums over the 4 threads of a row.
#pragma unroll
  for (int x = 1; x < 4; x <<= 1) {
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, x);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, x);
  }
  // Combine the 4 warps (each covered a different quarter of every block).
  __syncthreads();
  if (t == 0) {
    sML[(warp * 16 + g) * 2 + 0] = m_lo;
    sML[(warp * 16 + g) * 2 + 1] = l_lo;
    sML[(warp * 16 + g + 8) * 2 + 0] = m_hi;
    sML[(warp * 16 + g + 8) * 2 + 1] = l_hi;
  }
  __syncthreads();
  float M_lo = kNegInf, M_hi = kNegInf;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    M_lo = fmaxf(M_lo, sML[(w * 16 + g) * 2]);
    M_hi = fmaxf(M_hi, sML[(w * 16 + g + 8) * 2]);
  }
  const float sc_lo = m_lo == kNegInf ? 0.f : ex2_approx(m_lo - M_lo);
  const float sc_hi = m_hi == kNegInf ? 0.f : ex2_approx(m_hi - M_hi);
  float* sO = reinterpret_cast<float*>(smem);   // [4][16][D] fp32, over the K/V buffers
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) {
    const int col = dt * 8 + 2 * t;
    sO[(warp * 16 + g) * D + col] = oacc[dt][0] * sc_lo;
    sO[(warp * 16 + g) * D + col + 1] = oacc[dt][1] * sc_lo;
    sO[(warp * 16 + g + 8) * D + col] = oacc[dt][2] * sc_hi;
    sO[(warp * 16 + g + 8) * D + col + 1] = oacc[dt][3] * sc_hi;
  }
  __syncthreads();
  const size_t stride = D + 4;   // 16-byte rows for the float4 combine
  for (int e = tid; e < 16 * D; e += kAttnThreads) {
    const int row = e / D, col = e % D;
    if (row >= rows) continue;
    const float v = sO[(0 * 16 + row) * D + col] + sO[(1 * 16 + row) * D + col] + sO[(2 * 16 + row) * D + col] +
                    sO[(3 * 16 + row) * D + col];
    a.part[((static_cast<size_t>(b) * a.h_q + h0 + row) * a.splits + split) * stride + col] = v;
  }
  if (tid < rows) {
    const int row = tid;
    float M = kNegInf, Lsum = 0.f;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sML[(w * 16 + row) * 2]);
    for (int w = 0; w < 4; ++w) {
      const float mw = sML[(w * 16 + row) * 2];
      if (mw != kNegInf) Lsum += sML[(w * 16 + row) * 2 + 1] * ex2_approx(mw - M);
    }
    float* pp = a.part + ((static_cast<size_t>(b) * a.h_q + h0 + row) * a.splits + split) * stride;
    pp[D] = M;
    pp[D + 1] = Lsum;
  }
  // The last split CTA of this (sequence, group, head tile) combines: per
  // row, weights w_s = exp2(m_s - M) / sum_s w_s l_s, then O = sum_s w_s o_s.
  __shared__ int s_last;
  __shared__ float s_w[16][32];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&a.grp_count[blockIdx.z * gridDim.y + blockIdx.y], 1) == a.splits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* pbase = a.part + (static_cast<size_t>(b) * a.h_q + h0) * a.splits * stride;
  for (int row = warp; row < rows; row += kAttnThreads / 32) {
    const float* pr = pbase + static_cast<size_t>(row) * a.splits * stride;
    const float m = lane < a.splits ? __ldcg(pr + lane * stride + D) : kNegInf;
    const float l = lane < a.splits ? __ldcg(pr + lane * stride + D + 1) : 0.f;
    float M = m;
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    const float w = (m == kNegInf) ? 0.f : ex2_approx(m - M);
    float den = w * l;
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) den += __shfl_xor_sync(0xffffffffu, den, x);
    s_w[row][lane] = den > 0.f ? w / den : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < rows * (D / 4); e += kAttnThreads) {
    const int row = e / (D / 4), c4 = e % (D / 4);
    const float* pr = pbase + static_cast<size_t>(row) * a.splits * stride + c4 * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int sp = 0; sp < a.splits; ++sp) {
      const float ws = s_w[row][sp];
      const float4 v = __ldcg(reinterpret_cast<const float4*>(pr + sp * stride));
      acc.x += ws * v.x;
      acc.y += ws * v.y;
      acc.z += ws * v.z;
      acc.w += ws * v.w;
    }
    uint2 out;
    out.x = pack_bf16x2(acc.x, acc.y);
    out.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(a.o + (static_cast<size_t>(b) * a.h_q + h0 + row) * D + c4 * 4) = out;
  }
}

// ---------------------------------------------------------------------------
// 3s. sparse decode attention, persistent and TMA-fed
// ---------------------------------------------------------------------------
// Work is a flat list of items g = u * topk + slot over units
// u = (b, r, head tile); a grid of kStreamCtas CTAs gives CTA c the contiguous
// range [c T / n, (c + 1) T / n), so every SM streams the same number of K/V
// blocks whatever the batch and selection look like.  Per CTA: one producer
// warp issues TMA loads (Q tile, K block, V block) into a ring of stages;
// four consumer warps run the online softmax on mma.sync.  Warp w computes
// S for keys [w BK/4, (w+1) BK/4) of the block, the four warps agree on the
// row maxima through shared memory, write P (bf16) to shared memory, and warp
// w then accumulates O for output columns [w D/4, (w+1) D/4) over the whole
// block, so no cross-warp reduction of O is ever needed.  A unit that lies in
// one CTA is normalised and written directly; a unit split between CTAs
// leaves an (o, m, l) partial per CTA and the last of them to finish merges.
constexpr int kStreamConsumers = 4;
constexpr int kStreamThreads = 32 * (kStreamConsumers + 1);
constexpr int kStreamCtas = 148;       // persistent grid: one CTA per SM
constexpr int kStreamIdsCap = 1024;    // items per CTA held in shared memory

template <int D, int BK, bool F8 = false>
struct StreamCfg {
  static constexpr int kHalves = D / 64;                  // 128-byte column halves
  static constexpr int kQBytes = 16 * 128 * kHalves;      // 16 head rows x D
  static constexpr int kKBytes = BK * 128 * kHalves;      // BK keys x D (bf16)
  // MXFP8 caches: the stage holds E4M3 K and V blocks (BK x D bytes each,
  // 128B-swizzled rows of D bytes) and their scales (BK x D/32 bytes each);
  // the consumers dequantise a stage into one bf16 K/V tile pair (kDeqBytes).
  static constexpr int kK8Bytes = BK * D;
  static constexpr int kScBytes = BK * (D / 32);
  static constexpr int kStageBytes =
      F8 ? ((kQBytes + 2 * kK8Bytes + 2 * kScBytes + 1023) / 1024) * 1024 : kQBytes + 2 * kKBytes;
  static constexpr int kDeqBytes = F8 ? 2 * kKBytes : 0;
  static constexpr int kFit = (212 * 1024 - kDeqBytes) / kStageBytes;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;
  static constexpr int kPBytes = 16 * BK * 2;
  static constexpr int kOffDeq = kStages * kStageBytes;
  static constexpr int kOffP = kOffDeq + kDeqBytes;
  static constexpr int kOffRed = kOffP + kPBytes;                       // red_m[4][16], red_l[4][16]
  static constexpr int kOffIds = kOffRed + 2 * kStreamConsumers * 16 * 4;
  static constexpr int kOffMeta = kOffIds + kStreamIdsCap * 4;          // int4 per stage
  static constexpr int kOffBar = kOffMeta + kStages * 16;               // full[], empty[]
  static constexpr int kOffFlags = kOffBar + 2 * kStages * 8;
  static constexpr int kSmemBytes = kOffFlags + 16;
  static_assert(kStages >= 2, "stage ring");
  static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory");
};

struct StreamArgs {
  const int32_t* block_ids;   // [B, h_kv, topk]
  const int64_t* cu_kv;       // [B + 1]
  uint16_t* o;                // [B, h_q, d]
  float* part;                // [n_cta + U][16][d + 4]
  int* unit_count;            // [U] CTAs finished per unit (zeroed per call)
  int* status;
  long long total_items;      // T = U * topk
  int n_cta, h_q, h_kv, topk, head_tiles, group;
  float scale_log2;
  const uint8_t* k_sc;        // MXFP8 caches: E8M0 scales [sum L, h_kv, d / 32] (null for bf16)
  const uint8_t* v_sc;
};

// Byte offset of 16-byte chunk ch of row x in a TMA 128B-swizzled tile of
// `rows` rows stored as D/64 column halves of rows x 128 bytes.
__device__ __forceinline__ uint32_t sw128(uint32_t base, int rows, int x, int ch) {
  return base + (ch >> 3) * rows * 128 + x * 128 + (((ch & 7) ^ (x & 7)) << 4);
}

__device__ __forceinline__ int cta_of_item(long long g, long long T, int n) {
  return static_cast<int>(((g + 1) * n - 1) / T);
}

// The attention, as run by the streaming kernel below and by the second
// phase of the fused decode kernel (smem_raw: the dynamic shared memory;
// seq_ready non-null: wait until the ids of this CTA's sequences are out).
// Warps past the producer take no part.
template <int D, int BK, bool F8>
__device__ __forceinline__ void decode_attn_body(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                                 const CUtensorMap* tm_v, const StreamArgs& a, uint8_t* smem_raw,
                                                 const int* seq_ready) {
  using C = StreamCfg<D, BK, F8>;
  constexpr int KPW = BK / kStreamConsumers;   // S keys per warp
  constexpr int NT = KPW / 8;
  constexpr int NCOL = D / kStreamConsumers;   // O columns per warp
  constexpr int NTO = NCOL / 8;
  constexpr int PST = D + 4;                   // partial row stride (floats)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red_m = reinterpret_cast<float*>(smem + C::kOffRed);
  float* red_l = red_m + kStreamConsumers * 16;
  int* s_ids = reinterpret_cast<int*>(smem + C::kOffIds);
  int4* meta = reinterpret_cast<int4*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::kStages;
  int* flags = reinterpret_cast<int*>(smem + C::kOffFlags);   // [0] abort, [1] last
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sP = sbase + C::kOffP;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long T = a.total_items;
  const int cta = blockIdx.x;
  // CTAs past n_cta (the fused grid is one CTA per SM, n_cta <= T) hold no
  // items: every CTA inside a unit's span then holds at least one of its
  // items, which the last-arriver count of a split unit relies on.
  const long long g0 = cta < a.n_cta ? cta * T / a.n_cta : T;
  const long long g1 = cta < a.n_cta ? (cta + 1) * T / a.n_cta : T;
  const int n_items = static_cast<int>(g1 - g0);
  const int upb = a.h_kv * a.head_tiles;   // units per sequence

  if (seq_ready) {
    // Fused step: the ids of this CTA's sequences come from the index phase
    // of (possibly) other CTAs; wait, bounded, for each to be published.
    if (tid == 0 && n_items > 0) {
      const int b_lo = static_cast<int>((g0 / a.topk) / upb), b_hi = static_cast<int>(((g1 - 1) / a.topk) / upb);
      const unsigned long long t0 = globaltimer();
      for (int b = b_lo; b <= b_hi; ++b) {
        while (atomicAdd(const_cast<int*>(&seq_ready[b]), 0) == 0) {
          if (globaltimer() - t0 > kWaitNs) {
            if (a.status) atomicExch(a.status, kDevTimeout);
            break;
          }
          __nanosleep(256);
        }
      }
      __threadfence();
    }
    __syncthreads();
  }
  // Block ids of this CTA's items, -1 where the slot is padding or out of range.
  for (int i = tid; i < n_items; i += blockDim.x) {
    const long long g = g0 + i;
    const long long u = g / a.topk;
    const int slot = static_cast<int>(g - u * a.topk);
    const int b = static_cast<int>(u / upb), r = static_cast<int>(u % upb) / a.head_tiles;
    const int L = static_cast<int>(a.cu_kv[b + 1] - a.cu_kv[b]);
    const int nb = (L + BK - 1) / BK;
    const int blk = __ldcg(a.block_ids + (static_cast<size_t>(b) * a.h_kv + r) * a.topk + slot);
    s_ids[i] = (blk >= 0 && blk < nb) ? blk : -1;
  }
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // MXFP8: the TMA bytes, then one cp.async arrival per producer lane
      // once its share of the block's scales has landed.
      mbar_init(&full[s], F8 ? 33 : 1);
      mbar_init(&empty[s], kStreamConsumers);
    }
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  WaitCtx wc{reinterpret_cast<volatile int*>(&flags[0]), a.status};
  if (warp > kStreamConsumers) return;

  if (warp == kStreamConsumers) {
    // ---------------- producer ----------------
    // Lane 0 waits for a free stage and issues the TMA loads; with MXFP8
    // caches the whole warp then gathers the K and V scales of the block into
    // the stage (a second arrival on its full barrier).
    if (!F8 && lane != 0) return;
    if (lane == 0) {
      tma_prefetch_desc(tm_q);
      tma_prefetch_desc(tm_k);
      tma_prefetch_desc(tm_v);
    }
    long long cur_u = -1;
    long long off = 0;
    int L = 0, qrow = 0, r = 0;
    int issued = 0;
    for (int i = 0; i < n_items; ++i) {
      const int blk = s_ids[i];
      if (blk < 0) continue;
      const long long u = (g0 + i) / a.topk;
      if (u != cur_u) {
        const int b = static_cast<int>(u / upb), rt = static_cast<int>(u % upb);
        r = rt / a.head_tiles;
        qrow = b * a.h_q + r * a.group + (rt % a.head_tiles) * 16;
        off = a.cu_kv[b];
        L = static_cast<int>(a.cu_kv[b + 1] - off);
        cur_u = u;
      }
      const int stage = issued % C::kStages;
      const uint32_t ph = (issued / C::kStages) & 1;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[stage], ph ^ 1, wc);
      if (F8) ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int j0 = blk * BK;
      // The last (partial) block is fetched as the BK keys ending at L, so no
      // box reaches past this sequence; rows before j0 are masked.
      const int kbase = j0 + BK <= L ? j0 : L - BK;
      uint8_t* st = smem + stage * C::kStageBytes;
      const int krow = static_cast<int>(off + kbase);
      if (lane == 0) {
        meta[stage] = make_int4(j0, kbase, min(j0 + BK, L), 0);
        if (F8) {
          mbar_arrive_expect_tx(&full[stage], C::kQBytes + 2 * C::kK8Bytes);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) tma_load_2d(st + h * 16 * 128, tm_q, &full[stage], h * 64, qrow);
          tma_load_3d(st + C::kQBytes, tm_k, &full[stage], 0, r, krow);
          tma_load_3d(st + C::kQBytes + C::kK8Bytes, tm_v, &full[stage], 0, r, krow);
        } else {
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            tma_load_2d(st + h * 16 * 128, tm_q, &full[stage], h * 64, qrow);
            tma_load_3d(st + C::kQBytes + h * BK * 128, tm_k, &full[stage], h * 64, r, krow);
            tma_load_3d(st + C::kQBytes + C::kKBytes + h * BK * 128, tm_v, &full[stage], h * 64, r, krow);
          }
        }
      }
      if (F8) {
        // Scales of keys krow .. krow + BK - 1 of group r (D/32 = 4 bytes per
        // key), copied asynchronously; each lane's arrival on the stage's full
        // barrier fires when its copies have landed.
        static_assert(!F8 || D / 32 == 4, "MXFP8 decode: 4 scale bytes per key row");
        const uint32_t ssc = smem_u32(st + C::kQBytes + 2 * C::kK8Bytes);
        for (int x = lane; x < BK; x += 32) {
          const size_t at = ((static_cast<size_t>(krow) + x) * a.h_kv + r) * 4;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ssc + x * 4), "l"(a.k_sc + at) : "memory");
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ssc + C::kScBytes + x * 4), "l"(a.v_sc + at)
                       : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[stage])) : "memory");
      }
      ++issued;
    }
    // Loads still in flight (only possible after an abort) land before exit.
    if (F8) asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      WaitCtx drain{reinterpret_cast<volatile int*>(&flags[2]), a.status};
      for (int k = issued > C::kStages ? issued - C::kStages : 0; k < issued; ++k)
        mbar_wait(&full[k % C::kStages], (k / C::kStages) & 1, drain);
    }
    return;
  }

  // ---------------- consumers (warps 0..3) ----------------
  const int g = lane >> 2, t = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  float oacc[NTO][4];
  float m_lo = kNegInf, m_hi = kNegInf, l_lo = 0.f, l_hi = 0.f;
#pragma unroll
  for (int i = 0; i < NTO; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  int consumed = 0;

  for (int i = 0; i < n_items; ++i) {
    const long long gi = g0 + i;
    const long long u = gi / a.topk;
    if (s_ids[i] >= 0) {
      const int stage = consumed % C::kStages;
      const uint32_t ph = (consumed / C::kStages) & 1;
      ++consumed;
      mbar_wait(&full[stage], ph, wc);   // on timeout the flag is set and the data is ignored
      const int4 md = meta[stage];
      const int j0 = md.x, kbase = md.y, jend = md.z;
      const uint32_t sQ = sbase + stage * C::kStageBytes;
      uint32_t sK = sQ + C::kQBytes;
      uint32_t sV = sK + C::kKBytes;
      if (F8) {
        // Dequantise the stage's E4M3 K and V blocks into the bf16 tile pair
        // (the layout the bf16 path reads: 128B-swizzled rows of D/64 column
        // halves).  The previous item's S and PV have finished with that pair
        // (every consumer warp is past the barrier); the stage itself, which
        // still holds the Q tile, is released at the end of the item.
        sK = sbase + C::kOffDeq;
        sV = sK + C::kKBytes;
        named_bar(1, 32 * kStreamConsumers);
        const uint8_t* s8 = smem + stage * C::kStageBytes + C::kQBytes;
        const uint8_t* ssc = s8 + 2 * C::kK8Bytes;
        constexpr int CPR = D / 16;                      // 16-byte chunks per E4M3 row
        // Four chunks in flight per thread: the loop is bound by the latency of
        // its shared-memory loads, not by the conversions.
#pragma unroll 4
        for (int e = tid; e < 2 * BK * CPR; e += 32 * kStreamConsumers) {
          const int kv = e / (BK * CPR), rem = e - kv * (BK * CPR);
          const int x = rem / CPR, c = rem - x * CPR;   // row, chunk (16 elements from column 16c)
          // E4M3 rows of D = 128 bytes, 128B-swizzled by TMA (16-byte chunk c of row x at c ^ (x & 7)).
          const uint4 raw = *reinterpret_cast<const uint4*>(s8 + kv * C::kK8Bytes + x * D + ((c ^ (x & 7)) << 4));
          const float sc = e8m0_scale(ssc[kv * C::kScBytes + x * (D / 32) + c / 2]);
          const uint4 lo = dq_e4m3x8(make_uint2(raw.x, raw.y), sc), hi = dq_e4m3x8(make_uint2(raw.z, raw.w), sc);
          const uint32_t dst = (kv ? sV : sK);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sw128(dst, BK, x, 2 * c)), "r"(lo.x),
                       "r"(lo.y), "r"(lo.z), "r"(lo.w)
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sw128(dst, BK, x, 2 * c + 1)), "r"(hi.x),
                       "r"(hi.y), "r"(hi.z), "r"(hi.w)
                       : "memory");
        }
        named_bar(1, 32 * kStreamConsumers);
      }

      uint32_t qf[D / 16][4];
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        ldsm_x4(sw128(sQ, 16, (mi & 1) * 8 + rr, 2 * ks + (mi >> 1)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sw128(sK, BK, warp * KPW + nt * 8 + rr, 2 * ks + mi), b0, b1, b2, b3);
          mma_bf16_16816(sacc[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
          mma_bf16_16816(sacc[nt], qf[ks + 1][0], qf[ks + 1][1], qf[ks + 1][2], qf[ks + 1][3], b2, b3);
        }
      }
      float mx_lo = kNegInf, mx_hi = kNegInf;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = kbase + warp * KPW + nt * 8 + 2 * t + e;
          const bool ok = key >= j0 && key < jend;
          sacc[nt][e] = ok ? sacc[nt][e] * a.scale_log2 : kNegInf;
          sacc[nt][2 + e] = ok ? sacc[nt][2 + e] * a.scale_log2 : kNegInf;
          mx_lo = fmaxf(mx_lo, sacc[nt][e]);
          mx_hi = fmaxf(mx_hi, sacc[nt][2 + e]);
        }
      }
#pragma unroll
      for (int x = 1; x < 4; x <<= 1) {
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, x));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, x));
      }
      if (t == 0) {
        red_m[warp * 16 + g] = mx_lo;
        red_m[warp * 16 + g + 8] = mx_hi;
      }
      named_bar(1, 32 * kStreamConsumers);
#pragma unroll
      for (int w = 0; w < kStreamConsumers; ++w) {
        mx_lo = fmaxf(mx_lo, red_m[w * 16 + g]);
        mx_hi = fmaxf(mx_hi, red_m[w * 16 + g + 8]);
      }
      const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
      const float al_lo = mn_lo == kNegInf ? 1.f : ex2_approx(m_lo - mn_lo);
      const float al_hi = mn_hi == kNegInf ? 1.f : ex2_approx(m_hi - mn_hi);
      const float bi_lo = mn_lo == kNegInf ? 0.f : mn_lo, bi_hi = mn_hi == kNegInf ? 0.f : mn_hi;
      m_lo = mn_lo;
      m_hi = mn_hi;
      float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float p0 = ex2_approx(sacc[nt][0] - bi_lo), p1 = ex2_approx(sacc[nt][1] - bi_lo);
        const float p2 = ex2_approx(sacc[nt][2] - bi_hi), p3 = ex2_approx(sacc[nt][3] - bi_hi);
        ps_lo += p0 + p1;
        ps_hi += p2 + p3;
        const int ch = warp * NT + nt;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + g * (BK * 2) + ((ch ^ (g & 7)) << 4) + 4 * t),
                     "r"(pack_bf16x2(p0, p1)));
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + (g + 8) * (BK * 2) + ((ch ^ (g & 7)) << 4) + 4 * t),
                     "r"(pack_bf16x2(p2, p3)));
      }
#pragma unroll
      for (int x = 1; x < 4; x <<= 1) {
        ps_lo += __shfl_xor_sync(0xffffffffu, ps_lo, x);
        ps_hi += __shfl_xor_sync(0xffffffffu, ps_hi, x);
      }
      if (t == 0) {
        red_l[warp * 16 + g] = ps_lo;
        red_l[warp * 16 + g + 8] = ps_hi;
      }
      // Rows of a partial block before j0 hold other keys: zero this warp's
      // V columns there so that 0 * V stays 0 whatever those rows contain.
      const bool zap = kbase < j0;
      if (zap) {
        const int nz = j0 - kbase;
        for (int e = lane; e < nz * NTO; e += 32) {
          const int x = e / NTO, ch = warp * NTO + e % NTO;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sw128(sV, BK, x, ch)), "r"(0u)
                       : "memory");
        }
      }
      named_bar(1, 32 * kStreamConsumers);
      float ls_lo = 0.f, ls_hi = 0.f;
#pragma unroll
      for (int w = 0; w < kStreamConsumers; ++w) {
        ls_lo += red_l[w * 16 + g];
        ls_hi += red_l[w * 16 + g + 8];
      }
      l_lo = l_lo * al_lo + ls_lo;
      l_hi = l_hi * al_hi + ls_hi;
#pragma unroll
      for (int i2 = 0; i2 < NTO; ++i2) {
        oacc[i2][0] *= al_lo;
        oacc[i2][1] *= al_lo;
        oacc[i2][2] *= al_hi;
        oacc[i2][3] *= al_hi;
      }
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        const int prow = (mi & 1) * 8 + rr, pch = 2 * kk + (mi >> 1);
        ldsm_x4(sP + prow * (BK * 2) + ((pch ^ (prow & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int dt = 0; dt < NTO; dt += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sw128(sV, BK, kk * 16 + (mi & 1) * 8 + rr, warp * NTO + dt + (mi >> 1)), b0, b1, b2, b3);
          mma_bf16_16816(oacc[dt], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(oacc[dt + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      if (!F8 && zap) fence_proxy_async_smem();   // generic writes before the stage's next TMA fill
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }

    // End of this CTA's share of unit u: write it out.
    if ((gi + 1) % a.topk != 0 && i + 1 != n_items) continue;
    const int b = static_cast<int>(u / upb), rt = static_cast<int>(u % upb);
    const int r = rt / a.head_tiles, ht = rt % a.head_tiles;
    const int rows = min(16, a.group - ht * 16);
    const int h0 = r * a.group + ht * 16;
    const int c_lo = cta_of_item(u * a.topk, T, a.n_cta);
    const int c_hi = cta_of_item(u * a.topk + a.topk - 1, T, a.n_cta);
    uint16_t* orow = a.o + (static_cast<size_t>(b) * a.h_q + h0) * D;
    if (c_lo == c_hi) {
      const float in_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, in_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
#pragma unroll
      for (int dt = 0; dt < NTO; ++dt) {
        const int col = warp * NCOL + dt * 8 + 2 * t;
        if (g < rows)
          *reinterpret_cast<uint32_t*>(orow + g * D + col) = pack_bf16x2(oacc[dt][0] * in_lo, oacc[dt][1] * in_lo);
        if (g + 8 < rows)
          *reinterpret_cast<uint32_t*>(orow + (g + 8) * D + col) =
              pack_bf16x2(oacc[dt][2] * in_hi, oacc[dt][3] * in_hi);
      }
    } else {
      float* pp = a.part + (static_cast<size_t>(cta) + u) * 16 * PST;
#pragma unroll
      for (int dt = 0; dt < NTO; ++dt) {
        const int col = warp * NCOL + dt * 8 + 2 * t;
        *reinterpret_cast<float2*>(pp + g * PST + col) = make_float2(oacc[dt][0], oacc[dt][1]);
        *reinterpret_cast<float2*>(pp + (g + 8) * PST + col) = make_float2(oacc[dt][2], oacc[dt][3]);
      }
      if (warp == 0 && t == 0) {
        *reinterpret_cast<float2*>(pp + g * PST + D) = make_float2(m_lo, l_lo);
        *reinterpret_cast<float2*>(pp + (g + 8) * PST + D) = make_float2(m_hi, l_hi);
      }
      __threadfence();
      named_bar(1, 32 * kStreamConsumers);
      if (tid == 0) {
        flags[1] = atomicAdd(&a.unit_count[u], 1) == c_hi - c_lo;
        __threadfence();
      }
      named_bar(1, 32 * kStreamConsumers);
      if (flags[1]) {
        // Last CTA of the unit: LSE-weighted merge of the c_hi - c_lo + 1 partials.
        float M_lo = kNegInf, M_hi = kNegInf;
        for (int c = c_lo; c <= c_hi; ++c) {
          const float* q = a.part + (static_cast<size_t>(c) + u) * 16 * PST;
          M_lo = fmaxf(M_lo, __ldcg(q + g * PST + D));
          M_hi = fmaxf(M_hi, __ldcg(q + (g + 8) * PST + D));
        }
        float acc[NTO][4];
#pragma unroll
        for (int dt = 0; dt < NTO; ++dt) acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
        float den_lo = 0.f, den_hi = 0.f;
        for (int c = c_lo; c <= c_hi; ++c) {
          const float* q = a.part + (static_cast<size_t>(c) + u) * 16 * PST;
          const float2 ml_lo = __ldcg(reinterpret_cast<const float2*>(q + g * PST + D));
          const float2 ml_hi = __ldcg(reinterpret_cast<const float2*>(q + (g + 8) * PST + D));
          const float w_lo = ml_lo.x == kNegInf ? 0.f : ex2_approx(ml_lo.x - M_lo);
          const float w_hi = ml_hi.x == kNegInf ? 0.f : ex2_approx(ml_hi.x - M_hi);
          den_lo += w_lo * ml_lo.y;
          den_hi += w_hi * ml_hi.y;
#pragma unroll
          for (int dt = 0; dt < NTO; ++dt) {
            const int col = warp * NCOL + dt * 8 + 2 * t;
            const float2 v0 = __ldcg(reinterpret_cast<const float2*>(q + g * PST + col));
            const float2 v1 = __ldcg(reinterpret_cast<const float2*>(q + (g + 8) * PST + col));
            acc[dt][0] += w_lo * v0.x;
            acc[dt][1] += w_lo * v0.y;
            acc[dt][2] += w_hi * v1.x;
            acc[dt][3] += w_hi * v1.y;
          }
        }
        const float in_lo = den_lo > 0.f ? 1.f / den_lo : 0.f, in_hi = den_hi > 0.f ? 1.f / den_hi : 0.f;
#pragma unroll
        for (int dt = 0; dt < NTO; ++dt) {
          const int col = warp * NCOL + dt * 8 + 2 * t;
          if (g < rows)
            *reinterpret_cast<uint32_t*>(orow + g * D + col) = pack_bf16x2(acc[dt][0] * in_lo, acc[dt][1] * in_lo);
          if (g + 8 < rows)
            *reinterpret_cast<uint32_t*>(orow + (g + 8) * D + col) =
                pack_bf16x2(acc[dt][2] * in_hi, acc[dt][3] * in_hi);
        }
      }
    }
    m_lo = m_hi = kNegInf;
    l_lo = l_hi = 0.f;
#pragma unroll
    for (int i2 = 0; i2 < NTO; ++i2) oacc[i2][0] = oacc[i2][1] = oacc[i2][2] = oacc[i2][3] = 0.f;
  }
}

template <int D, int BK, bool F8>
__global__ void __launch_bounds__(kStreamThreads, 1)
    decode_attn_stream_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const StreamArgs a) {
  extern __shared__ uint8_t smem_raw[];
  decode_attn_body<D, BK, F8>(&tm_q, &tm_k, &tm_v, a, smem_raw, nullptr);
}

// ---------------------------------------------------------------------------
// 4. fused decode step: one cooperative persistent launch, one CTA per SM.
//    Phase 1 is the index scan above over this grid (the CTA that completes
//    a sequence merges its top-k and publishes it in seq_ready); phase 2 is
//    the streaming attention above, whose CTAs wait (bounded) until the ids
//    of their own sequences are published -- CTAs whose sequences finish
//    early start attending while others still scan, and the ids never leave
//    the L2 between the two.  All CTAs are co-resident (cooperative launch),
//    and a publishing CTA never waits on anyone, so every wait ends.
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = kIdxThreads;   // the scan's 8 warps; the attention uses 5 of them
// Tiles in flight per warp in the fused scan: up to 32 16-byte loads a thread.
template <int DIDX, int BK>
constexpr int kFusedUnroll = (BK / 16) < 16 / (DIDX / 32) ? (BK / 16) : 16 / (DIDX / 32);

template <int DIDX, int BK, int POOL, int D, bool F8>
__global__ void __launch_bounds__(kFusedThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecArgs a, const StreamArgs sa,
                        int* seq_ready) {
  extern __shared__ __align__(1024) uint8_t fsmem[];
  decode_index_body<DIDX, BK, POOL, F8, kFusedUnroll<DIDX, BK>>(a, fsmem, seq_ready);
  __syncthreads();   // the scan's shared memory is reused by the attention
  decode_attn_body<D, BK, F8>(&tm_q, &tm_k, &tm_v, sa, fsmem, seq_ready);
}

// Split plan of the dense run, shared by the workspace query and the launch.
struct SplitPlan {
  int splits, slots_per_split;
};

SplitPlan plan_dense_splits(const msa_params& p, int max_kv) {
  SplitPlan s;
  const int nb = (max_kv + p.block_k - 1) / p.block_k;
  s.splits = nb < 32 ? nb : 32;
  s.slots_per_split = (nb + s.splits - 1) / s.splits;
  return s;
}

// Index grid: at least kIdxCtas CTAs, and enough that no CTA holds more than
// kIdxWCap blocks when every sequence is max_kv long.
struct IdxPlan {
  int ctas, wmax;
  size_t smem;
};

IdxPlan plan_index(const msa_params& p, int batch, int max_kv) {
  IdxPlan ip;
  const long long tmax = static_cast<long long>(batch) * ((max_kv + p.block_k - 1) / p.block_k);
  long long n = (tmax + kIdxWCap - 1) / kIdxWCap;
  if (n < kIdxCtas) n = kIdxCtas;
  ip.ctas = static_cast<int>(n);
  ip.wmax = static_cast<int>((tmax + n - 1) / n);
  if (ip.wmax < 1) ip.wmax = 1;
  ip.smem = align_up(static_cast<size_t>(batch + 1) * 4, 16) + static_cast<size_t>(p.h_kv) * ip.wmax * 4 +
            static_cast<size_t>(ip.wmax + 1) * 4;
  return ip;
}

template <int D, int BK>
int launch_attn_combine(const DecArgs& a, cudaStream_t st) {
  const int smem = 2 * BK * D * 2 + 16 * D * 2 + 4 * 16 * 2 * 4;
  auto kern = decode_attn_kernel<D, BK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MSA_ERR_CUDA;
  dim3 grid(a.splits, a.h_kv * a.head_tiles, a.batch);
  kern<<<grid, kAttnThreads, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

long long stream_items(const msa_params& p, int batch) {
  return static_cast<long long>(batch) * p.h_kv * ((p.h_q / p.h_kv + 15) / 16) * p.topk;
}

int stream_ctas(long long T) {
  long long n = (T + kStreamIdsCap - 1) / kStreamIdsCap;
  if (n < kStreamCtas) n = kStreamCtas;
  return static_cast<int>(n < T ? n : T);
}

// Tensor maps and arguments of the streaming attention over n_cta CTAs.
template <int D, int BK, bool F8>
int stream_setup(const DecArgs& a, int max_kv, int* status, CUtensorMap& tq, CUtensorMap& tk, CUtensorMap& tv,
                 StreamArgs& s) {
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.batch) * a.h_q};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64, 16};
    if (!encode_tma_bf16(&tq, 2, a.q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
  }
  {
    // Rows of the packed caches: the sum of L_b is at most batch * max_kv.
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.h_kv),
                              static_cast<uint64_t>(a.batch) * max_kv};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(a.h_kv) * D * 2};
    if (F8) {   // E4M3 codes: one byte per element, a whole D = 128-byte row per box row
      const uint64_t strides8[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.h_kv) * D};
      const uint32_t box8[3] = {D, 1, BK};
      if (!encode_tma_u8(&tk, 3, a.k8, dims, strides8, box8, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
      if (!encode_tma_u8(&tv, 3, a.v8, dims, strides8, box8, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
    } else {
      const uint32_t box[3] = {64, 1, BK};
      if (!encode_tma_bf16(&tk, 3, a.k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
      if (!encode_tma_bf16(&tv, 3, a.v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MSA_ERR_CUDA;
    }
  }
  s.block_ids = a.block_ids;
  s.cu_kv = a.cu_kv;
  s.o = a.o;
  s.part = a.part;
  s.unit_count = a.grp_count;
  s.status = status;
  s.total_items = static_cast<long long>(a.batch) * a.h_kv * a.head_tiles * a.topk;
  s.n_cta = stream_ctas(s.total_items);
  s.h_q = a.h_q;
  s.h_kv = a.h_kv;
  s.topk = a.topk;
  s.head_tiles = a.head_tiles;
  s.group = a.h_q / a.h_kv;
  s.scale_log2 = a.scale_log2;
  s.k_sc = a.k_sc;
  s.v_sc = a.v_sc;
  return MSA_OK;
}

template <int D, int BK, bool F8>
int launch_attn_stream(const DecArgs& a, int max_kv, int* status, cudaStream_t st) {
  using C = StreamCfg<D, BK, F8>;
  CUtensorMap tq, tk, tv;
  StreamArgs s;
  int rc = stream_setup<D, BK, F8>(a, max_kv, status, tq, tk, tv, s);
  if (rc) return rc;
  const int smem = C::kSmemBytes + 1024;
  auto kern = decode_attn_stream_kernel<D, BK, F8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MSA_ERR_CUDA;
  kern<<<s.n_cta, kStreamThreads, smem, st>>>(tq, tk, tv, s);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

// The fused step (decode_fused_kernel), when the whole step fits one
// co-resident wave: every attention CTA holds its items' ids in shared memory
// (kStreamIdsCap) and every scan CTA its blocks' maxima (kIdxWCap).
// Returns kNotFused (positive) to ask for the two-launch step instead.
constexpr int kNotFused = 1;

template <int DIDX, int BK, int D, bool F8>
int launch_fused(DecArgs a, int max_kv, int* status, int* seq_ready, cudaStream_t st) {
  using C = StreamCfg<D, BK, F8>;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess)
    return MSA_ERR_CUDA;
  const int grid = sms;
  CUtensorMap tq, tk, tv;
  StreamArgs sa;
  int rc = stream_setup<D, BK, F8>(a, max_kv, status, tq, tk, tv, sa);
  if (rc) return rc;
  if (sa.n_cta > grid) return kNotFused;   // stream_ctas: at most one CTA per item
  const long long tmax = static_cast<long long>(a.batch) * ((max_kv + BK - 1) / BK);
  const long long wmax = (tmax + grid - 1) / grid;
  if (wmax > kIdxWCap) return kNotFused;
  const size_t idx_smem = align_up(static_cast<size_t>(a.batch + 1) * 4, 16) + static_cast<size_t>(a.h_kv) * wmax * 4 +
                          static_cast<size_t>(wmax + 1) * 4;
  if (idx_smem > static_cast<size_t>(C::kSmemBytes)) return kNotFused;
  a.idx_ctas = grid;
  a.idx_wmax = static_cast<int>(wmax < 1 ? 1 : wmax);
  const int smem = C::kSmemBytes + 1024;
  auto kern = a.pool ? decode_fused_kernel<DIDX, BK, 1, D, F8> : decode_fused_kernel<DIDX, BK, 0, D, F8>;
  // The scan's static shared memory comes on top of the attention's ring.
  cudaFuncAttributes fa;
  int smem_max = 0;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (fa.sharedSizeBytes + smem > static_cast<size_t>(smem_max)) return kNotFused;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MSA_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, smem) != cudaSuccess || per_sm < 1)
    return kNotFused;
  void* args[] = {&tq, &tk, &tv, &a, &sa, &seq_ready};
  const cudaError_t e =
      cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), grid, kFusedThreads, args, smem, st);
  if (e == cudaErrorCooperativeLaunchTooLarge) {   // not every CTA can be resident (a shared GPU): two launches
    cudaGetLastError();
    return kNotFused;
  }
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

template <int DIDX, int BK>
int launch_fused_d(const DecArgs& a, int d, int max_kv, int* status, int* seq_ready, cudaStream_t st) {
  if (a.k8) return launch_fused<DIDX, BK, 128, true>(a, max_kv, status, seq_ready, st);
  return d == 64 ? launch_fused<DIDX, BK, 64, false>(a, max_kv, status, seq_ready, st)
                 : launch_fused<DIDX, BK, 128, false>(a, max_kv, status, seq_ready, st);
}

template <int DIDX, int BK>
int launch_index(const DecArgs& a, size_t smem, cudaStream_t st) {
  if (a.kfree > 0) {
    auto kern = a.k_idx8 ? (a.pool ? decode_index_kernel<DIDX, BK, 1, true> : decode_index_kernel<DIDX, BK, 0, true>)
                         : (a.pool ? decode_index_kernel<DIDX, BK, 1, false> : decode_index_kernel<DIDX, BK, 0, false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return MSA_ERR_CUDA;
    kern<<<a.idx_ctas, kIdxThreads, smem, st>>>(a);
  } else {   // topk == 1 with the forced local block needs no scan
    decode_local_only_kernel<BK><<<a.batch * a.h_kv, 32, 0, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace

// Completion counters at the front of the decode workspace.  The caller
// zeroes them (with the status word) before every call.
size_t decode_counter_bytes(const msa_params& p, int batch) {
  // [B] index CTAs per sequence, [B, h_kv, head_tiles] attention CTAs per
  // unit, [B] sequence-ready flags of the fused step.
  const size_t n = static_cast<size_t>(batch) * (2 + p.h_kv * ((p.h_q / p.h_kv + 15) / 16));
  return align_up(n * 4, 256);
}

// Workspace of one call: the counters, then the sparse run's top-k candidates
// and per-share partials, or the dense run's split partials.  dense < 0 gives
// the larger of the two (what msa_workspace_size reports, since it does not
// know which run the caller will make).
size_t decode_workspace_bytes(const msa_params& p, int batch, int max_kv, int dense) {
  const int kfree = p.topk;   // upper bound on topk - force_local
  const size_t cand = static_cast<size_t>(plan_index(p, batch, max_kv).ctas + batch) * p.h_kv * kfree;
  const size_t part_dense = static_cast<size_t>(batch) * p.h_q * plan_dense_splits(p, max_kv).splits * (p.d + 4);
  const long long T = stream_items(p, batch);
  const long long units = T / p.topk;
  const size_t part_stream = static_cast<size_t>(stream_ctas(T) + units) * 16 * (p.d + 4);
  const size_t sparse = align_up(cand * 4, 256) * 2 + align_up(part_stream * 4, 256);
  const size_t dense_b = align_up(cand * 4, 256) * 2 + align_up(part_dense * 4, 256);
  const size_t body = dense > 0 ? dense_b : (dense == 0 ? sparse : (sparse > dense_b ? sparse : dense_b));
  return decode_counter_bytes(p, batch) + body;
}

int run_sparse_attn_decode(const msa_params& p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t /*ws_bytes*/,
                           int* status, cudaStream_t stream, const int32_t* topk_seq, const DecodeMx8* mx8) {
  if (p.h_kv > kDecodeMaxGroups) return MSA_ERR_UNSUPPORTED;
  // TMA row coordinates of the caches are 32-bit.
  if (!dense && static_cast<long long>(batch) * max_kv > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  // The index scan keeps the block prefix of all sequences in shared memory.
  if (!dense && batch > kIdxMaxBatch) return MSA_ERR_UNSUPPORTED;
  DecArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.q_idx = static_cast<const uint16_t*>(q_idx);
  a.k_cache = static_cast<const uint16_t*>(k_cache);
  a.v_cache = static_cast<const uint16_t*>(v_cache);
  a.k_idx = static_cast<const uint16_t*>(k_idx_cache);
  a.cu_kv = cu_kv;
  a.block_ids = block_ids;
  a.o = static_cast<uint16_t*>(o);
  a.batch = batch;
  a.h_q = p.h_q;
  a.h_kv = p.h_kv;
  a.topk = p.topk;
  a.causal = p.causal;
  a.force_local = p.force_local;
  a.kfree = p.topk - (p.force_local ? 1 : 0);
  a.pool = p.pool;
  a.topk_seq = topk_seq;
  a.k8 = mx8 ? static_cast<const uint8_t*>(mx8->k8) : nullptr;
  a.k_sc = mx8 ? static_cast<const uint8_t*>(mx8->k_sc) : nullptr;
  a.v8 = mx8 ? static_cast<const uint8_t*>(mx8->v8) : nullptr;
  a.v_sc = mx8 ? static_cast<const uint8_t*>(mx8->v_sc) : nullptr;
  a.k_idx8 = mx8 ? static_cast<const uint8_t*>(mx8->k_idx8) : nullptr;
  a.k_idx_sc = mx8 ? static_cast<const uint8_t*>(mx8->k_idx_sc) : nullptr;
  const IdxPlan ip = plan_index(p, batch, max_kv);
  a.idx_ctas = ip.ctas;
  a.idx_wmax = ip.wmax;
  const SplitPlan sp = plan_dense_splits(p, max_kv);   // read by the dense run only
  a.splits = sp.splits;
  a.slots_per_split = sp.slots_per_split;
  a.dense = dense;
  const int G = p.h_q / p.h_kv;
  a.head_tiles = (G + 15) / 16;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf(static_cast<float>(p.d));
  a.scale_log2 = scale * kLog2e;
  const size_t cand = static_cast<size_t>(ip.ctas + batch) * p.h_kv * p.topk;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.seq_count = reinterpret_cast<int*>(w);
  a.grp_count = a.seq_count + batch;
  w += decode_counter_bytes(p, batch);
  a.cand_s = reinterpret_cast<float*>(w);
  a.cand_b = reinterpret_cast<int*>(w + align_up(cand * 4, 256));
  a.part = reinterpret_cast<float*>(w + 2 * align_up(cand * 4, 256));

  int rc = MSA_OK;
  if (!dense && a.kfree > 0 && g_decode_fused.load(std::memory_order_relaxed)) {
    // One fused launch when the step fits one co-resident wave.
    int* seq_ready = a.grp_count + static_cast<size_t>(batch) * p.h_kv * a.head_tiles;
    if (p.block_k == 64) {
      rc = p.d_idx == 32 ? launch_fused_d<32, 64>(a, p.d, max_kv, status, seq_ready, stream)
                         : (p.d_idx == 64 ? launch_fused_d<64, 64>(a, p.d, max_kv, status, seq_ready, stream)
                                          : launch_fused_d<128, 64>(a, p.d, max_kv, status, seq_ready, stream));
    } else {
      rc = p.d_idx == 32 ? launch_fused_d<32, 128>(a, p.d, max_kv, status, seq_ready, stream)
                         : (p.d_idx == 64 ? launch_fused_d<64, 128>(a, p.d, max_kv, status, seq_ready, stream)
                                          : launch_fused_d<128, 128>(a, p.d, max_kv, status, seq_ready, stream));
    }
    if (rc != kNotFused) return rc;
    rc = MSA_OK;
  }
  if (!dense) {
    if (p.block_k == 64) {
      rc = p.d_idx == 32 ? launch_index<32, 64>(a, ip.smem, stream)
                         : (p.d_idx == 64 ? launch_index<64, 64>(a, ip.smem, stream) : launch_index<128, 64>(a, ip.smem, stream));
    } else {
      rc = p.d_idx == 32 ? launch_index<32, 128>(a, ip.smem, stream)
                         : (p.d_idx == 64 ? launch_index<64, 128>(a, ip.smem, stream) : launch_index<128, 128>(a, ip.smem, stream));
    }
  }
  if (rc) return rc;
  if (!dense) {
    if (a.k8)   // MXFP8 caches (d = 128, checked on the host)
      return p.block_k == 64 ? launch_attn_stream<128, 64, true>(a, max_kv, status, stream)
                             : launch_attn_stream<128, 128, true>(a, max_kv, status, stream);
    if (p.d == 64)
      return p.block_k == 64 ? launch_attn_stream<64, 64, false>(a, max_kv, status, stream)
                             : launch_attn_stream<64, 128, false>(a, max_kv, status, stream);
    return p.block_k == 64 ? launch_attn_stream<128, 64, false>(a, max_kv, status, stream)
                           : launch_attn_stream<128, 128, false>(a, max_kv, status, stream);
  }
  if (p.d == 64) {
    return p.block_k == 64 ? launch_attn_combine<64, 64>(a, stream) : launch_attn_combine<64, 128>(a, stream);
  }
  return p.block_k == 64 ? launch_attn_combine<128, 64>(a, stream) : launch_attn_combine<128, 128>(a, stream);
}

}  // namespace msa

// ---------------------------------------------------------------------------
// Allocation-free decode step.
//
// For callers that cannot allocate device memory at all: code running where
// cudaMalloc is not allowed (for example while a serving runtime owns and
// pre-partitions every byte of the GPU, or a plugin that is handed only its
// input and output buffers).  The scratch the decode step needs lives in a
// fixed file-scope device array of MSA_NOALLOC_SCRATCH_BYTES, which every GPU
// that loads this library holds until the process exits.
// ---------------------------------------------------------------------------
namespace msa {
namespace {

constexpr int kMaxDevices = 64;
static __device__ __align__(256) uint8_t g_noalloc_scratch[MSA_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of this device's copy of the array.  In host code the
// array's name is only a host-side stand-in, never a device address, so the
// address is looked up once per device with that device current.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" MSA_API int msa_sparse_attn_decode_noalloc(const msa_params* p, const void* q, const void* q_idx,
                                                      const void* k_cache, const void* v_cache,
                                                      const void* k_idx_cache, const int64_t* cu_kv, int batch,
                                                      int max_kv, int dense, int32_t* block_ids, void* o,
                                                      void* stream) {
  void* scratch = nullptr;
  const int rc = msa::noalloc_scratch(&scratch);
  if (rc) return rc;
  // Same validation and kernels as msa_sparse_attn_decode; a problem whose
  // scratch exceeds the array is rejected there with MSA_ERR_WORKSPACE.
  return msa_sparse_attn_decode(p, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, batch, max_kv, dense, block_ids,
                                o, scratch, MSA_NOALLOC_SCRATCH_BYTES, stream);
}
