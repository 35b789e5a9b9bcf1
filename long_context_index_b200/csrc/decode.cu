// decode.cu -- one batched decode step of MiniMax Sparse Attention on sm_100a.
//
// For every sequence b the query sits at position p = L_b - 1 of its own
// contiguous caches.  The step is the prefill math of one row
// (titansim.online summary of "MiniMax Sparse Attention": eq. (6) and the
// local-block rule in section 4.2, eq. (8) in section 4.3), split so that the
// HBM-bound scans use the whole GPU:
//
//   1. decode_index_kernel   grid (chunks of CB blocks, batch).  Streams the
//      index-key cache once for all groups with 16-byte coalesced loads that
//      feed mma.sync directly (a fixed permutation of the d_idx axis, applied
//      to Q_idx and K_idx alike, makes each loaded 16-byte vector a fragment;
//      the dot product does not depend on the order of d_idx).  Max-pools per
//      block and keeps the chunk's top (k - 1) non-local blocks per group.
//   2. decode_topk_merge_kernel  one warp per (sequence, group): top (k - 1)
//      of the chunk lists (score desc, block asc: exact because every global
//      winner is a winner of its chunk), plus the local block, ascending.
//   3. decode_attn_kernel    grid (splits, group x head tile, batch).  Each
//      CTA stages whole K/V blocks with cp.async (16-byte, coalesced), shares
//      them among the 16 heads of its head tile, and runs QK^T and PV on
//      mma.sync with an fp32 online softmax; writes an (m, l, o) partial.
//   4. decode_combine_kernel  per (sequence, head): LSE-weighted sum of the
//      partials, rounded to bf16.
// The dense run skips 1-2 and lets step 3 enumerate every causal block.
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kIdxThreads = 256;    // 8 warps
constexpr int kIdxChunkBlocks = 64; // CB: blocks per index CTA
constexpr int kAttnThreads = 128;   // 4 warps, 32 keys each
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
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
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
  float* cand_s;            // [B, max_chunks, h_kv, kfree]
  int* cand_b;
  float* part;              // [B, h_q, splits, d + 2]  (o[d], m, l)
  int batch, h_q, h_kv, topk, causal, force_local, kfree, max_chunks;
  int splits, slots_per_split, dense, head_tiles;
  float scale_log2;
};

// ---------------------------------------------------------------------------
// 1. index scan: block max-pool + per-chunk top-(k-1) per group
// ---------------------------------------------------------------------------
template <int DIDX, int BK>
__global__ void __launch_bounds__(kIdxThreads) decode_index_kernel(const DecArgs a) {
  constexpr int kHalves = DIDX / 32;   // 16-byte vectors per token row per thread
  __shared__ float smax[8][kIdxChunkBlocks];
  const int b = blockIdx.y;
  const int chunk = blockIdx.x;
  const int64_t off = a.cu_kv[b];
  const int L = static_cast<int>(a.cu_kv[b + 1] - off);
  const int nb = (L + BK - 1) / BK;
  const int blk0 = chunk * kIdxChunkBlocks;
  if (blk0 >= nb) return;
  const int nblk = min(kIdxChunkBlocks, nb - blk0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  // Q_idx fragment (B operand): column n = group g, permuted d_idx order.
  uint4 qv[kHalves];
#pragma unroll
  for (int h = 0; h < kHalves; ++h) {
    qv[h] = make_uint4(0, 0, 0, 0);
    if (g < a.h_kv)
      qv[h] = *reinterpret_cast<const uint4*>(a.q_idx + (static_cast<size_t>(b) * a.h_kv + g) * DIDX + 8 * t + 32 * h);
  }
  const uint16_t* kbase = a.k_idx + static_cast<size_t>(off) * DIDX;

  for (int lb = warp; lb < nblk; lb += kIdxThreads / 32) {
    const int j0 = (blk0 + lb) * BK;
    float m0 = kNegInf, m1 = kNegInf;   // groups 2t, 2t+1
#pragma unroll 2
    for (int mt = 0; mt < BK / 16; ++mt) {
      const int ja = j0 + mt * 16 + g, jb = ja + 8;
      uint4 ra[kHalves], rb[kHalves];
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        ra[h] = ja < L ? ldg_nc_v4(kbase + static_cast<size_t>(ja) * DIDX + 8 * t + 32 * h) : make_uint4(0, 0, 0, 0);
        rb[h] = jb < L ? ldg_nc_v4(kbase + static_cast<size_t>(jb) * DIDX + 8 * t + 32 * h) : make_uint4(0, 0, 0, 0);
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        mma_bf16_16816(c, ra[h].x, rb[h].x, ra[h].y, rb[h].y, qv[h].x, qv[h].y);
        mma_bf16_16816(c, ra[h].z, rb[h].z, ra[h].w, rb[h].w, qv[h].z, qv[h].w);
      }
      if (ja < L) {
        m0 = fmaxf(m0, c[0]);
        m1 = fmaxf(m1, c[1]);
      }
      if (jb < L) {
        m0 = fmaxf(m0, c[2]);
        m1 = fmaxf(m1, c[3]);
      }
    }
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, x));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, x));
    }
    if (g == 0) {
      smax[2 * t][lb] = m0;
      smax[2 * t + 1][lb] = m1;
    }
  }
  __syncthreads();

  // Per group: top-kfree eligible non-local blocks of this chunk.
  const int p = L - 1;
  const int b_loc = p / BK;
  for (int r = warp; r < a.h_kv; r += kIdxThreads / 32) {
    float s0 = kNegInf, s1 = kNegInf;
    int i0 = -1, i1 = -1;
    {
      const int lb0 = lane, lb1 = lane + 32;
      // Decode: every cached key is visible (j <= p), so every block is eligible.
      if (lb0 < nblk && !(a.force_local && blk0 + lb0 == b_loc)) { s0 = smax[r][lb0]; i0 = blk0 + lb0; }
      if (lb1 < nblk && !(a.force_local && blk0 + lb1 == b_loc)) { s1 = smax[r][lb1]; i1 = blk0 + lb1; }
      if (i1 >= 0 && (i0 < 0 || better(s1, i1, s0, i0))) {
        float ts = s0; s0 = s1; s1 = ts;
        int ti = i0; i0 = i1; i1 = ti;
      }
    }
    const size_t base = ((static_cast<size_t>(b) * a.max_chunks + chunk) * a.h_kv + r) * a.kfree;
    for (int k = 0; k < a.kfree; ++k) {
      float bs = i0 >= 0 ? s0 : kNegInf;
      int bi = i0 >= 0 ? i0 : 0x7fffffff;
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, x);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, x);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || better(os, oi, bs, bi))) { bs = os; bi = oi; }
      }
      if (lane == 0) {
        a.cand_s[base + k] = bi == 0x7fffffff ? kNegInf : bs;
        a.cand_b[base + k] = bi == 0x7fffffff ? -1 : bi;
      }
      if (i0 >= 0 && i0 == bi) {   // the owner pops its head
        s0 = s1; i0 = i1;
        s1 = kNegInf; i1 = -1;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 2. merge of the chunk lists + local block -> block_ids (ascending, -1 pad)
// ---------------------------------------------------------------------------
template <int BK>
__global__ void __launch_bounds__(32) decode_topk_merge_kernel(const DecArgs a) {
  const int b = blockIdx.x / a.h_kv;
  const int r = blockIdx.x % a.h_kv;
  const int lane = threadIdx.x;
  const int L = static_cast<int>(a.cu_kv[b + 1] - a.cu_kv[b]);
  const int nb = (L + BK - 1) / BK;
  // Clamp to the chunks the workspace holds (a caller that understated max_kv
  // gets a wrong answer, never an out-of-bounds read).
  const int nch = min((nb + kIdxChunkBlocks - 1) / kIdxChunkBlocks, a.max_chunks);
  const int ncand = nch * a.kfree;
  const int b_loc = (L - 1) / BK;
  __shared__ int chosen[33];
  int nsel = 0;
  // Repeated warp argmax over the candidates with a strictly decreasing bound:
  // each round picks the best candidate that is worse than the previous pick.
  float last_s = __builtin_huge_valf();
  int last_b = -1;
  for (int k = 0; k < a.kfree; ++k) {
    float bs = kNegInf;
    int bi = 0x7fffffff;
    for (int c = lane; c < ncand; c += 32) {
      const int ch = c / a.kfree, slot = c % a.kfree;
      const size_t idx = ((static_cast<size_t>(b) * a.max_chunks + ch) * a.h_kv + r) * a.kfree + slot;
      const int cb = a.cand_b[idx];
      if (cb < 0) continue;
      const float cs = a.cand_s[idx];
      // Only candidates strictly after the previous pick in (score desc, block asc).
      if (k > 0 && !better(last_s, last_b, cs, cb)) continue;
      if (bi == 0x7fffffff || better(cs, cb, bs, bi)) { bs = cs; bi = cb; }
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, x);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, x);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || better(os, oi, bs, bi))) { bs = os; bi = oi; }
    }
    if (bi == 0x7fffffff) break;
    if (lane == 0) chosen[nsel] = bi;
    ++nsel;
    last_s = bs;
    last_b = bi;
  }
  if (lane == 0) {
    if (a.force_local) chosen[nsel++] = b_loc;
    // insertion sort (<= 32 entries)
    for (int i = 1; i < nsel; ++i) {
      const int v = chosen[i];
      int j = i - 1;
      while (j >= 0 && chosen[j] > v) { chosen[j + 1] = chosen[j]; --j; }
      chosen[j + 1] = v;
    }
    int32_t* out = a.block_ids + (static_cast<size_t>(b) * a.h_kv + r) * a.topk;
    for (int i = 0; i < a.topk; ++i) out[i] = i < nsel ? chosen[i] : -1;
  }
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

  // Q rows of this head tile (zero rows beyond the group).
  for (int c = tid; c < 16 * kChunks; c += kAttnThreads) {
    const int row = c / kChunks, ch = c % kChunks;
    cp_async16(swz<D>(smem_u32(sQ), row, ch), a.q + (static_cast<size_t>(b) * a.h_q + h0 + min(row, rows - 1)) * D + ch * 8,
               row < rows);
  }
  cp_async_wait_all();
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

  const int s_begin = split * a.slots_per_split;
  const int n_slots = a.dense ? nb : a.topk;
  const int s_end = min(n_slots, s_begin + a.slots_per_split);
  for (int s = s_begin; s < s_end; ++s) {
    const int blk = a.dense ? s : a.block_ids[(static_cast<size_t>(b) * a.h_kv + r) * a.topk + s];
    if (blk < 0 || blk >= nb) continue;    // padding
    const int j0 = blk * BK;
    __syncthreads();   // previous block fully consumed
    for (int c = tid; c < BK * kChunks; c += kAttnThreads) {
      const int row = c / kChunks, ch = c % kChunks;
      const bool ok = j0 + row < L;
      const size_t src = ((static_cast<size_t>(off) + (ok ? j0 + row : 0)) * a.h_kv + r) * D + ch * 8;
      cp_async16(swz<D>(smem_u32(sK), row, ch), a.k_cache + src, ok);
      cp_async16(swz<D>(smem_u32(sV), row, ch), a.v_cache + src, ok);
    }
    cp_async_wait_all();
    __syncthreads();

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
  }

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
  const size_t stride = D + 2;
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
}

// ---------------------------------------------------------------------------
// 4. combine the split partials of each (sequence, head)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecArgs a) {
  const int bh = blockIdx.x;   // b * h_q + h
  const int col = threadIdx.x;
  const size_t stride = D + 2;
  const float* pp = a.part + static_cast<size_t>(bh) * a.splits * stride;
  float M = kNegInf;
  for (int s = 0; s < a.splits; ++s) M = fmaxf(M, pp[s * stride + D]);
  float num = 0.f, den = 0.f;
  if (M != kNegInf) {
    for (int s = 0; s < a.splits; ++s) {
      const float m = pp[s * stride + D];
      if (m == kNegInf) continue;
      const float w = ex2_approx(m - M);
      num += w * pp[s * stride + col];
      den += w * pp[s * stride + D + 1];
    }
  }
  const float v = den > 0.f ? num / den : 0.f;
  const uint32_t pk = pack_bf16x2(v, 0.f);
  a.o[static_cast<size_t>(bh) * D + col] = static_cast<uint16_t>(pk & 0xffffu);
}

// Split plan shared by the workspace query and the launch.
struct SplitPlan {
  int splits, slots_per_split;
};

SplitPlan plan_splits(const msa_params& p, int max_kv, int dense) {
  SplitPlan s;
  if (dense) {
    const int nb = (max_kv + p.block_k - 1) / p.block_k;
    s.splits = nb < 32 ? nb : 32;
    s.slots_per_split = (nb + s.splits - 1) / s.splits;
  } else {
    s.splits = p.topk;
    s.slots_per_split = 1;
  }
  return s;
}

int max_chunks_for(const msa_params& p, int max_kv) {
  const int nb = (max_kv + p.block_k - 1) / p.block_k;
  return (nb + kIdxChunkBlocks - 1) / kIdxChunkBlocks;
}

template <int D, int BK>
int launch_attn_combine(const DecArgs& a, cudaStream_t st) {
  const int smem = 2 * BK * D * 2 + 16 * D * 2 + 4 * 16 * 2 * 4;
  auto kern = decode_attn_kernel<D, BK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MSA_ERR_CUDA;
  dim3 grid(a.splits, a.h_kv * a.head_tiles, a.batch);
  kern<<<grid, kAttnThreads, smem, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;
  decode_combine_kernel<D><<<a.batch * a.h_q, D, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

template <int DIDX, int BK>
int launch_index(const DecArgs& a, cudaStream_t st) {
  if (a.kfree > 0) {   // topk == 1 with the forced local block needs no scan
    dim3 grid(a.max_chunks, a.batch);
    decode_index_kernel<DIDX, BK><<<grid, kIdxThreads, 0, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;
  }
  decode_topk_merge_kernel<BK><<<a.batch * a.h_kv, 32, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace

size_t decode_workspace_bytes(const msa_params& p, int batch, int max_kv) {
  const int kfree = p.topk;   // upper bound on topk - force_local
  const size_t cand = static_cast<size_t>(batch) * max_chunks_for(p, max_kv) * p.h_kv * kfree;
  const SplitPlan sd = plan_splits(p, max_kv, 1), ss = plan_splits(p, max_kv, 0);
  const int splits = sd.splits > ss.splits ? sd.splits : ss.splits;
  const size_t part = static_cast<size_t>(batch) * p.h_q * splits * (p.d + 2);
  return align_up(cand * 4, 256) * 2 + align_up(part * 4, 256);
}

int run_sparse_attn_decode(const msa_params& p, const void* q, const void* q_idx, const void* k_cache,
                           const void* v_cache, const void* k_idx_cache, const int64_t* cu_kv, int batch,
                           int max_kv, int dense, int32_t* block_ids, void* o, void* ws, size_t /*ws_bytes*/,
                           int* /*status*/, cudaStream_t stream) {
  if (p.h_kv > 8) return MSA_ERR_UNSUPPORTED;
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
  a.max_chunks = max_chunks_for(p, max_kv);
  const SplitPlan sp = plan_splits(p, max_kv, dense);
  a.splits = sp.splits;
  a.slots_per_split = sp.slots_per_split;
  a.dense = dense;
  const int G = p.h_q / p.h_kv;
  a.head_tiles = (G + 15) / 16;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf(static_cast<float>(p.d));
  a.scale_log2 = scale * kLog2e;
  const size_t cand = static_cast<size_t>(batch) * a.max_chunks * p.h_kv * p.topk;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.cand_s = reinterpret_cast<float*>(w);
  a.cand_b = reinterpret_cast<int*>(w + align_up(cand * 4, 256));
  a.part = reinterpret_cast<float*>(w + 2 * align_up(cand * 4, 256));

  int rc = MSA_OK;
  if (!dense) {
    if (p.block_k == 64) {
      rc = p.d_idx == 32 ? launch_index<32, 64>(a, stream)
                         : (p.d_idx == 64 ? launch_index<64, 64>(a, stream) : launch_index<128, 64>(a, stream));
    } else {
      rc = p.d_idx == 32 ? launch_index<32, 128>(a, stream)
                         : (p.d_idx == 64 ? launch_index<64, 128>(a, stream) : launch_index<128, 128>(a, stream));
    }
  }
  if (rc) return rc;
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
