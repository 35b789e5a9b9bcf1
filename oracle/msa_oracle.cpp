// msa_oracle.cpp -- plain fp64 CPU reference of the MiniMax Sparse Attention
// (MSA) hot path.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
// CPU-baseline leg load this library.  The CUDA path never calls it, and the
// two share no code: no kernels, headers, helpers, tables or pre/post-processing.
//
// Sources (titles and sections of the pages the method is described on):
//   [T]  titansim.online, "MiniMax Sparse Attention" summary:
//        eq. (1)  dense causal attention (section 2.2);
//        eq. (6)  index score and causal block max-pool (section 4.2);
//        "the local block is always included" (section 4.2, after eq. 6);
//        eq. (8)  main-branch softmax attention over the gathered blocks (4.3);
//        section 4.4.1: softmax is monotone, so selection ranks raw scores.
//   [M]  m.163.com post, "Step 1 Index Attention": Q_idx in R^{n x h x d},
//        K_idx in R^{n x 1 x d}: one index query per GQA group, one shared key;
//        and its comparison of the block max-pool with MoBA's mean pooling.
//
// Every input is a bf16 bit pattern widened exactly to double; all arithmetic
// is double.  Rows are independent, so the OpenMP split over (row, group)
// does not change any result.
//
// Readings where the pages are silent (each also listed in the design notes):
//   * Local block = floor(p / B_k) for absolute query position p; it is always
//     selected when force_local != 0 and counts toward k.
//   * Ranking is by M descending, ties to the lower block index; ids are
//     emitted ascending, padded with -1 when fewer than k blocks are eligible.
//   * A block is eligible when it holds at least one visible key (j <= p when
//     causal).  A partial last block is pooled over its valid keys only.
//   * The main branch masks keys j > p inside the selected blocks (causal).
//   * Head h belongs to group r = floor(h / (h_q / h_kv)).
//   * Main-branch scale defaults to 1/sqrt(d) (eq. 8); index scale 1/sqrt(d_idx).
//
// Parity status of each function is stated in its comment.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

typedef struct {
  int h_q, h_kv, d, d_idx, block_k, topk, causal, force_local;
  double scale;   // main-branch softmax scale; <= 0 means 1/sqrt(d)
  int threads;    // OpenMP threads; <= 0 means the runtime default
  int pool;       // block pooling of the token scores: 0 = max (eq. 6), 1 = mean (MoBA-style ablation)
} msa_oracle_params;

}  // extern "C"

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

inline double bf16(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

inline int n_blocks(int n_kv, int block_k) { return (n_kv + block_k - 1) / block_k; }

// Is key j visible from absolute query position p?
inline bool visible(const msa_oracle_params& P, long long p, long long j, int n_kv) {
  if (j < 0 || j >= n_kv) return false;
  return P.causal ? (j <= p) : true;
}

void set_threads(const msa_oracle_params& P) {
#ifdef _OPENMP
  if (P.threads > 0 && !omp_in_parallel()) omp_set_num_threads(P.threads);
#else
  (void)P;
#endif
}

int check(const msa_oracle_params* P, int n_q, int n_kv, long long q_pos0) {
  if (!P || P->h_q <= 0 || P->h_kv <= 0 || P->h_q % P->h_kv != 0) return -1;
  if (P->d <= 0 || P->d_idx <= 0 || P->block_k <= 0 || P->topk <= 0) return -1;
  if (n_q < 0 || n_kv <= 0 || q_pos0 < 0 || q_pos0 + n_q > n_kv) return -1;
  return 0;
}

// Eq. (6), [T] section 4.2: block scores of one (query row, group).
//   S_j = <Q_idx_i^(r), K_idx_j> / sqrt(d_idx)        (token score)
//   M_b = max over j in B_b with j visible of S_j     (causal block max-pool)
// With P.pool = 1, M_b is instead the mean of S_j over the visible keys of
// the block: the mean pooling of MoBA that [M] compares the max-pool with
// (the mean of <q, k_j> is <q, mean of k_j>, MoBA's block score).  A mean
// over a partial block is a ratio that the kernel ranks in fp32, so the
// ranking key here is the same fp32 rounding of (sum of raw dot products) /
// (visible keys), times 1/sqrt(d_idx); with integer-valued index inputs the
// sum is exact and the key is exactly the kernel's.
// Blocks with no visible key get -inf (they are not eligible).
void block_scores_row(const msa_oracle_params& P, const uint16_t* q_idx, const uint16_t* k_idx,
                      int n_kv, int i, long long p, int r, double* M) {
  const int nb = n_blocks(n_kv, P.block_k);
  const double inv = 1.0 / std::sqrt(static_cast<double>(P.d_idx));
  const uint16_t* qv = q_idx + (static_cast<size_t>(i) * P.h_kv + r) * P.d_idx;
  for (int b = 0; b < nb; ++b) {
    double best = kNegInf;
    double raw_sum = 0.0;
    long long count = 0;
    for (long long j = static_cast<long long>(b) * P.block_k;
         j < std::min<long long>(static_cast<long long>(b + 1) * P.block_k, n_kv); ++j) {
      if (!visible(P, p, j, n_kv)) continue;
      const uint16_t* kv = k_idx + static_cast<size_t>(j) * P.d_idx;  // K_idx[j, 0, :]
      double s = 0.0;
      for (int t = 0; t < P.d_idx; ++t) s += bf16(qv[t]) * bf16(kv[t]);
      raw_sum += s;
      ++count;
      s *= inv;
      if (s > best) best = s;
    }
    if (P.pool == 1)
      M[b] = count == 0 ? kNegInf
                        : static_cast<double>(static_cast<float>(raw_sum / static_cast<double>(count))) * inv;
    else
      M[b] = best;
  }
}

// Top-k block selection, [T] section 4.2 (after eq. 6): the top-k blocks by
// M form I_i^(r); the local block is always in the set.  Ranking uses the raw
// pooled scores (no exponentiation: [T] section 4.4.1).  Writes `topk` ids,
// ascending, padded with -1.
void select_row(const msa_oracle_params& P, const double* M, int nb, long long p, int32_t* out) {
  std::vector<int> sel;
  const int local = static_cast<int>(p / P.block_k);
  if (P.force_local && local < nb) sel.push_back(local);
  std::vector<int> cand;
  for (int b = 0; b < nb; ++b) {
    if (M[b] == kNegInf) continue;           // no visible key: not eligible
    if (P.force_local && b == local) continue;
    cand.push_back(b);
  }
  std::sort(cand.begin(), cand.end(), [&](int a, int b) {
    if (M[a] != M[b]) return M[a] > M[b];    // higher pooled score first
    return a < b;                            // ties: lower block index first
  });
  for (size_t c = 0; c < cand.size() && static_cast<int>(sel.size()) < P.topk; ++c)
    sel.push_back(cand[c]);
  std::sort(sel.begin(), sel.end());
  for (int t = 0; t < P.topk; ++t) out[t] = t < static_cast<int>(sel.size()) ? sel[t] : -1;
}

// Softmax attention of one query head over an explicit key list, eq. (1)/(8):
//   z_j = scale * <q, k_j>,  a_j = exp(z_j - max z) / sum exp(z - max z),
//   o = sum_j a_j v_j,  lse = max z + log(sum exp(z - max z)).
void attend(const msa_oracle_params& P, const uint16_t* qh, const uint16_t* k, const uint16_t* v,
            int r, const std::vector<long long>& keys, double* o, double* lse) {
  const double scale = P.scale > 0 ? P.scale : 1.0 / std::sqrt(static_cast<double>(P.d));
  for (int t = 0; t < P.d; ++t) o[t] = 0.0;
  if (keys.empty()) {
    if (lse) *lse = kNegInf;
    return;
  }
  std::vector<double> z(keys.size());
  double zmax = kNegInf;
  for (size_t c = 0; c < keys.size(); ++c) {
    const uint16_t* kj = k + (static_cast<size_t>(keys[c]) * P.h_kv + r) * P.d;
    double s = 0.0;
    for (int t = 0; t < P.d; ++t) s += bf16(qh[t]) * bf16(kj[t]);
    z[c] = s * scale;
    zmax = std::max(zmax, z[c]);
  }
  double den = 0.0;
  for (size_t c = 0; c < keys.size(); ++c) {
    z[c] = std::exp(z[c] - zmax);
    den += z[c];
  }
  for (size_t c = 0; c < keys.size(); ++c) {
    const double a = z[c] / den;
    const uint16_t* vj = v + (static_cast<size_t>(keys[c]) * P.h_kv + r) * P.d;
    for (int t = 0; t < P.d; ++t) o[t] += a * bf16(vj[t]);
  }
  if (lse) *lse = zmax + std::log(den);
}

inline int row_of(const int* rows, int idx) { return rows ? rows[idx] : idx; }

}  // namespace

extern "C" {

// Block scores M (eq. 6) for the listed query rows: out[n_rows, h_kv, nb]
// with nb = ceil(n_kv / B_k).  Pinned by the CPU tests (brute force, needle,
// invariants).
int msa_oracle_block_scores(const msa_oracle_params* P, const uint16_t* q_idx, const uint16_t* k_idx,
                            int n_q, int n_kv, long long q_pos0, const int* rows, int n_rows,
                            double* out) {
  if (check(P, n_q, n_kv, q_pos0)) return -1;
  set_threads(*P);
  const int nb = n_blocks(n_kv, P->block_k);
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int x = 0; x < n_rows; ++x)
    for (int r = 0; r < P->h_kv; ++r) {
      const int i = row_of(rows, x);
      block_scores_row(*P, q_idx, k_idx, n_kv, i, q_pos0 + i, r,
                       out + (static_cast<size_t>(x) * P->h_kv + r) * nb);
    }
  return 0;
}

// Index branch (eq. 6 + top-k with the local block): ids[n_rows, h_kv, topk].
int msa_oracle_index_topk(const msa_oracle_params* P, const uint16_t* q_idx, const uint16_t* k_idx,
                          int n_q, int n_kv, long long q_pos0, const int* rows, int n_rows,
                          int32_t* ids) {
  if (check(P, n_q, n_kv, q_pos0)) return -1;
  set_threads(*P);
  const int nb = n_blocks(n_kv, P->block_k);
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int x = 0; x < n_rows; ++x)
    for (int r = 0; r < P->h_kv; ++r) {
      const int i = row_of(rows, x);
      const long long p = q_pos0 + i;
      std::vector<double> M(nb);
      block_scores_row(*P, q_idx, k_idx, n_kv, i, p, r, M.data());
      select_row(*P, M.data(), nb, p, ids + (static_cast<size_t>(x) * P->h_kv + r) * P->topk);
    }
  return 0;
}

// Main branch, eq. (8): for each listed row and every head h of group r,
// softmax attention over the visible keys of the blocks in ids[x, r, :]
// (entries < 0 are padding).  o[n_rows, h_q, d]; lse[n_rows, h_q] optional.
int msa_oracle_sparse_attn(const msa_oracle_params* P, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const int32_t* ids, int n_q, int n_kv, long long q_pos0,
                           const int* rows, int n_rows, double* o, double* lse) {
  if (check(P, n_q, n_kv, q_pos0)) return -1;
  set_threads(*P);
  const int G = P->h_q / P->h_kv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int x = 0; x < n_rows; ++x)
    for (int r = 0; r < P->h_kv; ++r) {
      const int i = row_of(rows, x);
      const long long p = q_pos0 + i;
      const int32_t* sel = ids + (static_cast<size_t>(x) * P->h_kv + r) * P->topk;
      std::vector<int32_t> blocks;
      for (int t = 0; t < P->topk; ++t)
        if (sel[t] >= 0) blocks.push_back(sel[t]);
      std::sort(blocks.begin(), blocks.end());
      blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
      std::vector<long long> keys;   // K^(r)[I_i^(r)], causally visible keys only
      for (int32_t b : blocks)
        for (long long j = static_cast<long long>(b) * P->block_k;
             j < static_cast<long long>(b + 1) * P->block_k; ++j)
          if (visible(*P, p, j, n_kv)) keys.push_back(j);
      for (int hh = 0; hh < G; ++hh) {
        const int h = r * G + hh;
        attend(*P, q + (static_cast<size_t>(i) * P->h_q + h) * P->d, k, v, r, keys,
               o + (static_cast<size_t>(x) * P->h_q + h) * P->d,
               lse ? lse + static_cast<size_t>(x) * P->h_q + h : nullptr);
      }
    }
  return 0;
}

// Dense GQA attention, eq. (1): every head attends to all visible keys (no
// block logic at all).  Used as the dense special case the sparse branch must
// reduce to, and pinned against a library attention routine in the tests.
int msa_oracle_dense_attn(const msa_oracle_params* P, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, int n_q, int n_kv, long long q_pos0, const int* rows,
                          int n_rows, double* o, double* lse) {
  if (check(P, n_q, n_kv, q_pos0)) return -1;
  set_threads(*P);
  const int G = P->h_q / P->h_kv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int x = 0; x < n_rows; ++x)
    for (int h = 0; h < P->h_q; ++h) {
      const int i = row_of(rows, x);
      const long long p = q_pos0 + i;
      std::vector<long long> keys;
      for (long long j = 0; j < n_kv; ++j)
        if (visible(*P, p, j, n_kv)) keys.push_back(j);
      attend(*P, q + (static_cast<size_t>(i) * P->h_q + h) * P->d, k, v, h / G, keys,
             o + (static_cast<size_t>(x) * P->h_q + h) * P->d,
             lse ? lse + static_cast<size_t>(x) * P->h_q + h : nullptr);
    }
  return 0;
}

// Decode step: for each listed sequence b (query at p = L_b - 1 over its own
// contiguous caches [cu_kv[b], cu_kv[b+1])), the index branch then the main
// branch, exactly as for a one-row chunked prefill with q_pos0 = L_b - 1.
// ids[n_seq, h_kv, topk], o[n_seq, h_q, d].  dense != 0 uses every causal
// block instead of the index branch (ids are then left untouched).
int msa_oracle_decode(const msa_oracle_params* P, const uint16_t* q, const uint16_t* q_idx,
                      const uint16_t* k_cache, const uint16_t* v_cache, const uint16_t* k_idx_cache,
                      const long long* cu_kv, int batch, const int* seqs, int n_seq, int dense,
                      int32_t* ids, double* o) {
  if (!P || batch <= 0) return -1;
  set_threads(*P);
  std::vector<int> status(n_seq > 0 ? n_seq : 1, 0);
  // Sequences are independent; the per-sequence calls below run serially
  // inside this parallel loop (nested parallel regions are off).
#pragma omp parallel for schedule(dynamic, 1)
  for (int x = 0; x < n_seq; ++x) {
    const int b = seqs ? seqs[x] : x;
    if (b < 0 || b >= batch || cu_kv[b + 1] - cu_kv[b] <= 0) {
      status[x] = -1;
      continue;
    }
    const long long off = cu_kv[b];
    const int L = static_cast<int>(cu_kv[b + 1] - off);
    const uint16_t* qb = q + static_cast<size_t>(b) * P->h_q * P->d;
    const uint16_t* kb = k_cache + static_cast<size_t>(off) * P->h_kv * P->d;
    const uint16_t* vb = v_cache + static_cast<size_t>(off) * P->h_kv * P->d;
    double* ob = o + static_cast<size_t>(x) * P->h_q * P->d;
    int rc;
    if (dense) {
      rc = msa_oracle_dense_attn(P, qb, kb, vb, 1, L, L - 1, nullptr, 1, ob, nullptr);
    } else {
      int32_t* idb = ids + static_cast<size_t>(x) * P->h_kv * P->topk;
      rc = msa_oracle_index_topk(P, q_idx + static_cast<size_t>(b) * P->h_kv * P->d_idx,
                                 k_idx_cache + static_cast<size_t>(off) * P->d_idx, 1, L, L - 1,
                                 nullptr, 1, idb);
      if (!rc) rc = msa_oracle_sparse_attn(P, qb, kb, vb, idb, 1, L, L - 1, nullptr, 1, ob, nullptr);
    }
    status[x] = rc;
  }
  for (int x = 0; x < n_seq; ++x)
    if (status[x]) return status[x];
  return 0;
}

}  // extern "C"
