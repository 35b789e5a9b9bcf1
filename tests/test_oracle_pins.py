"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test constructs inputs whose answer is fixed by construction (closed
forms), by an invariant of the method, by exhaustive search on tiny inputs,
or by a library routine (torch's scaled_dot_product_attention in float64 on
the CPU).  A plausible mistake in the oracle -- a dropped causal mask, mean
instead of max pooling, a wrong tie break, a wrong head->group map, a wrong
softmax scale, the local block not counting toward k -- fails at least one.

Passages: titansim.online summary eq. (1), eq. (6) and the local-block rule
(section 4.2), eq. (8) (section 4.3), exp-free ranking (section 4.4.1);
m.163.com post "Step 1 Index Attention" (shared index key, max-pool).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from synth import Workload, bf16_bits_to_f32, f32_to_bf16_bits, make_decode, make_prefill

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def P(**kw):
    base = dict(h_q=4, h_kv=2, d=8, d_idx=4, block_k=4, topk=3, causal=1, force_local=1)
    base.update(kw)
    return oracle.params(**base)


# ----------------------------------------------------------------------------
# Index branch: eq. (6) block max-pool and the top-k rule, by construction.
# ----------------------------------------------------------------------------

def peak_inputs(n, h_kv, d_idx, block_k, peaks):
    """Q_idx[i, r] = e_r; K_idx[j, 0, r] = -1 except one peak per (block, group).

    With this construction S_j^(r) = K_idx[j, r] / sqrt(d_idx), so the pooled
    score of block b is peak/sqrt(d_idx) when the peak is visible, else
    -1/sqrt(d_idx) when any other key of the block is visible.
    peaks[r][b] = (offset_in_block, value).
    """
    q_idx = np.zeros((n, h_kv, d_idx), np.float32)
    for r in range(h_kv):
        q_idx[:, r, r] = 1.0
    k_idx = -np.ones((n, 1, d_idx), np.float32)
    for r in range(h_kv):
        for b, (off, val) in enumerate(peaks[r]):
            k_idx[b * block_k + off, 0, r] = val
    return bf(q_idx), bf(k_idx)


def test_block_max_closed_form():
    n, h_kv, d_idx, B = 32, 2, 4, 4
    nb = n // B
    peaks = [[((b * 3) % B, 10 + b) for b in range(nb)],
             [((b * 5 + 1) % B, 30 - 2 * b) for b in range(nb)]]
    q_idx, k_idx = peak_inputs(n, h_kv, d_idx, B, peaks)
    prm = P(h_kv=h_kv, d_idx=d_idx, block_k=B)
    M = oracle.block_scores(prm, q_idx, k_idx)
    s = 1.0 / math.sqrt(d_idx)
    for i in range(n):
        loc = i // B
        for r in range(h_kv):
            for b in range(nb):
                off, val = peaks[r][b]
                if b < loc:
                    want = val * s
                elif b == loc:
                    want = val * s if b * B + off <= i else -1.0 * s
                else:
                    want = -np.inf
                assert M[i, r, b] == want, (i, r, b)


def test_noncausal_pools_every_block():
    n, h_kv, d_idx, B = 16, 2, 4, 4
    peaks = [[(3, 7)] * 4, [(0, 9)] * 4]
    q_idx, k_idx = peak_inputs(n, h_kv, d_idx, B, peaks)
    M = oracle.block_scores(P(h_kv=h_kv, d_idx=d_idx, block_k=B, causal=0), q_idx, k_idx)
    assert np.all(M[:, 0, :] == 3.5) and np.all(M[:, 1, :] == 4.5)


def test_partial_last_block_pools_valid_keys_only():
    # n_kv = 10 with B_k = 4: block 2 holds keys 8, 9 only.
    n, B = 10, 4
    q_idx = bf(np.tile(np.array([1, 0, 0, 0], np.float32), (n, 1, 1)).reshape(n, 1, 4))
    k_idx = np.full((n, 1, 4), 0.0, np.float32)
    k_idx[:, 0, 0] = [1, 2, 3, 4, 5, 6, 7, 8, 9, 10]
    M = oracle.block_scores(P(h_q=2, h_kv=1, d_idx=4, block_k=B, causal=0), q_idx, bf(k_idx))
    assert M.shape == (n, 1, 3)
    assert np.all(M[:, 0, 2] == 5.0)  # max(9, 10) / sqrt(4)


def test_max_not_mean_pool():
    # Block 0: one strong key among weak ones (high max, low mean).
    # Block 1: uniformly medium keys (higher mean, lower max).
    # Max-pooling (m.163.com "Block Max Pool") must pick block 0.
    n, B = 12, 4
    q_idx = np.zeros((n, 1, 4), np.float32)
    q_idx[:, 0, 0] = 1
    k_idx = np.zeros((n, 1, 4), np.float32)
    k_idx[0:4, 0, 0] = [-3, -3, 12, -3]
    k_idx[4:8, 0, 0] = [3, 3, 3, 3]
    ids = oracle.index_topk(P(h_q=1, h_kv=1, d_idx=4, block_k=B, topk=2), bf(q_idx), bf(k_idx))
    assert list(ids[11, 0]) == [0, 2]
    assert list(ids[10, 0]) == [0, 2]


def test_ties_go_to_lower_block_index():
    n, B = 64, 4
    q_idx = bf(np.ones((n, 1, 4), np.float32))
    k_idx = bf(np.ones((n, 1, 4), np.float32))       # every score equal
    prm = P(h_q=1, h_kv=1, d_idx=4, block_k=B, topk=4)
    ids = oracle.index_topk(prm, q_idx, k_idx)
    for i in range(n):
        loc = i // B
        if loc <= 3:
            want = list(range(loc + 1))
        else:
            want = [0, 1, 2, loc]
        got = [x for x in ids[i, 0] if x >= 0]
        assert got == want, (i, got, want)


def test_local_block_counts_toward_k_and_padding():
    n, B, k = 40, 4, 3
    rng = np.random.default_rng(5)
    q_idx = bf(rng.integers(-3, 4, (n, 2, 4)))
    k_idx = bf(rng.integers(-3, 4, (n, 1, 4)))
    ids = oracle.index_topk(P(block_k=B, topk=k), q_idx, k_idx)
    for i in range(n):
        loc = i // B
        for r in range(2):
            row = ids[i, r]
            valid = row[row >= 0]
            assert len(valid) == min(k, loc + 1)            # budget includes the local block
            assert loc in valid                              # local block always selected
            assert np.all(np.diff(valid) > 0)                # ascending, unique
            assert np.all(row[len(valid):] == -1)            # -1 padding at the end
            assert valid.max() <= loc                        # causal blocks only


def brute_force_select(M_row, local, k, force_local):
    """Exhaustive search: the unique subset S (|S| = min(k, #eligible), holding
    the local block when forced) in which every chosen non-forced block beats
    every unchosen eligible block under (score desc, index asc)."""
    elig = [b for b in range(len(M_row)) if M_row[b] != -np.inf]
    size = min(k, len(elig))
    found = []
    for S in itertools.combinations(elig, size):
        if force_local and local not in S:
            continue
        free = [b for b in S if not (force_local and b == local)]
        out = [b for b in elig if b not in S]
        ok = all((M_row[a] > M_row[c]) or (M_row[a] == M_row[c] and a < c) for a in free for c in out)
        if ok:
            found.append(list(S))
    assert len(found) == 1, found
    return found[0]


@pytest.mark.parametrize("force_local", [1, 0])
@pytest.mark.parametrize("k", [1, 2, 3, 5])
def test_topk_matches_exhaustive_search(k, force_local):
    n, B, h_kv = 48, 8, 2
    rng = np.random.default_rng(100 + k)
    # Values in {-1, 0, 1} and d_idx = 2: many exact ties.
    q_idx = bf(rng.integers(-1, 2, (n, h_kv, 2)))
    k_idx = bf(rng.integers(-1, 2, (n, 1, 2)))
    prm = P(h_kv=h_kv, d_idx=2, block_k=B, topk=k, force_local=force_local)
    M = oracle.block_scores(prm, q_idx, k_idx)
    ids = oracle.index_topk(prm, q_idx, k_idx)
    for i in range(n):
        for r in range(h_kv):
            want = brute_force_select(M[i, r], i // B, k, force_local)
            got = [x for x in ids[i, r] if x >= 0]
            assert got == want, (i, r, got, want)


def random_index_case(seed=7, n=256, h_kv=2, d_idx=8, B=16):
    rng = np.random.default_rng(seed)
    return bf(rng.integers(-3, 4, (n, h_kv, d_idx))), bf(rng.integers(-3, 4, (n, 1, d_idx)))


def test_positive_scaling_of_index_query_keeps_ids():
    q_idx, k_idx = random_index_case()
    prm = P(h_kv=2, d_idx=8, block_k=16, topk=4)
    a = oracle.index_topk(prm, q_idx, k_idx)
    b = oracle.index_topk(prm, bf(bf16_bits_to_f32(q_idx) * 2), k_idx)
    assert np.array_equal(a, b)


def test_permuting_keys_inside_a_block_keeps_ids():
    q_idx, k_idx = random_index_case()
    prm = P(h_kv=2, d_idx=8, block_k=16, topk=4)
    a = oracle.index_topk(prm, q_idx, k_idx)
    k2 = k_idx.copy()
    rng = np.random.default_rng(3)
    for b in range(256 // 16):
        perm = rng.permutation(16)
        k2[b * 16:(b + 1) * 16] = k_idx[b * 16 + perm]
    b_ = oracle.index_topk(prm, q_idx, k2)
    # Rows whose own block is fully visible after the permutation: the last
    # key of their block is <= p, i.e. rows at the end of each block.
    rows = [i for i in range(256) if i % 16 == 15]
    assert np.array_equal(a[rows], b_[rows])
    # Earlier rows: only their local block can be affected, and it is forced.
    assert np.array_equal(a, b_)


def test_future_keys_do_not_change_causal_ids():
    q_idx, k_idx = random_index_case()
    prm = P(h_kv=2, d_idx=8, block_k=16, topk=4)
    a = oracle.index_topk(prm, q_idx, k_idx)
    for p in (40, 100, 170):
        k2 = k_idx.copy()
        k2[p + 1:] = bf(np.full((256 - p - 1, 1, 8), 3.0))   # strong keys in the future
        b = oracle.index_topk(prm, q_idx, k2, rows=[p])
        assert np.array_equal(a[p], b[0])
    # Without the causal mask the same change must matter (sanity of the test).
    prm_nc = P(h_kv=2, d_idx=8, block_k=16, topk=4, causal=0)
    k2 = k_idx.copy()
    k2[200] = bf(np.full((1, 8), 3.0))
    q1 = q_idx.copy()
    q1[40] = bf(np.full((2, 8), 3.0))
    a1 = oracle.index_topk(prm_nc, q1, k_idx, rows=[40])
    b1 = oracle.index_topk(prm_nc, q1, k2, rows=[40])
    assert not np.array_equal(a1, b1)


def test_argmax_block_is_always_selected():
    q_idx, k_idx = random_index_case(seed=11, n=512, d_idx=8, B=32)
    prm = P(h_kv=2, d_idx=8, block_k=32, topk=3)
    ids = oracle.index_topk(prm, q_idx, k_idx)
    q = bf16_bits_to_f32(q_idx).astype(np.float64)
    k = bf16_bits_to_f32(k_idx)[:, 0, :].astype(np.float64)
    for i in range(0, 512, 7):
        for r in range(2):
            s = k[: i + 1] @ q[i, r]            # plain dot products of visible keys
            j = int(np.argmax(s))               # first index of the maximum
            assert j // 32 in ids[i, r], (i, r)


def test_needles_are_recalled():
    w = Workload("needle_test", "prefill", h_q=8, h_kv=2, d=16, d_idx=32, block_k=64, topk=8,
                 seed=9, n_q=4096, n_kv=4096, needles=8)
    t = make_prefill(w)
    prm = oracle.params(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    rows = sorted({qi for (_, qi, _) in t["needles"]})
    ids = oracle.index_topk(prm, t["q_idx"], t["k_idx"], rows=rows)
    pos = {q: x for x, q in enumerate(rows)}
    assert len(t["needles"]) == 16
    for r, qi, pk in t["needles"]:
        assert pk // w.block_k in ids[pos[qi], r], (r, qi, pk)


# ----------------------------------------------------------------------------
# Main branch: eq. (1) and eq. (8) against a library attention routine.
# ----------------------------------------------------------------------------

def attn_case(seed=0, n_q=40, n_kv=40, h_q=4, h_kv=2, d=8):
    rng = np.random.default_rng(seed)
    q = bf(rng.standard_normal((n_q, h_q, d)))
    k = bf(rng.standard_normal((n_kv, h_kv, d)))
    v = bf(rng.standard_normal((n_kv, h_kv, d)))
    return q, k, v


def sdpa_masked(q, k, v, allow, h_q, h_kv):
    """torch SDPA (float64, CPU) with GQA by contiguous head groups."""
    G = h_q // h_kv
    Q = torch.from_numpy(bf16_bits_to_f32(q).astype(np.float64)).permute(1, 0, 2)[None]
    K = torch.from_numpy(bf16_bits_to_f32(k).astype(np.float64)).permute(1, 0, 2)
    V = torch.from_numpy(bf16_bits_to_f32(v).astype(np.float64)).permute(1, 0, 2)
    K = K.repeat_interleave(G, dim=0)[None]
    V = V.repeat_interleave(G, dim=0)[None]
    mask = torch.from_numpy(allow)           # [h_q, n_q, n_kv] bool
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask[None])
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("q_pos0", [0, 16])
def test_dense_matches_library_attention(q_pos0):
    n_kv = 40
    q, k, v = attn_case(n_q=n_kv - q_pos0, n_kv=n_kv)
    prm = P()
    o = oracle.dense_attn(prm, q, k, v, q_pos0=q_pos0)
    allow = np.zeros((4, n_kv - q_pos0, n_kv), bool)
    for i in range(n_kv - q_pos0):
        allow[:, i, : q_pos0 + i + 1] = True
    ref = sdpa_masked(q, k, v, allow, 4, 2)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_sparse_matches_library_attention_with_block_mask():
    n, B, k_ = 48, 4, 3
    q, k, v = attn_case(seed=1, n_q=n, n_kv=n)
    rng = np.random.default_rng(2)
    ids = np.full((n, 2, k_), -1, np.int32)
    for i in range(n):
        loc = i // B
        for r in range(2):
            others = [b for b in range(loc) if rng.random() < 0.5][: k_ - 1]
            sel = sorted(others + [loc])
            ids[i, r, : len(sel)] = sel
    prm = P(block_k=B, topk=k_)
    o = oracle.sparse_attn(prm, q, k, v, ids)
    allow = np.zeros((4, n, n), bool)
    for i in range(n):
        for h in range(4):
            r = h // 2
            for b in ids[i, r]:
                if b < 0:
                    continue
                for j in range(b * B, (b + 1) * B):
                    if j <= i:
                        allow[h, i, j] = True
    ref = sdpa_masked(q, k, v, allow, 4, 2)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_all_blocks_selected_equals_dense():
    # k >= number of causal blocks: MSA reduces to dense causal GQA attention.
    n = 64
    q, k, v = attn_case(seed=3, n_q=n, n_kv=n, h_q=8, h_kv=2, d=16)
    rng = np.random.default_rng(4)
    q_idx = bf(rng.integers(-3, 4, (n, 2, 8)))
    k_idx = bf(rng.integers(-3, 4, (n, 1, 8)))
    prm = oracle.params(8, 2, 16, 8, 8, 8)
    ids = oracle.index_topk(prm, q_idx, k_idx)
    o_sparse = oracle.sparse_attn(prm, q, k, v, ids)
    o_dense = oracle.dense_attn(prm, q, k, v)
    assert np.max(np.abs(o_sparse - o_dense)) < 1e-13


def test_softmax_weights_sum_to_one():
    n = 48
    q, k, _ = attn_case(seed=5, n_q=n, n_kv=n)
    ones = bf(np.ones((n, 2, 8)))
    rng = np.random.default_rng(6)
    q_idx = bf(rng.integers(-3, 4, (n, 2, 4)))
    k_idx = bf(rng.integers(-3, 4, (n, 1, 4)))
    prm = P(block_k=4, topk=3)
    ids = oracle.index_topk(prm, q_idx, k_idx)
    assert np.max(np.abs(oracle.sparse_attn(prm, q, k, ones, ids) - 1.0)) < 1e-12
    assert np.max(np.abs(oracle.dense_attn(prm, q, k, ones) - 1.0)) < 1e-12


def test_zero_query_gives_uniform_average_and_log_count():
    # q = 0: all logits are 0, so O is the plain mean of the visible values and
    # lse = log(number of visible keys).
    n = 24
    _, k, v = attn_case(seed=7, n_q=n, n_kv=n)
    q = bf(np.zeros((n, 4, 8)))
    prm = P(block_k=4, topk=2)
    ids = np.full((n, 2, 2), -1, np.int32)
    for i in range(n):
        ids[i, :, 0] = 0
        ids[i, :, 1] = i // 4 if i // 4 != 0 else -1
    o, lse = oracle.sparse_attn(prm, q, k, v, ids, want_lse=True)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    for i in range(n):
        keys = sorted(set(list(range(min(4, i + 1))) + list(range((i // 4) * 4, i + 1))))
        for h in range(4):
            want = vf[keys, h // 2].mean(axis=0)
            assert np.max(np.abs(o[i, h] - want)) < 1e-12
            assert abs(lse[i, h] - math.log(len(keys))) < 1e-12


def test_custom_scale_is_used():
    n = 20
    q, k, v = attn_case(seed=8, n_q=n, n_kv=n)
    # scale = 2/sqrt(d) on q must equal the default 1/sqrt(d) on 2q (exact in bf16).
    o1 = oracle.dense_attn(P(scale=2.0 / math.sqrt(8)), q, k, v)
    o2 = oracle.dense_attn(P(), bf(bf16_bits_to_f32(q) * 2.0), k, v)
    assert np.max(np.abs(o1 - o2)) < 1e-12


# ----------------------------------------------------------------------------
# Entry-point consistency: chunked prefill and decode rows = full prefill rows.
# ----------------------------------------------------------------------------

def small_prefill():
    w = Workload("small", "prefill", h_q=8, h_kv=2, d=16, d_idx=8, block_k=16, topk=4, seed=21,
                 n_q=300, n_kv=300, needles=2)
    return w, make_prefill(w)


def test_chunked_prefill_rows_equal_full_prefill_rows():
    w, t = small_prefill()
    prm = oracle.params(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids_full = oracle.index_topk(prm, t["q_idx"], t["k_idx"])
    o_full = oracle.sparse_attn(prm, t["q"], t["k"], t["v"], ids_full)
    n_q = 77
    q0 = 300 - n_q
    ids_c = oracle.index_topk(prm, t["q_idx"][q0:], t["k_idx"], q_pos0=q0)
    o_c = oracle.sparse_attn(prm, t["q"][q0:], t["k"], t["v"], ids_c, q_pos0=q0)
    assert np.array_equal(ids_c, ids_full[q0:])
    assert np.max(np.abs(o_c - o_full[q0:])) < 1e-14


def test_decode_equals_last_prefill_row():
    w = Workload("dec", "decode", h_q=8, h_kv=2, d=16, d_idx=8, block_k=16, topk=4, seed=22, batch=3,
                 kv_min=100, kv_max=260, needles=2)
    t = make_decode(w)
    prm = oracle.params(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids, o = oracle.decode(prm, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"], t["cu_kv"])
    for b in range(3):
        lo, hi = int(t["cu_kv"][b]), int(t["cu_kv"][b + 1])
        L = hi - lo
        # Build a prefill whose last row is the decode token.
        qi = np.zeros((L, 2, 8), np.uint16)
        qi[-1] = t["q_idx"][b]
        qq = np.zeros((L, 8, 16), np.uint16)
        qq[-1] = t["q"][b]
        ids_p = oracle.index_topk(prm, qi, t["k_idx_cache"][lo:hi], rows=[L - 1])
        o_p = oracle.sparse_attn(prm, qq, t["k_cache"][lo:hi], t["v_cache"][lo:hi], ids_p, rows=[L - 1])
        assert np.array_equal(ids[b], ids_p[0])
        assert np.max(np.abs(o[b] - o_p[0])) < 1e-14
    # Decode needles are recalled.
    for b, r, pk in t["needles"]:
        assert pk // w.block_k in ids[b, r]
    # Dense decode equals dense attention of the last row.
    _, od = oracle.decode(prm, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"],
                          t["cu_kv"], dense=True)
    lo, hi = int(t["cu_kv"][0]), int(t["cu_kv"][1])
    qq = np.zeros((hi - lo, 8, 16), np.uint16)
    qq[-1] = t["q"][0]
    ref = oracle.dense_attn(prm, qq, t["k_cache"][lo:hi], t["v_cache"][lo:hi], rows=[hi - lo - 1])
    assert np.max(np.abs(od[0] - ref[0])) < 1e-14


def test_bad_arguments_are_rejected():
    q_idx, k_idx = random_index_case(n=32)
    with pytest.raises(ValueError):
        oracle.index_topk(P(h_kv=2, d_idx=8, block_k=16, topk=0), q_idx, k_idx)
    with pytest.raises(ValueError):
        oracle.index_topk(P(h_q=3, h_kv=2, d_idx=8, block_k=16), q_idx, k_idx)
