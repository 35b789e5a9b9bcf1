"""GPU parity of the index branch (msa_index_topk) against the fp64 oracle.

Block ids must match bit for bit: index inputs are integers, so every score
is exact on both sides, and ties break to the lower block index on both.
"""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import WORKLOADS, Workload, make_prefill
from tests.gpu_util import dev, params_pair

pytestmark = pytest.mark.gpu


def run_case(w: Workload, n_q=None, n_kv=None, rows=None, causal=1, force_local=1, topk=None, pool=0):
    t = make_prefill(w, n_q=n_q, n_kv=n_kv)
    k = w.topk if topk is None else topk
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, k, causal, force_local, pool=pool)
    ids = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]), q_pos0=t["q_pos0"])
    torch.cuda.synchronize()
    got = ids.cpu().numpy()
    nq = t["q_idx"].shape[0]
    if rows is None:
        rows = np.arange(nq)
    rows = np.asarray(sorted(set(int(r) for r in rows if 0 <= r < nq)), dtype=np.int32)
    ref = oracle.index_topk(po, t["q_idx"], t["k_idx"], q_pos0=t["q_pos0"], rows=rows)
    mism = np.argwhere(got[rows] != ref)
    assert mism.size == 0, "ids differ at %d places, first (row,group,slot)=%s got %s ref %s" % (
        len(mism), [(int(rows[m[0]]), int(m[1]), int(m[2])) for m in mism[:3]],
        [got[rows[m[0]], m[1]].tolist() for m in mism[:2]], [ref[m[0], m[1]].tolist() for m in mism[:2]])
    return t, got


def small(**kw):
    base = dict(name="case", kind="prefill", h_q=8, h_kv=2, d=64, d_idx=32, block_k=64, topk=4, seed=100,
                n_q=1024, n_kv=1024, needles=0)
    base.update(kw)
    return Workload(**base)


def test_tiny_prefill_1k_all_rows():
    run_case(WORKLOADS["tiny_prefill_1k"])


@pytest.mark.parametrize("kw", [
    dict(n_q=1000, n_kv=1000),                                  # ragged last query and key tiles
    dict(n_q=77, n_kv=1000),                                    # chunked: q_pos0 = 923, not block aligned
    dict(n_q=300, n_kv=300, d_idx=64, block_k=128, topk=3),
    dict(n_q=700, n_kv=900, d_idx=128, block_k=128, topk=5),
    dict(n_q=640, n_kv=640, topk=16),
    dict(n_q=600, n_kv=600, topk=32, block_k=64),
    dict(n_q=520, n_kv=520, h_kv=3, h_q=12),                    # odd group count
    dict(n_q=50, n_kv=50),                                      # shorter than one tile
    dict(n_q=1, n_kv=1),                                        # one token
])
def test_shapes(kw):
    run_case(small(seed=kw.get("n_q", 1) + 7, **kw))


@pytest.mark.parametrize("force_local", [0, 1])
def test_force_local_setting(force_local):
    run_case(small(n_q=513, n_kv=513, seed=5), force_local=force_local)


def test_topk_one_is_the_local_block():
    _, got = run_case(small(n_q=400, n_kv=400, seed=6), topk=1)
    assert np.array_equal(got[:, :, 0], np.repeat((np.arange(400) // 64)[:, None], 2, axis=1))


def test_noncausal():
    run_case(small(n_q=256, n_kv=512, seed=8), causal=0)


def test_zero_rows_is_a_noop():
    p, _ = params_pair(8, 2, 64, 32, 64, 4)
    qi = torch.zeros((0, 2, 32), dtype=torch.bfloat16, device="cuda")
    ki = torch.zeros((64, 1, 32), dtype=torch.bfloat16, device="cuda")
    ids = msa.index_topk(p, qi, ki, q_pos0=64)
    assert ids.shape == (0, 2, 4)


def sample_rows(t, n, w, count=192, seed=0):
    rng = np.random.default_rng(seed)
    rows = list(rng.integers(0, n, count)) + [0, 1, n - 1, n - 2, w.block_k - 1, w.block_k, 2 * w.block_k + 5]
    rows += [qi for (_, qi, _) in t.get("needles", [])]
    return rows


def check_needles(t, got, w):
    for r, qi, pk in t["needles"]:
        assert pk // w.block_k in got[qi, r], (r, qi, pk)


def test_prefill_32k_sampled_rows_and_needles():
    w = WORKLOADS["prefill_32k"]
    t = make_prefill(w)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    got = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"])).cpu().numpy()
    rows = np.asarray(sorted(set(sample_rows(t, w.n_q, w))), dtype=np.int32)
    ref = oracle.index_topk(po, t["q_idx"], t["k_idx"], rows=rows)
    assert np.array_equal(got[rows], ref)
    check_needles(t, got, w)
    # Properties that hold on every row: ascending unique ids, local block present, causal.
    loc = np.arange(w.n_q) // w.block_k
    assert np.all(got[:, :, :] <= loc[:, None, None])
    assert np.all((got == loc[:, None, None]).sum(axis=2) == 1)
    v = np.where(got < 0, 1 << 30, got)
    assert np.all((np.diff(v, axis=2) > 0) | (v[:, :, 1:] == 1 << 30))


def test_prefill_128k_sampled_rows_and_needles():
    w = WORKLOADS["prefill_128k"]
    t = make_prefill(w)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    got = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"])).cpu().numpy()
    rows = np.asarray(sorted(set(sample_rows(t, w.n_q, w, count=96))), dtype=np.int32)
    ref = oracle.index_topk(po, t["q_idx"], t["k_idx"], rows=rows)
    assert np.array_equal(got[rows], ref)
    check_needles(t, got, w)


def test_chunked_prefill_1m_sampled_rows():
    w = WORKLOADS["chunked_prefill_1m"]
    t = make_prefill(w)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    got = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]), q_pos0=t["q_pos0"]).cpu().numpy()
    rows = np.asarray(sorted(set(sample_rows(t, w.n_q, w, count=24))), dtype=np.int32)
    ref = oracle.index_topk(po, t["q_idx"], t["k_idx"], q_pos0=t["q_pos0"], rows=rows)
    assert np.array_equal(got[rows], ref)
    check_needles(t, got, w)


# Mean-pool ablation (the MoBA-style pooling the m.163.com post compares the
# max-pool with): ids must still match the oracle bit for bit, partial
# (ragged or causal) blocks included.
@pytest.mark.parametrize("kw", [
    dict(n_q=1000, n_kv=1000),
    dict(n_q=77, n_kv=1000),
    dict(n_q=700, n_kv=900, d_idx=128, block_k=128, topk=5),
    dict(n_q=600, n_kv=600, topk=32, block_k=64),
])
@pytest.mark.parametrize("force_local", [1, 0])
def test_mean_pool_shapes(kw, force_local):
    run_case(small(seed=kw.get("n_q", 1) + 17, **kw), force_local=force_local, pool=msa.POOL_MEAN)


def test_mean_pool_prefill_32k_sampled_rows():
    w = WORKLOADS["prefill_32k"]
    rng = np.random.default_rng(11)
    run_case(w, rows=list(rng.integers(0, w.n_q, 48)) + [0, 127, 128, w.n_q - 1], pool=msa.POOL_MEAN)


def test_mean_and_max_pool_select_differently():
    # On the 32K workload the two poolings must disagree somewhere (the
    # ablation is not a no-op), while each matches its oracle above.
    w = WORKLOADS["prefill_32k"]
    _, a = run_case(w, rows=[w.n_q - 1], pool=msa.POOL_MAX)
    _, b = run_case(w, rows=[w.n_q - 1], pool=msa.POOL_MEAN)
    assert not np.array_equal(a, b)
