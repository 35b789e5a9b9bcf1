"""GPU parity of the prefill main branch (msa_sparse_attn_prefill) against the
fp64 oracle: |O_gpu - O_ref| <= 1e-2 + 1e-2 |O_ref| elementwise (bf16 inputs,
fp32 accumulation, bf16 output).  The oracle uses its own block ids, which
the index tests prove equal to the GPU's."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import WORKLOADS, Workload, make_prefill
from tests.gpu_util import assert_close, dev, host_f64, params_pair

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(name="case", kind="prefill", h_q=8, h_kv=2, d=64, d_idx=32, block_k=64, topk=4, seed=200,
                n_q=1024, n_kv=1024, needles=0)
    base.update(kw)
    return Workload(**base)


def run_case(w, n_q=None, n_kv=None, rows=None, causal=1, force_local=1, dense=False):
    t = make_prefill(w, n_q=n_q, n_kv=n_kv)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, causal, force_local)
    q, k, v = dev(t["q"]), dev(t["k"]), dev(t["v"])
    nq = t["q"].shape[0]
    if rows is None:
        rows = np.arange(nq)
    rows = np.asarray(sorted(set(int(r) for r in rows if 0 <= r < nq)), dtype=np.int32)
    if dense:
        o = msa.sparse_attn_prefill(p, q, k, v, None, q_pos0=t["q_pos0"])
        ref = oracle.dense_attn(po, t["q"], t["k"], t["v"], q_pos0=t["q_pos0"], rows=rows)
    else:
        ids = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]), q_pos0=t["q_pos0"])
        o = msa.sparse_attn_prefill(p, q, k, v, ids, q_pos0=t["q_pos0"])
        ids_ref = oracle.index_topk(po, t["q_idx"], t["k_idx"], q_pos0=t["q_pos0"], rows=rows)
        assert np.array_equal(ids.cpu().numpy()[rows], ids_ref)
        ref = oracle.sparse_attn(po, t["q"], t["k"], t["v"], ids_ref, q_pos0=t["q_pos0"], rows=rows)
    torch.cuda.synchronize()
    got = host_f64(o)[rows]
    assert_close(got, ref, what="O")
    return got, ref


def test_tiny_prefill_1k_sparse_all_rows():
    run_case(WORKLOADS["tiny_prefill_1k"])


def test_tiny_prefill_1k_dense_all_rows():
    run_case(WORKLOADS["tiny_prefill_1k"], dense=True)


def test_all_blocks_selected_equals_dense():
    # k >= number of blocks: the sparse kernel must reproduce dense attention.
    w = small(n_q=512, n_kv=512, topk=8, seed=3)
    got_s, _ = run_case(w)
    got_d, _ = run_case(w, dense=True)
    assert np.max(np.abs(got_s - got_d)) < 2e-2


@pytest.mark.parametrize("kw", [
    dict(n_q=1000, n_kv=1000),                                       # ragged tails
    dict(n_q=77, n_kv=1000),                                         # chunked, unaligned q_pos0
    dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, n_q=2048, n_kv=2048),
    dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=4, n_q=300, n_kv=1300),
    dict(h_q=16, h_kv=4, d=128, d_idx=64, block_k=64, topk=6, n_q=700, n_kv=700),
    dict(h_q=8, h_kv=8, d=64, d_idx=32, block_k=128, topk=3, n_q=500, n_kv=500),   # MHA (group size 1)
    dict(n_q=1, n_kv=1),
])
def test_shapes(kw):
    run_case(small(seed=kw.get("n_q", 1) + 11, **kw))


@pytest.mark.parametrize("kw", [
    dict(n_q=640, n_kv=640),
    dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, n_q=100, n_kv=1100),
])
def test_dense_shapes(kw):
    run_case(small(seed=kw.get("n_q", 1) + 13, **kw), dense=True)


def test_force_local_off():
    run_case(small(n_q=600, n_kv=600, seed=17), force_local=0)


def test_noncausal():
    run_case(small(n_q=256, n_kv=520, seed=19), causal=0)
    run_case(small(n_q=256, n_kv=520, seed=19), causal=0, dense=True)


def sampled(w, count, seed=0):
    rng = np.random.default_rng(seed)
    return list(rng.integers(0, w.n_q, count)) + [0, 1, 127, 128, w.n_q - 1]


def test_prefill_32k_sampled_rows():
    w = WORKLOADS["prefill_32k"]
    run_case(w, rows=sampled(w, 64))


# Rows on both sides of the block-major schedule's query-wave boundaries
# (waves of 4096 rows), where a list of one wave ends and the next begins.
WAVE_EDGES = [4095, 4096, 8191, 8192, 65535, 65536]


def test_prefill_128k_sampled_rows():
    w = WORKLOADS["prefill_128k"]
    run_case(w, rows=sampled(w, 32) + WAVE_EDGES)


def test_prefill_128k_dense_sampled_rows():
    # The dense run (every causal block, eq. (1)) that the sparse/dense ratio
    # of the benchmark divides by, on 64 sampled rows of the 128K prefill.
    w = WORKLOADS["prefill_128k"]
    run_case(w, rows=sampled(w, 59, seed=5), dense=True)


def test_chunked_prefill_1m_dense_sampled_rows():
    w = WORKLOADS["chunked_prefill_1m"]
    rng = np.random.default_rng(6)
    run_case(w, rows=list(rng.integers(0, w.n_q, 62)) + [0, w.n_q - 1], dense=True)


def test_chunked_prefill_1m_sampled_rows():
    w = WORKLOADS["chunked_prefill_1m"]
    rng = np.random.default_rng(4)
    rows = list(rng.integers(0, w.n_q, 12)) + [0, w.n_q - 1]
    run_case(w, rows=rows)
