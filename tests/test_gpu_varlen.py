"""GPU parity of the packed-batch (varlen) prefill entry points against the
oracle: each sequence of the batch is an independent causal prefill, so the
reference is the fp64 oracle on each sequence's rows.  Block ids bit for bit,
O within 1e-2 abs + 1e-2 rel; adaptive per-sequence k; a batch of one
sequence equals the single-sequence calls exactly."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import Workload, make_varlen_prefill
from tests.gpu_util import assert_close, dev, host_f64, params_pair

pytestmark = pytest.mark.gpu


def wl(**kw):
    base = dict(name="varlen", kind="varlen", h_q=8, h_kv=2, d=64, d_idx=32, block_k=64, topk=4, seed=500,
                batch=6, kv_min=1, kv_max=1500, needles=2)
    base.update(kw)
    return Workload(**base)


def run_case(w, lens=None, topk_seq=None, rows=None, force_local=1, pool=0):
    t = make_varlen_prefill(w, lens)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, 1, force_local, pool=pool)
    cu = torch.from_numpy(t["cu_seqlens"]).cuda()
    kseq = None if topk_seq is None else torch.tensor(topk_seq, dtype=torch.int32, device="cuda")
    ids = msa.index_topk_varlen(p, dev(t["q_idx"]), dev(t["k_idx"]), cu, kseq)
    o = msa.sparse_attn_prefill_varlen(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), cu, ids)
    torch.cuda.synchronize()
    total = t["q"].shape[0]
    rows = np.arange(total) if rows is None else np.asarray(sorted(set(int(r) for r in rows if 0 <= r < total)))
    ids_ref = oracle.index_topk_varlen(po, t["q_idx"], t["k_idx"], t["cu_seqlens"], topk_seq, rows=rows)
    got_ids = ids.cpu().numpy()[rows]
    bad = np.argwhere(got_ids != ids_ref)
    assert bad.size == 0, ("ids differ", bad[:4].tolist(), got_ids[bad[0][0]].tolist(), ids_ref[bad[0][0]].tolist())
    o_ref = oracle.sparse_attn_varlen(po, t["q"], t["k"], t["v"], ids_ref, t["cu_seqlens"], rows=rows)
    assert_close(host_f64(o)[rows], o_ref, what="varlen O")
    return t, ids.cpu().numpy(), host_f64(o)


def test_ragged_lengths_all_rows():
    # Empty, single-token, block-edge and multi-tile sequences in one batch.
    run_case(wl(), lens=[1, 63, 64, 65, 0, 1000, 129, 300])


def test_random_lengths_all_rows():
    run_case(wl(batch=9, seed=501))


@pytest.mark.parametrize("force_local", [1, 0])
def test_adaptive_k_per_sequence(force_local):
    w = wl(topk=8, seed=502)
    run_case(w, lens=[900, 40, 1300, 513, 700], topk_seq=[8, 1, 3, 5, 100], force_local=force_local)


def test_mean_pool_varlen():
    run_case(wl(seed=503), lens=[700, 65, 1100], pool=msa.POOL_MEAN)


def test_model_shaped_batch_sampled_rows():
    # 64 query heads, 4 KV heads, d = 128, B_k = 128, k = 16; 8 sequences of
    # 1K-9K tokens with planted needles; every sequence edge sampled.
    w = wl(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=8, kv_min=1000, kv_max=9000, seed=504,
           needles=8)
    t = make_varlen_prefill(w)
    cu = t["cu_seqlens"]
    rng = np.random.default_rng(1)
    rows = list(rng.integers(0, int(cu[-1]), 96)) + [int(x) for x in cu[1:-1]] + [int(x) - 1 for x in cu[1:]]
    _, ids, _ = run_case(w, rows=rows)
    for s, r, i, pk in t["needles"]:      # needles recalled (their key block is selected)
        assert pk // w.block_k in ids[int(cu[s]) + i, r]


def test_batch_of_one_equals_single_sequence_calls():
    w = wl(h_q=16, h_kv=4, d=128, d_idx=64, block_k=128, topk=6, seed=505)
    t = make_varlen_prefill(w, lens=[1777])
    p, _ = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    cu = torch.from_numpy(t["cu_seqlens"]).cuda()
    ids_v = msa.index_topk_varlen(p, dev(t["q_idx"]), dev(t["k_idx"]), cu)
    o_v = msa.sparse_attn_prefill_varlen(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), cu, ids_v)
    ids_1 = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]))
    o_1 = msa.sparse_attn_prefill(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), ids_1)
    torch.cuda.synchronize()
    assert torch.equal(ids_v, ids_1)
    assert torch.equal(o_v, o_1)


def test_invalid_cu_seqlens_is_reported_not_computed():
    w = wl(seed=506)
    t = make_varlen_prefill(w, lens=[100, 200])
    p, _ = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    bad = torch.tensor([0, 200, 150], dtype=torch.int32, device="cuda")   # decreasing: a negative length
    out = torch.full((300, w.h_kv, w.topk), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MSAError) as err:
        msa.index_topk_varlen(p, dev(t["q_idx"]), dev(t["k_idx"]), bad, block_ids=out)
    assert err.value.code == -1
    assert torch.all(out == -7)           # nothing was written
    short = torch.tensor([0, 100, 250], dtype=torch.int32, device="cuda")  # cu[batch] != total rows (300)
    with pytest.raises(msa.MSAError) as err:
        msa.index_topk_varlen(p, dev(t["q_idx"]), dev(t["k_idx"]), short, block_ids=out)
    assert err.value.code == -1
