"""GPU parity of one batched decode step (msa_sparse_attn_decode) against the
fp64 oracle: block ids bit for bit, O within 1e-2 abs + 1e-2 rel."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import WORKLOADS, Workload, make_decode
from tests.gpu_util import assert_close, dev, host_f64, params_pair

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(name="dcase", kind="decode", h_q=8, h_kv=2, d=64, d_idx=32, block_k=64, topk=4, seed=300,
                batch=5, kv_min=300, kv_max=1500, needles=2)
    base.update(kw)
    return Workload(**base)


def run_case(w, seqs=None, dense=False, force_local=1, pool=0):
    t = make_decode(w)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, 1, force_local, pool=pool)
    ids, o = msa.sparse_attn_decode(p, dev(t["q"]), dev(t["q_idx"]), dev(t["k_cache"]), dev(t["v_cache"]),
                                    dev(t["k_idx_cache"]), dev(t["cu_kv"]), int(t["lens"].max()), dense=dense)
    torch.cuda.synchronize()
    B = t["q"].shape[0]
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    ids_ref, o_ref = oracle.decode(po, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"],
                                   t["cu_kv"], seqs=seqs, dense=dense)
    if not dense:
        got_ids = ids.cpu().numpy()[seqs]
        assert np.array_equal(got_ids, ids_ref), (np.argwhere(got_ids != ids_ref)[:4])
        # Needles are recalled when the free slots can hold them all (max
        # pooling; a block mean dilutes a single planted key).
        for b, r, pk in (t["needles"] if w.topk - force_local >= w.needles and pool == 0 else []):
            if b in set(seqs.tolist()):
                assert pk // w.block_k in ids.cpu().numpy()[b, r]
    assert_close(host_f64(o)[seqs], o_ref, what="decode O")


def test_small_decode():
    run_case(small())


def test_small_decode_dense():
    run_case(small(), dense=True)


@pytest.mark.parametrize("kw", [
    dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=3, kv_min=5000, kv_max=20000),
    dict(h_q=16, h_kv=4, d=128, d_idx=64, block_k=64, topk=6, batch=4, kv_min=1, kv_max=700),
    dict(h_q=64, h_kv=2, d=64, d_idx=128, block_k=128, topk=32, batch=2, kv_min=9000, kv_max=9000),  # 2 head tiles
    dict(batch=7, kv_min=64, kv_max=64),           # one full block per sequence
    dict(batch=3, kv_min=1, kv_max=3),             # tiny caches
    dict(topk=1, batch=3),                         # the local block alone
    dict(h_q=4, h_kv=4, d=128, d_idx=32, block_k=128, topk=3, batch=9, kv_min=100, kv_max=3000),  # group of 1
    dict(h_q=128, h_kv=1, d=128, d_idx=64, block_k=64, topk=8, batch=2, kv_min=2000, kv_max=4000),  # 8 head tiles
])
def test_shapes(kw):
    run_case(small(seed=kw.get("batch", 1) * 31 + kw.get("kv_max", 0), **kw))


def test_force_local_off():
    run_case(small(seed=41), force_local=0)


@pytest.mark.parametrize("force_local", [1, 0])
def test_mean_pool_decode(force_local):
    # Mean-pool ablation: ids bit for bit, including the partial last block
    # (ranked when force_local = 0).
    run_case(small(seed=43, batch=6, kv_min=100, kv_max=3000), force_local=force_local, pool=msa.POOL_MEAN)
    run_case(small(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=3, kv_min=5000, kv_max=20000,
                   seed=44), force_local=force_local, pool=msa.POOL_MEAN)


def test_decode_b64_64k_128k():
    run_case(WORKLOADS["decode_b64_64k_128k"])


def test_decode_b64_64k_128k_dense_sampled():
    run_case(WORKLOADS["decode_b64_64k_128k"], dense=True, seqs=[0, 17, 63])


def test_decode_b8_1m():
    run_case(WORKLOADS["decode_b8_1m"])


def test_decode_b8_1m_dense():
    # The dense decode run at 2^20 that the decode sparse/dense ratio divides by.
    run_case(WORKLOADS["decode_b8_1m"], dense=True)


@pytest.mark.parametrize("kw", [
    dict(batch=1, kv_min=200000, kv_max=200000, topk=8),          # one sequence over every index CTA
    dict(batch=3, kv_min=500, kv_max=150000, topk=16, seed=81),   # one long, two short
])
def test_top_k_merge_over_many_shares(kw):
    # A sequence whose blocks span hundreds of index CTAs: its top-k merge
    # takes many candidate chunks (the later ones by insertion).
    run_case(small(**kw))


def test_many_items_per_cta():
    # 2048 x 8 x 16 = 262144 (sequence, group, slot) items: more than 1024 per
    # CTA at 148 CTAs, so the persistent attention grid grows; sampled rows.
    w = small(h_q=32, h_kv=8, d=64, d_idx=32, block_k=64, topk=16, batch=2048, kv_min=100, kv_max=1500, seed=77)
    run_case(w, seqs=[0, 1, 777, 2047])


@pytest.mark.parametrize("pool", [0, 1])
def test_adaptive_k_per_sequence(pool):
    # Each sequence keeps its own number of blocks: ids equal the oracle's
    # selection with that k (local block included), padded with -1.
    w = small(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=7, kv_min=3000, kv_max=30000, seed=45)
    t = make_decode(w)
    ks = np.array([16, 1, 5, 2, 40, 9, 16], dtype=np.int32)
    p, _ = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, pool=pool)
    ids, o = msa.sparse_attn_decode(p, dev(t["q"]), dev(t["q_idx"]), dev(t["k_cache"]), dev(t["v_cache"]),
                                    dev(t["k_idx_cache"]), dev(t["cu_kv"]), int(t["lens"].max()),
                                    topk_per_seq=torch.from_numpy(ks).cuda())
    torch.cuda.synchronize()
    got_ids, got_o = ids.cpu().numpy(), host_f64(o)
    for b in range(w.batch):
        kb = int(min(max(ks[b], 1), w.topk))
        _, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, kb, pool=pool)
        ids_ref, o_ref = oracle.decode(po, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"],
                                       t["cu_kv"], seqs=[b])
        assert np.array_equal(got_ids[b, :, :kb], ids_ref[0]) and np.all(got_ids[b, :, kb:] == -1), b
        assert_close(got_o[b], o_ref[0], what="adaptive-k decode O, sequence %d" % b)


def test_decode_equals_prefill_row_at_last_position():
    # Entry-point consistency: a decode step and a one-row chunked prefill at
    # q_pos0 = L_b - 1 over the same caches run different kernels but must
    # select the same blocks (bit for bit) and agree on O within tolerance.
    w = small(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=4, kv_min=3000, kv_max=9000, seed=91)
    t = make_decode(w)
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids, o = msa.sparse_attn_decode(p, dev(t["q"]), dev(t["q_idx"]), dev(t["k_cache"]), dev(t["v_cache"]),
                                    dev(t["k_idx_cache"]), dev(t["cu_kv"]), int(t["lens"].max()))
    torch.cuda.synchronize()
    cu = t["cu_kv"]
    for b in range(w.batch):
        lo, hi = int(cu[b]), int(cu[b + 1])
        L = hi - lo
        pid = msa.index_topk(p, dev(t["q_idx"][b:b + 1]), dev(t["k_idx_cache"][lo:hi]), L - 1)
        po = msa.sparse_attn_prefill(p, dev(t["q"][b:b + 1]), dev(t["k_cache"][lo:hi]), dev(t["v_cache"][lo:hi]),
                                     pid, L - 1)
        torch.cuda.synchronize()
        assert torch.equal(pid[0].cpu(), ids[b].cpu()), b
        assert_close(host_f64(o[b]), host_f64(po[0]), what="decode vs prefill row, sequence %d" % b)


def test_sparse_decode_rejects_batches_beyond_the_index_prefix():
    # The sparse index scan keeps the block prefix of every sequence in shared
    # memory: batches above 4096 are refused before any launch.
    B = 4097
    p = msa.Params.make(8, 2, 64, 32, 64, 4)
    q = torch.zeros((B, 8, 64), dtype=torch.bfloat16, device="cuda")
    qi = torch.zeros((B, 2, 32), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, 2, 64), dtype=torch.bfloat16, device="cuda")
    ki = torch.zeros((B, 1, 32), dtype=torch.bfloat16, device="cuda")
    cu = torch.arange(B + 1, dtype=torch.int64, device="cuda")
    with pytest.raises(msa.MSAError) as err:
        msa.sparse_attn_decode(p, q, qi, kc, kc, ki, cu, 1)
    assert err.value.code == -2


@pytest.fixture
def fused_form():
    prev = msa.get_option(msa.OPT_DECODE_FUSED)
    msa.set_option(msa.OPT_DECODE_FUSED, 1)
    yield
    msa.set_option(msa.OPT_DECODE_FUSED, prev)


def decode_kernels(fn):
    """Names of the kernels one call of fn launches (CUPTI via torch.profiler)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events() if e.device_type.name == "CUDA"]


@pytest.mark.parametrize("kw,pool", [
    (dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, batch=3, kv_min=5000, kv_max=20000), 0),
    (dict(h_q=16, h_kv=4, d=128, d_idx=64, block_k=64, topk=6, batch=4, kv_min=1, kv_max=700), 0),
    (dict(h_q=64, h_kv=2, d=64, d_idx=128, block_k=128, topk=32, batch=2, kv_min=9000, kv_max=9000), 0),
    (dict(h_q=4, h_kv=4, d=128, d_idx=32, block_k=128, topk=3, batch=9, kv_min=100, kv_max=3000), 1),
    (dict(batch=6, kv_min=100, kv_max=3000, seed=43), 1),
])
def test_fused_decode_form(fused_form, kw, pool):
    # The one-launch form: the oracle's ids bit for bit and O within
    # tolerance, and the same ids and O bit for bit as the two launches.
    w = small(**kw)
    run_case(w, pool=pool)
    t = make_decode(w)
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, pool=pool)
    args = (p, dev(t["q"]), dev(t["q_idx"]), dev(t["k_cache"]), dev(t["v_cache"]), dev(t["k_idx_cache"]),
            dev(t["cu_kv"]), int(t["lens"].max()))
    out = {}
    names = decode_kernels(lambda: out.setdefault(1, msa.sparse_attn_decode(*args)))
    assert any("decode_fused_kernel" in n for n in names), names
    msa.set_option(msa.OPT_DECODE_FUSED, 0)
    names = decode_kernels(lambda: out.setdefault(0, msa.sparse_attn_decode(*args)))
    assert not any("decode_fused_kernel" in n for n in names), names
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])


def test_fused_decode_b64_64k_128k(fused_form):
    run_case(WORKLOADS["decode_b64_64k_128k"])
