"""GPU parity of the MXFP8 path: the quantiser bit for bit against the
oracle's, and the decode step over MXFP8 caches against the fp64 oracle run
on the caches the oracle itself dequantises (ids bit for bit, O within
1e-2 abs + 1e-2 rel).  Integer index inputs quantise exactly, so the ids also
equal those of the bf16 caches."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import WORKLOADS, Workload, bf16_bits_to_f32, f32_to_bf16_bits, make_decode
from tests.gpu_util import assert_close, dev, host_f64, params_pair

pytestmark = pytest.mark.gpu


def test_quantiser_bit_exact():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((777, 4, 128)).astype(np.float32)
    x *= np.exp2(rng.integers(-40, 40, size=(777, 4, 1))).astype(np.float32)   # wide block ranges
    x[3, 1, :32] = 0                                                            # a zero block
    x[5, 0, 7] = 3.0e38                                                          # near the bf16 maximum
    x[6, 2, :32] = rng.standard_normal(32).astype(np.float32) * 1e-38            # bf16 subnormals
    xb = f32_to_bf16_bits(x)
    q, s = msa.quantize_mxfp8(dev(xb))
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_mxfp8(xb)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def dequant_bits(q, s):
    return f32_to_bf16_bits(oracle.dequantize_mxfp8(q, s).astype(np.float32))


def run_case(w, seqs=None, force_local=1, big_qidx=()):
    t = make_decode(w)
    for b in big_qidx:
        # Q_idx of sequence b times 2^18: exact in bf16, beyond the f16 range
        # (scores stay exact integers times 2^18).
        t["q_idx"][b] = f32_to_bf16_bits(bf16_bits_to_f32(t["q_idx"][b]) * np.float32(2.0 ** 18))
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk, 1, force_local)
    q8 = {}
    for name in ("k_cache", "v_cache", "k_idx_cache"):
        qq, ss = msa.quantize_mxfp8(dev(t[name]))
        q8[name] = (qq, ss)
    ids, o = msa.sparse_attn_decode_mxfp8(p, dev(t["q"]), dev(t["q_idx"]), q8["k_cache"][0], q8["k_cache"][1],
                                          q8["v_cache"][0], q8["v_cache"][1], q8["k_idx_cache"][0],
                                          q8["k_idx_cache"][1], dev(t["cu_kv"]), int(t["lens"].max()))
    torch.cuda.synchronize()
    # The oracle quantises and dequantises with its own code, on the sampled
    # sequences only (a compact copy of their cache rows).
    B = t["q"].shape[0]
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    cu = t["cu_kv"]
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in seqs])
    cu_s = np.zeros(len(seqs) + 1, dtype=np.int64)
    cu_s[1:] = np.cumsum([cu[b + 1] - cu[b] for b in seqs])
    sub = {n: t[n][rows] for n in ("k_cache", "v_cache", "k_idx_cache")}
    deq = {n: dequant_bits(*oracle.quantize_mxfp8(sub[n])) for n in sub}
    qs, qis = t["q"][seqs], t["q_idx"][seqs]
    ids_ref, o_ref = oracle.decode(po, qs, qis, deq["k_cache"], deq["v_cache"], deq["k_idx_cache"], cu_s)
    got_ids = ids.cpu().numpy()[seqs]
    assert np.array_equal(got_ids, ids_ref)
    # Integer index inputs survive MXFP8 exactly: the same ids as the bf16 caches.
    ids_bf16, _ = oracle.decode(po, qs, qis, sub["k_cache"], sub["v_cache"], sub["k_idx_cache"], cu_s)
    assert np.array_equal(got_ids, ids_bf16)
    assert_close(host_f64(o)[seqs], o_ref, what="MXFP8 decode O")
    return t, ids, o


def test_mxfp8_decode_small():
    run_case(Workload("m8", "decode", h_q=16, h_kv=4, d=128, d_idx=64, block_k=64, topk=6, seed=601, batch=5,
                      kv_min=1, kv_max=3000, needles=2))


@pytest.mark.parametrize("force_local", [1, 0])
def test_mxfp8_decode_model_shape(force_local):
    run_case(Workload("m8", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=602, batch=6,
                      kv_min=5000, kv_max=40000, needles=8), force_local=force_local)


def test_mxfp8_decode_b64_64k_128k_sampled():
    run_case(WORKLOADS["decode_b64_64k_128k"], seqs=[0, 5, 31, 63])


def test_mxfp8_decode_q_idx_beyond_f16():
    # Index queries of very different magnitudes in one batch.
    run_case(Workload("m8", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=603, batch=5,
                      kv_min=3000, kv_max=20000, needles=4), big_qidx=(1, 3))


@pytest.mark.parametrize("d_idx", [32, 128])
def test_mxfp8_decode_index_widths(d_idx):
    # One and four scale blocks per index key.
    run_case(Workload("m8", "decode", h_q=32, h_kv=2, d=128, d_idx=d_idx, block_k=64, topk=8, seed=604, batch=4,
                      kv_min=100, kv_max=5000, needles=2), big_qidx=(2,))


def test_mxfp8_fused_form_matches_two_launches():
    w = Workload("m8", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=605, batch=6,
                 kv_min=5000, kv_max=30000, needles=4)
    prev = msa.get_option(msa.OPT_DECODE_FUSED)
    try:
        msa.set_option(msa.OPT_DECODE_FUSED, 1)
        _, ids1, o1 = run_case(w)
        msa.set_option(msa.OPT_DECODE_FUSED, 0)
        _, ids0, o0 = run_case(w)
    finally:
        msa.set_option(msa.OPT_DECODE_FUSED, prev)
    assert torch.equal(ids0, ids1) and torch.equal(o0, o1)
