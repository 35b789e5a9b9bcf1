"""The C ABI library loads, exports every entry point include/msa.h declares,
and rejects bad arguments on the host (no GPU needed: every call here fails
validation before anything touches CUDA)."""
import ctypes as C
import os
import re

import pytest

import long_context_index_b200 as msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in ("msa.h", "msa_testing.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"^MSA_API [^(]*?\b(msa_\w+)\(", src, re.M))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = msa.lib()
    names = declared_symbols()
    assert set(names) == set(msa.SYMBOLS), names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    assert msa.status_string(0) == "ok"
    assert msa.status_string(-4) == "workspace too small"
    assert msa.status_string(-6) == "kernel wait timed out"


def test_options_are_host_only_and_validated():
    prev = msa.get_option(msa.OPT_DECODE_FUSED)
    assert prev in (0, 1)
    try:
        for v in (1, 0):
            msa.set_option(msa.OPT_DECODE_FUSED, v)
            assert msa.get_option(msa.OPT_DECODE_FUSED) == v
        for opt, v in ((msa.OPT_DECODE_FUSED, 2), (msa.OPT_DECODE_FUSED, -1), (7, 0)):
            with pytest.raises(msa.MSAError) as err:
                msa.set_option(opt, v)
            assert err.value.code == -1
        with pytest.raises(msa.MSAError):
            msa.get_option(7)
    finally:
        msa.set_option(msa.OPT_DECODE_FUSED, prev)


def P(**kw):
    base = dict(h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16)
    base.update(kw)
    return msa.Params.make(**base)


def test_workspace_size_is_host_only_and_validates():
    assert msa.workspace_size(msa.OP_INDEX_TOPK, P(), 1024, 1024) >= 256
    assert msa.workspace_size(msa.OP_PREFILL, P(), 131072, 131072) >= 256
    dec = msa.workspace_size(msa.OP_DECODE, P(), batch=64, max_kv=131072)
    assert dec > 64 * 64 * 16 * 130 * 4      # holds the split partials
    assert msa.workspace_size(msa.OP_INDEX_TOPK, P(d=96), 10, 10) == 0
    assert msa.workspace_size(msa.OP_INDEX_TOPK, P(h_q=6, h_kv=4), 10, 10) == 0
    assert msa.workspace_size(msa.OP_DECODE, P(), batch=0, max_kv=10) == 0
    assert msa.workspace_size(7, P(), 10, 10) == 0
    assert msa.workspace_size(msa.OP_INDEX_TOPK, P(pool=msa.POOL_MEAN), 10, 10) >= 256
    assert msa.workspace_size(msa.OP_INDEX_TOPK, P(pool=-1), 10, 10) == 0


def call_index(p, n_q=128, n_kv=128, q_pos0=0, qi=16, ki=16, ids=16, ws=256, ws_bytes=1 << 20):
    return msa.lib().msa_index_topk(C.byref(p), qi, ki, n_q, n_kv, q_pos0, ids, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), -2), (dict(d_idx=48), -2), (dict(block_k=32), -2), (dict(topk=33), -2),
    (dict(h_q=48, h_kv=32), -2), (dict(h_q=6, h_kv=4), -2), (dict(topk=0), -1), (dict(causal=2), -1),
    (dict(pool=2), -1),
])
def test_index_rejects_bad_params(kw, code):
    assert call_index(P(**kw)) == code


def test_index_rejects_bad_sizes_pointers_and_workspace():
    p = P()
    assert call_index(p, n_q=-1) == -1
    assert call_index(p, n_q=200, n_kv=100) == -1           # q_pos0 + n_q > n_kv
    assert call_index(p, q_pos0=-3) == -1
    assert call_index(p, n_kv=(1 << 24) + 1) == -2
    assert call_index(p, qi=None) == -1
    assert call_index(p, qi=18) == -3                        # not 16-byte aligned
    assert call_index(p, ws=None) == -1
    assert call_index(p, ws=512 + 16) == -3                  # workspace not 256-byte aligned
    assert call_index(p, ws_bytes=100) == -4


def test_prefill_and_decode_reject_bad_arguments():
    L = msa.lib()
    p = P()
    assert L.msa_sparse_attn_prefill(C.byref(p), 16, 16, 16, None, 10, 5, 0, 16, 256, 1 << 20, None) == -1
    assert L.msa_sparse_attn_prefill(C.byref(p), 16, 16, 16, 8, 10, 10, 0, 16, 256, 1 << 40, None) == -3
    assert L.msa_sparse_attn_decode(C.byref(p), 16, 16, 16, 16, 16, 16, 0, 100, 0, 16, 16, 256, 1 << 30,
                                    None) == -1
    assert L.msa_sparse_attn_decode(C.byref(p), 16, 16, 16, 16, 16, 16, 4, 100, 0, 16, 16, 256, 10, None) == -4
    assert L.msa_sparse_attn_decode(C.byref(p), 16, None, 16, 16, None, 16, 4, 100, 0, None, 16, 256,
                                    1 << 30, None) == -1
    # Sparse prefill sizes whose schedule would overflow its 32-bit indices:
    # 2^24 rows x 128 groups x 32 slots, refused before any launch.
    big = P(h_q=128, h_kv=128, d=64, d_idx=32, block_k=64, topk=32)
    n = 1 << 24
    assert L.msa_sparse_attn_prefill(C.byref(big), 16, 16, 16, 16, n, n, 0, 16, 256, 1 << 62, None) == -2
    assert L.msa_sparse_attn_prefill_varlen(C.byref(big), 16, 16, 16, 16, 1, n, 16, 16, 256, 1 << 62,
                                            None) == -2
    # MXFP8 decode: code arrays 16-byte aligned, K/V scales 4-byte aligned.
    mx = L.msa_sparse_attn_decode_mxfp8
    args = lambda k8=16, k_sc=16: (C.byref(p), 16, 16, k8, k_sc, 16, 16, 16, 16, 16, None, 4, 100, 16,
                                   16, 256, 1 << 40, None)
    assert mx(*args(k8=24)) == -3
    assert mx(*args(k_sc=18)) == -3
    assert L.msa_sparse_attn_decode_mxfp8(C.byref(P(d=64)), *args(16)[1:]) == -2   # d = 128 only
    # Decode limits, refused on the host before any launch: more than 8 groups;
    # a sparse batch above 4096 or with batch * max_kv >= 2^31 (dense is fine).
    wide = P(h_q=32, h_kv=16)
    assert L.msa_sparse_attn_decode(C.byref(wide), 16, 16, 16, 16, 16, 16, 4, 100, 0, 16, 16, 256, 1 << 40,
                                    None) == -2
    assert L.msa_sparse_attn_decode(C.byref(p), 16, 16, 16, 16, 16, 16, 4097, 100, 0, 16, 16, 256, 1 << 40,
                                    None) == -2
    assert L.msa_sparse_attn_decode(C.byref(p), 16, 16, 16, 16, 16, 16, 4096, 1 << 20, 0, 16, 16, 256,
                                    1 << 40, None) == -2
