"""The allocation-free decode entry point (msa_sparse_attn_decode_noalloc).

Some callers cannot allocate device memory at all -- a runtime that owns and
pre-partitions the whole GPU, or a plugin handed only its inputs and outputs.
For them the library keeps the decode step's scratch in a fixed device array
(MSA_NOALLOC_SCRATCH_BYTES per GPU) and offers an entry point without a
workspace argument.  This test calls it through the C ABI twice in a row and
checks both results against the workspace entry point's, and that a problem
too large for the fixed array is refused.

The file is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
from synth import Workload, make_decode
from tests.gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 16 << 20   # MSA_NOALLOC_SCRATCH_BYTES in include/msa.h


def call_noalloc(p, t, max_kv, ids, out):
    L = msa.lib()
    rc = L.msa_sparse_attn_decode_noalloc(
        C.byref(p), t["q"].data_ptr(), t["q_idx"].data_ptr(), t["k_cache"].data_ptr(), t["v_cache"].data_ptr(),
        t["k_idx_cache"].data_ptr(), t["cu_kv"].data_ptr(), t["q"].shape[0], max_kv, 0, ids.data_ptr(),
        out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return rc


def test_noalloc_decode_matches_workspace_decode_twice():
    w = Workload("noalloc", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=77, batch=6,
                 kv_min=3000, kv_max=40000, needles=8)
    h = make_decode(w)
    t = {k: dev(h[k]) for k in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache", "cu_kv")}
    max_kv = int(h["lens"].max())
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    assert msa.workspace_size(msa.OP_DECODE, p, batch=w.batch, max_kv=max_kv) <= NOALLOC_BYTES
    ids_ref, o_ref = msa.sparse_attn_decode(p, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"],
                                            t["cu_kv"], max_kv)
    torch.cuda.synchronize()
    ids_ref = ids_ref.cpu().numpy()
    o_ref = host_f64(o_ref)
    for _ in range(2):
        ids = torch.full((w.batch, w.h_kv, w.topk), -7, dtype=torch.int32, device="cuda")
        out = torch.zeros((w.batch, w.h_q, w.d), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(p, t, max_kv, ids, out) == 0
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ids_ref)
        assert_close(host_f64(out), o_ref, what="no-alloc decode O")


def test_noalloc_decode_refuses_problems_beyond_its_scratch():
    p = msa.Params.make(64, 4, 128, 64, 128, 16)
    B, max_kv = 64, 131072
    assert msa.workspace_size(msa.OP_DECODE, p, batch=B, max_kv=max_kv) > NOALLOC_BYTES
    q = torch.zeros((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    q_idx = torch.zeros((B, 4, 64), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B * 8, 4, 128), dtype=torch.bfloat16, device="cuda")
    ki = torch.zeros((B * 8, 1, 64), dtype=torch.bfloat16, device="cuda")
    cu = torch.arange(0, B * 8 + 1, 8, dtype=torch.int64, device="cuda")
    t = {"q": q, "q_idx": q_idx, "k_cache": kc, "v_cache": kc, "k_idx_cache": ki, "cu_kv": cu}
    ids = torch.empty((B, 4, 16), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(p, t, max_kv, ids, out) == -4   # MSA_ERR_WORKSPACE: exceeds the fixed scratch
