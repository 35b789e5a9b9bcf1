"""The allocation-free decode entry point (msa_sparse_attn_decode_noalloc).

Some callers cannot allocate device memory at all -- a runtime that owns and
pre-partitions the whole GPU, or a plugin handed only its inputs and outputs.
For them the library keeps the decode step's scratch in a fixed device array
(MSA_NOALLOC_SCRATCH_BYTES per GPU) and offers an entry point without a
workspace argument.  These tests call it through the C ABI twice in a row and
check both results against the workspace entry point's and against the fp64
oracle, run it at the 64-sequence batch of the decode benchmark, and check
that a problem too large for the fixed array is refused.

The file is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
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


def run_twice(w, max_kv=None, oracle_seqs=None):
    h = make_decode(w)
    t = {k: dev(h[k]) for k in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache", "cu_kv")}
    max_kv = int(h["lens"].max()) if max_kv is None else max_kv
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids_ref, o_ref = msa.sparse_attn_decode(p, t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"],
                                            t["cu_kv"], max_kv)
    torch.cuda.synchronize()
    ids_ref = ids_ref.cpu().numpy()
    o_ref = host_f64(o_ref)
    seqs = np.arange(w.batch) if oracle_seqs is None else np.asarray(oracle_seqs)
    po = oracle.params(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids_or, o_or = oracle.decode(po, h["q"], h["q_idx"], h["k_cache"], h["v_cache"], h["k_idx_cache"], h["cu_kv"],
                                 seqs=seqs)
    for _ in range(2):
        ids = torch.full((w.batch, w.h_kv, w.topk), -7, dtype=torch.int32, device="cuda")
        out = torch.zeros((w.batch, w.h_q, w.d), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(p, t, max_kv, ids, out) == 0
        torch.cuda.synchronize()
        got_ids, got_o = ids.cpu().numpy(), host_f64(out)
        assert np.array_equal(got_ids, ids_ref)
        assert_close(got_o, o_ref, what="no-alloc decode O vs the workspace entry point")
        # Against the oracle as well: a fault shared by both entry points
        # would pass the comparison above.
        assert np.array_equal(got_ids[seqs], ids_or)
        assert_close(got_o[seqs], o_or, what="no-alloc decode O vs the oracle")


def test_noalloc_decode_matches_workspace_decode_and_oracle_twice():
    run_twice(Workload("noalloc", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=77,
                       batch=6, kv_min=3000, kv_max=40000, needles=8))


def test_noalloc_decode_at_the_benchmark_batch():
    # 64 sequences with max_kv = 131072 (the decode benchmark's bound): the
    # sparse run's scratch fits the fixed array.  Shorter caches keep the test
    # quick; the scratch depends on the batch and the bound, not on the data.
    w = Workload("noalloc64", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=78,
                 batch=64, kv_min=2000, kv_max=9000, needles=8)
    run_twice(w, max_kv=131072, oracle_seqs=[0, 1, 31, 62, 63])


def test_noalloc_decode_refuses_problems_beyond_its_scratch():
    # 512 sequences x 8 groups: the sparse run's per-share partials alone
    # (about 36 MB) exceed the fixed array.
    p = msa.Params.make(64, 8, 128, 64, 128, 16)
    B, max_kv = 512, 4096
    assert msa.workspace_size(msa.OP_DECODE, p, batch=B, max_kv=max_kv) > NOALLOC_BYTES
    q = torch.zeros((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    q_idx = torch.zeros((B, 8, 64), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B * 8, 8, 128), dtype=torch.bfloat16, device="cuda")
    ki = torch.zeros((B * 8, 1, 64), dtype=torch.bfloat16, device="cuda")
    cu = torch.arange(0, B * 8 + 1, 8, dtype=torch.int64, device="cuda")
    t = {"q": q, "q_idx": q_idx, "k_cache": kc, "v_cache": kc, "k_idx_cache": ki, "cu_kv": cu}
    ids = torch.empty((B, 8, 16), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(p, t, max_kv, ids, out) == -4   # MSA_ERR_WORKSPACE: exceeds the fixed scratch
