"""Out-of-bounds writes and malformed ids, checked on the host (no device-side
checks needed): every output of every entry point sits in a larger buffer
whose guard bytes before and after it must be untouched after the call, and
every block-id list must be ascending, -1 padded at the end only, and inside
the block range of its row."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
from synth import WORKLOADS, Workload, make_decode, make_index_projection, make_prefill, make_varlen_prefill
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes each side (keeps the output 4096-byte aligned)
FILL = 0xA5


class Guarded:
    """An output tensor of `shape` inside a buffer with guard bytes around it."""

    def __init__(self, shape, dtype):
        item = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * item
        self.buf = torch.full((2 * GUARD + self.n,), FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + self.n].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:GUARD].cpu().numpy()
        tail = self.buf[GUARD + self.n:].cpu().numpy()
        assert np.all(head == FILL) and np.all(tail == FILL), "%s wrote outside its output" % what


def check_ids(ids, n_blocks, what):
    """ids [rows, h_kv, k] int32: ascending, -1 only as a suffix, < the row's block count
    (n_blocks: scalar or [rows])."""
    ids = np.asarray(ids)
    valid = ids >= 0
    assert np.all(ids[~valid] == -1), what + ": negative ids other than -1"
    assert np.all(valid[..., 1:] <= valid[..., :-1]), what + ": -1 before a valid id"
    both = valid[..., 1:] & valid[..., :-1]
    assert np.all(ids[..., 1:][both] > ids[..., :-1][both]), what + ": ids not strictly ascending"
    nb = np.broadcast_to(np.asarray(n_blocks).reshape(-1, 1, 1), ids.shape)
    assert np.all(ids[valid] < nb[valid]), what + ": id past the row's blocks"
    assert np.all(valid[..., 0]) or what.startswith("dense"), what + ": a row with no block"


def test_prefill_outputs_stay_in_bounds():
    w = Workload(**{**WORKLOADS["tiny_prefill_1k"].__dict__, "n_q": 1000, "n_kv": 1000, "name": "g"})
    t = make_prefill(w)
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids = Guarded((w.n_q, w.h_kv, w.topk), torch.int32)
    msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]), block_ids=ids.t)
    ids.check("msa_index_topk")
    rows_blocks = np.arange(w.n_q) // w.block_k + 1          # causal blocks of row i
    check_ids(ids.t.cpu().numpy(), rows_blocks, "prefill ids")
    for block_ids in (ids.t, None):                            # sparse, then dense
        o = Guarded((w.n_q, w.h_q, w.d), torch.bfloat16)
        msa.sparse_attn_prefill(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), block_ids, out=o.t)
        o.check("msa_sparse_attn_prefill")
        assert torch.isfinite(o.t.float()).all()


def test_index_ids_well_formed_at_32k():
    # Every row of the 32K prefill (several waves of the block-major schedule).
    w = WORKLOADS["prefill_32k"]
    t = make_prefill(w)
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids = Guarded((w.n_q, w.h_kv, w.topk), torch.int32)
    msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]), block_ids=ids.t)
    ids.check("msa_index_topk")
    check_ids(ids.t.cpu().numpy(), np.arange(w.n_q) // w.block_k + 1, "32K ids")
    o = Guarded((w.n_q, w.h_q, w.d), torch.bfloat16)
    msa.sparse_attn_prefill(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), ids.t, out=o.t)
    o.check("msa_sparse_attn_prefill")


def test_decode_outputs_stay_in_bounds():
    w = Workload("g", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128, topk=16, seed=71, batch=9,
                 kv_min=1, kv_max=20000, needles=2)
    t = make_decode(w)
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    nb = (t["lens"] + w.block_k - 1) // w.block_k
    args = (dev(t["q"]), dev(t["q_idx"]), dev(t["k_cache"]), dev(t["v_cache"]), dev(t["k_idx_cache"]),
            dev(t["cu_kv"]), int(t["lens"].max()))
    ks = torch.tensor([16, 1, 3, 40, 7, 16, 2, 9, 5], dtype=torch.int32, device="cuda")
    for dense, topk_per_seq in ((False, None), (True, None), (False, ks)):
        ids = Guarded((w.batch, w.h_kv, w.topk), torch.int32)
        o = Guarded((w.batch, w.h_q, w.d), torch.bfloat16)
        msa.sparse_attn_decode(p, *args, dense=dense, block_ids=None if dense else ids.t, out=o.t,
                               topk_per_seq=topk_per_seq)
        o.check("msa_sparse_attn_decode")
        ids.check("msa_sparse_attn_decode ids")
        if not dense:
            check_ids(ids.t.cpu().numpy(), nb, "decode ids")
        assert torch.isfinite(o.t.float()).all()
    q8 = {k: msa.quantize_mxfp8(dev(t[k])) for k in ("k_cache", "v_cache", "k_idx_cache")}
    ids = Guarded((w.batch, w.h_kv, w.topk), torch.int32)
    o = Guarded((w.batch, w.h_q, w.d), torch.bfloat16)
    msa.sparse_attn_decode_mxfp8(p, dev(t["q"]), dev(t["q_idx"]), q8["k_cache"][0], q8["k_cache"][1],
                                 q8["v_cache"][0], q8["v_cache"][1], q8["k_idx_cache"][0], q8["k_idx_cache"][1],
                                 dev(t["cu_kv"]), int(t["lens"].max()), block_ids=ids.t, out=o.t)
    o.check("msa_sparse_attn_decode_mxfp8")
    ids.check("msa_sparse_attn_decode_mxfp8 ids")
    check_ids(ids.t.cpu().numpy(), nb, "MXFP8 decode ids")


def test_varlen_outputs_stay_in_bounds():
    w = WORKLOADS["tiny_prefill_1k"]
    lens = [1, 300, 0, 777, 64]
    t = make_varlen_prefill(w, lens)
    total = int(sum(lens))
    p = msa.Params.make(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    cu = dev(t["cu_seqlens"])
    ids = Guarded((total, w.h_kv, w.topk), torch.int32)
    msa.index_topk_varlen(p, dev(t["q_idx"]), dev(t["k_idx"]), cu, block_ids=ids.t)
    ids.check("msa_index_topk_varlen")
    local = np.concatenate([np.arange(L) for L in lens])       # position inside the sequence
    check_ids(ids.t.cpu().numpy(), local // w.block_k + 1, "varlen ids")
    o = Guarded((total, w.h_q, w.d), torch.bfloat16)
    msa.sparse_attn_prefill_varlen(p, dev(t["q"]), dev(t["k"]), dev(t["v"]), cu, ids.t, out=o.t)
    o.check("msa_sparse_attn_prefill_varlen")
    assert torch.isfinite(o.t.float()).all()


def test_projection_and_quantiser_stay_in_bounds():
    n, d_model, h_kv, d_idx = 333, 1024, 4, 64
    tp = make_index_projection(9, n, d_model, h_kv, d_idx)
    p = msa.Params.make(64, h_kv, 128, d_idx, 128, 16)
    qi = Guarded((n, h_kv, d_idx), torch.bfloat16)
    ki = Guarded((n, 1, d_idx), torch.bfloat16)
    msa.index_project(p, dev(tp["x"]), dev(tp["w_idx"]), q_idx=qi.t, k_idx=ki.t)
    qi.check("msa_index_project q_idx")
    ki.check("msa_index_project k_idx")
    x = dev(tp["x"]).view(n, 32, 32)
    q = Guarded((n, 32, 32), torch.uint8)
    sc = Guarded((n, 32, 1), torch.uint8)
    msa.quantize_mxfp8(x, q=q.t, scales=sc.t)
    q.check("msa_quantize_mxfp8 codes")
    sc.check("msa_quantize_mxfp8 scales")
