"""MiniMax Sparse Attention (MSA) hot path for NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libmsa.so`` (C ABI in ``include/msa.h``).  This module
only marshals arguments: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (bf16, int32, int64); the binding
passes their device pointers and the current CUDA stream.  There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

__all__ = ["MSAError", "Params", "lib", "workspace_size", "index_topk", "sparse_attn_prefill",
           "sparse_attn_decode", "index_topk_varlen", "sparse_attn_prefill_varlen", "device_status",
           "status_string", "OP_INDEX_TOPK", "OP_PREFILL", "OP_DECODE", "OP_INDEX_TOPK_VARLEN",
           "OP_PREFILL_VARLEN", "OP_INDEX_PROJECT", "index_project", "quantize_mxfp8", "sparse_attn_decode_mxfp8", "POOL_MAX",
           "POOL_MEAN"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

OP_INDEX_TOPK, OP_PREFILL, OP_DECODE, OP_INDEX_TOPK_VARLEN, OP_PREFILL_VARLEN, OP_INDEX_PROJECT = 0, 1, 2, 3, 4, 5
POOL_MAX, POOL_MEAN = 0, 1   # msa_params.pool

SYMBOLS = ("msa_workspace_size", "msa_index_project", "msa_quantize_mxfp8", "msa_sparse_attn_decode_mxfp8", "msa_index_topk", "msa_sparse_attn_prefill", "msa_sparse_attn_decode",
           "msa_index_topk_varlen", "msa_sparse_attn_prefill_varlen", "msa_sparse_attn_decode_adaptive_k",
           "msa_device_status", "msa_status_string", "msa_set_option", "msa_get_option",
           "msa_sparse_attn_decode_noalloc", "msa_test_never_ready_wait")


class MSAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, status_string(code) if _lib else "?", code))
        self.code = code


class Params(C.Structure):
    """Mirror of ``msa_params`` (include/msa.h)."""
    _fields_ = [("h_q", C.c_int), ("h_kv", C.c_int), ("d", C.c_int), ("d_idx", C.c_int),
                ("block_k", C.c_int), ("topk", C.c_int), ("causal", C.c_int), ("force_local", C.c_int),
                ("scale", C.c_float), ("pool", C.c_int)]

    @classmethod
    def make(cls, h_q, h_kv, d, d_idx, block_k, topk, causal=True, force_local=True, scale=0.0, pool=0):
        return cls(h_q, h_kv, d, d_idx, block_k, topk, int(causal), int(force_local), float(scale), int(pool))


_lib = None

# When True, every call synchronises its stream and raises MSAError if a
# kernel recorded a timeout in the workspace status word (used by the tests).
check_status = False


def lib():
    """Load libmsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmsa.so not built: run `python -m long_context_index_b200.build`")
        L = C.CDLL(LIB_PATH)
        P = C.POINTER(Params)
        vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
        L.msa_workspace_size.argtypes = [i32, P, i32, i32, i32, i32]
        L.msa_workspace_size.restype = sz
        L.msa_index_topk.argtypes = [P, vp, vp, i32, i32, i32, vp, vp, sz, vp]
        L.msa_sparse_attn_prefill.argtypes = [P, vp, vp, vp, vp, i32, i32, i32, vp, vp, sz, vp]
        L.msa_sparse_attn_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]
        L.msa_sparse_attn_decode_adaptive_k.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp,
                                                        vp, sz, vp]
        L.msa_quantize_mxfp8.argtypes = [vp, C.c_longlong, i32, vp, vp, vp]
        L.msa_quantize_mxfp8.restype = i32
        L.msa_sparse_attn_decode_mxfp8.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp,
                                                   vp, sz, vp]
        L.msa_sparse_attn_decode_mxfp8.restype = i32
        L.msa_index_project.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.msa_index_topk_varlen.argtypes = [P, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.msa_sparse_attn_prefill_varlen.argtypes = [P, vp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.msa_sparse_attn_decode_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]
        L.msa_sparse_attn_decode_noalloc.restype = i32
        L.msa_test_never_ready_wait.argtypes = [vp, sz, C.c_longlong, vp]
        L.msa_test_never_ready_wait.restype = i32
        L.msa_device_status.argtypes = [vp, vp]
        L.msa_status_string.argtypes = [i32]
        L.msa_set_option.argtypes = [i32, i32]
        L.msa_get_option.argtypes = [i32]
        L.msa_status_string.restype = C.c_char_p
        for f in ("msa_index_topk", "msa_sparse_attn_prefill", "msa_sparse_attn_decode", "msa_device_status",
                  "msa_index_topk_varlen", "msa_sparse_attn_prefill_varlen", "msa_sparse_attn_decode_adaptive_k",
                  "msa_index_project"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().msa_status_string(int(code)).decode()


OPT_DECODE_FUSED = 0


def set_option(option: int, value: int) -> None:
    """Process-wide option (``msa_set_option``): OPT_DECODE_FUSED 1 runs a
    sparse decode step as one cooperative launch when it fits one wave, 0 as
    the index-scan and attention launches."""
    rc = lib().msa_set_option(int(option), int(value))
    if rc:
        raise MSAError(rc, "msa_set_option")


def get_option(option: int) -> int:
    rc = lib().msa_get_option(int(option))
    if rc < 0:
        raise MSAError(rc, "msa_get_option")
    return rc


def workspace_size(op: int, p: Params, n_q: int = 0, n_kv: int = 0, batch: int = 0, max_kv: int = 0) -> int:
    """Host-only query of the workspace bytes one call needs (0 = invalid)."""
    return int(lib().msa_workspace_size(int(op), C.byref(p), int(n_q), int(n_kv), int(batch), int(max_kv)))


# ---------------------------------------------------------------------------
# torch-facing wrappers
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(t, name, dtypes, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype not in dtypes:
        raise TypeError("%s has dtype %s, expected one of %s" % (name, t.dtype, dtypes))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))


def _stream(stream) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _workspace(op, p, n_q=0, n_kv=0, batch=0, max_kv=0, ws=None, device=None):
    torch = _torch()
    need = workspace_size(op, p, n_q, n_kv, batch, max_kv)
    if need == 0:
        raise MSAError(-1, "msa_workspace_size")
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws


def _bf16():
    torch = _torch()
    return (torch.bfloat16, torch.uint16, torch.int16)


def index_project(p: Params, x, w_idx, q_idx=None, k_idx=None, ws=None, stream=None):
    """Index projections: (Q_idx [n, h_kv, d_idx], K_idx [n, 1, d_idx]) = x W_idx^T split by rows of the
    stacked weight w_idx [(h_kv + 1) d_idx, d_model] (group query projections, then the key projection)."""
    torch = _torch()
    n, d_model = x.shape
    _check(x, "x", _bf16(), (n, d_model))
    _check(w_idx, "w_idx", _bf16(), ((p.h_kv + 1) * p.d_idx, d_model))
    if q_idx is None:
        q_idx = torch.empty((n, p.h_kv, p.d_idx), dtype=torch.bfloat16, device=x.device)
    if k_idx is None:
        k_idx = torch.empty((n, 1, p.d_idx), dtype=torch.bfloat16, device=x.device)
    _check(q_idx, "q_idx", _bf16(), (n, p.h_kv, p.d_idx))
    _check(k_idx, "k_idx", _bf16(), (n, 1, p.d_idx))
    ws = _workspace(OP_INDEX_PROJECT, p, n, ws=ws, device=x.device)
    rc = lib().msa_index_project(C.byref(p), _ptr(x), _ptr(w_idx), n, d_model, _ptr(q_idx), _ptr(k_idx), _ptr(ws),
                                 ws.numel(), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_index_project")
    _after(ws, stream, "msa_index_project")
    return q_idx, k_idx


def quantize_mxfp8(x, q=None, scales=None, stream=None):
    """MXFP8 (E4M3 + E8M0 per 32 elements of the last dim) of a bf16 tensor: (q uint8, scales uint8)."""
    torch = _torch()
    _check(x, "x", _bf16())
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(tuple(x.shape[:-1]) + (cols // 32,), dtype=torch.uint8, device=x.device)
    _check(q, "q", (torch.uint8,), tuple(x.shape))
    _check(scales, "scales", (torch.uint8,), tuple(x.shape[:-1]) + (cols // 32,))
    rc = lib().msa_quantize_mxfp8(_ptr(x), rows, cols, _ptr(q), _ptr(scales), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_quantize_mxfp8")
    return q, scales


def index_topk(p: Params, q_idx, k_idx, q_pos0: int = 0, block_ids=None, ws=None, stream=None):
    """Index branch of a prefill: block ids [n_q, h_kv, topk] (int32, ascending, -1 padded)."""
    torch = _torch()
    n_q, n_kv = q_idx.shape[0], k_idx.shape[0]
    _check(q_idx, "q_idx", _bf16(), (n_q, p.h_kv, p.d_idx))
    _check(k_idx, "k_idx", _bf16(), (n_kv, 1, p.d_idx))
    if block_ids is None:
        block_ids = torch.empty((n_q, p.h_kv, p.topk), dtype=torch.int32, device=q_idx.device)
    _check(block_ids, "block_ids", (torch.int32,), (n_q, p.h_kv, p.topk))
    ws = _workspace(OP_INDEX_TOPK, p, n_q, n_kv, ws=ws, device=q_idx.device)
    rc = lib().msa_index_topk(C.byref(p), _ptr(q_idx), _ptr(k_idx), n_q, n_kv, int(q_pos0), _ptr(block_ids),
                              _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_index_topk")
    _after(ws, stream, "msa_index_topk")
    return block_ids


def sparse_attn_prefill(p: Params, q, k, v, block_ids=None, q_pos0: int = 0, out=None, ws=None, stream=None):
    """Main branch of a prefill: O [n_q, h_q, d] bf16.  block_ids=None runs dense."""
    torch = _torch()
    n_q, n_kv = q.shape[0], k.shape[0]
    _check(q, "q", _bf16(), (n_q, p.h_q, p.d))
    _check(k, "k", _bf16(), (n_kv, p.h_kv, p.d))
    _check(v, "v", _bf16(), (n_kv, p.h_kv, p.d))
    if block_ids is not None:
        _check(block_ids, "block_ids", (torch.int32,), (n_q, p.h_kv, p.topk))
    if out is None:
        out = torch.empty((n_q, p.h_q, p.d), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", _bf16(), (n_q, p.h_q, p.d))
    ws = _workspace(OP_PREFILL, p, n_q, n_kv, ws=ws, device=q.device)
    rc = lib().msa_sparse_attn_prefill(C.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(block_ids), n_q, n_kv,
                                       int(q_pos0), _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_sparse_attn_prefill")
    _after(ws, stream, "msa_sparse_attn_prefill")
    return out


def sparse_attn_decode(p: Params, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, max_kv: int, dense=False,
                       block_ids=None, out=None, ws=None, stream=None, topk_per_seq=None):
    """One decode step: (block_ids [B, h_kv, topk] or None when dense, O [B, h_q, d]).
    ``topk_per_seq`` (int32 [B], optional): blocks kept per sequence (adaptive k)."""
    torch = _torch()
    B = q.shape[0]
    tot = k_cache.shape[0]
    _check(q, "q", _bf16(), (B, p.h_q, p.d))
    _check(k_cache, "k_cache", _bf16(), (tot, p.h_kv, p.d))
    _check(v_cache, "v_cache", _bf16(), (tot, p.h_kv, p.d))
    _check(cu_kv, "cu_kv", (torch.int64,), (B + 1,))
    if not dense:
        _check(q_idx, "q_idx", _bf16(), (B, p.h_kv, p.d_idx))
        _check(k_idx_cache, "k_idx_cache", _bf16(), (tot, 1, p.d_idx))
        if block_ids is None:
            block_ids = torch.empty((B, p.h_kv, p.topk), dtype=torch.int32, device=q.device)
        _check(block_ids, "block_ids", (torch.int32,), (B, p.h_kv, p.topk))
    if out is None:
        out = torch.empty((B, p.h_q, p.d), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", _bf16(), (B, p.h_q, p.d))
    ws = _workspace(OP_DECODE, p, batch=B, max_kv=max_kv, ws=ws, device=q.device)
    if topk_per_seq is not None:
        _check(topk_per_seq, "topk_per_seq", (torch.int32,), (B,))
        rc = lib().msa_sparse_attn_decode_adaptive_k(
            C.byref(p), _ptr(q), _ptr(q_idx) if not dense else None, _ptr(k_cache), _ptr(v_cache),
            _ptr(k_idx_cache) if not dense else None, _ptr(cu_kv), _ptr(topk_per_seq), B, int(max_kv),
            int(bool(dense)), _ptr(block_ids) if not dense else None, _ptr(out), _ptr(ws), ws.numel(),
            _stream(stream))
    else:
        rc = lib().msa_sparse_attn_decode(C.byref(p), _ptr(q), _ptr(q_idx) if not dense else None,
                                          _ptr(k_cache), _ptr(v_cache), _ptr(k_idx_cache) if not dense else None,
                                          _ptr(cu_kv), B, int(max_kv), int(bool(dense)),
                                          _ptr(block_ids) if not dense else None, _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(stream))
    if rc:
        raise MSAError(rc, "msa_sparse_attn_decode")
    _after(ws, stream, "msa_sparse_attn_decode")
    return block_ids, out


def index_topk_varlen(p: Params, q_idx, k_idx, cu_seqlens, topk_per_seq=None, block_ids=None, ws=None,
                      stream=None):
    """Index branch of a packed batch of sequences (rows [cu[s], cu[s+1]) each):
    block ids [total, h_kv, topk], local to each sequence, -1 padded.
    ``topk_per_seq`` (int32 [batch], optional): blocks kept per sequence."""
    torch = _torch()
    total = q_idx.shape[0]
    batch = cu_seqlens.shape[0] - 1
    _check(q_idx, "q_idx", _bf16(), (total, p.h_kv, p.d_idx))
    _check(k_idx, "k_idx", _bf16(), (total, 1, p.d_idx))
    _check(cu_seqlens, "cu_seqlens", (torch.int32,), (batch + 1,))
    if topk_per_seq is not None:
        _check(topk_per_seq, "topk_per_seq", (torch.int32,), (batch,))
    if block_ids is None:
        block_ids = torch.empty((total, p.h_kv, p.topk), dtype=torch.int32, device=q_idx.device)
    _check(block_ids, "block_ids", (torch.int32,), (total, p.h_kv, p.topk))
    ws = _workspace(OP_INDEX_TOPK_VARLEN, p, total, total, batch=batch, ws=ws, device=q_idx.device)
    rc = lib().msa_index_topk_varlen(C.byref(p), _ptr(q_idx), _ptr(k_idx), _ptr(cu_seqlens), batch, total,
                                     _ptr(topk_per_seq), _ptr(block_ids), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_index_topk_varlen")
    _after(ws, stream, "msa_index_topk_varlen")
    return block_ids


def sparse_attn_prefill_varlen(p: Params, q, k, v, cu_seqlens, block_ids, out=None, ws=None, stream=None):
    """Main branch of a packed batch of sequences: O [total, h_q, d] bf16."""
    torch = _torch()
    total = q.shape[0]
    batch = cu_seqlens.shape[0] - 1
    _check(q, "q", _bf16(), (total, p.h_q, p.d))
    _check(k, "k", _bf16(), (total, p.h_kv, p.d))
    _check(v, "v", _bf16(), (total, p.h_kv, p.d))
    _check(cu_seqlens, "cu_seqlens", (torch.int32,), (batch + 1,))
    _check(block_ids, "block_ids", (torch.int32,), (total, p.h_kv, p.topk))
    if out is None:
        out = torch.empty((total, p.h_q, p.d), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", _bf16(), (total, p.h_q, p.d))
    ws = _workspace(OP_PREFILL_VARLEN, p, total, total, batch=batch, ws=ws, device=q.device)
    rc = lib().msa_sparse_attn_prefill_varlen(C.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch,
                                              total, _ptr(block_ids), _ptr(out), _ptr(ws), ws.numel(),
                                              _stream(stream))
    if rc:
        raise MSAError(rc, "msa_sparse_attn_prefill_varlen")
    _after(ws, stream, "msa_sparse_attn_prefill_varlen")
    return out


def sparse_attn_decode_mxfp8(p: Params, q, q_idx, k8, k_scale, v8, v_scale, k_idx8, k_idx_scale, cu_kv,
                             max_kv: int, block_ids=None, out=None, ws=None, stream=None, topk_per_seq=None):
    """One decode step over MXFP8 caches (uint8 codes and E8M0 scales from quantize_mxfp8):
    (block_ids [B, h_kv, topk], O [B, h_q, d])."""
    torch = _torch()
    B = q.shape[0]
    tot = k8.shape[0]
    _check(q, "q", _bf16(), (B, p.h_q, p.d))
    _check(q_idx, "q_idx", _bf16(), (B, p.h_kv, p.d_idx))
    for name, t, shape in (("k8", k8, (tot, p.h_kv, p.d)), ("v8", v8, (tot, p.h_kv, p.d)),
                           ("k_scale", k_scale, (tot, p.h_kv, p.d // 32)), ("v_scale", v_scale, (tot, p.h_kv, p.d // 32)),
                           ("k_idx8", k_idx8, (tot, 1, p.d_idx)), ("k_idx_scale", k_idx_scale, (tot, 1, p.d_idx // 32))):
        _check(t, name, (torch.uint8,), shape)
    _check(cu_kv, "cu_kv", (torch.int64,), (B + 1,))
    if topk_per_seq is not None:
        _check(topk_per_seq, "topk_per_seq", (torch.int32,), (B,))
    if block_ids is None:
        block_ids = torch.empty((B, p.h_kv, p.topk), dtype=torch.int32, device=q.device)
    _check(block_ids, "block_ids", (torch.int32,), (B, p.h_kv, p.topk))
    if out is None:
        out = torch.empty((B, p.h_q, p.d), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", _bf16(), (B, p.h_q, p.d))
    ws = _workspace(OP_DECODE, p, batch=B, max_kv=max_kv, ws=ws, device=q.device)
    rc = lib().msa_sparse_attn_decode_mxfp8(C.byref(p), _ptr(q), _ptr(q_idx), _ptr(k8), _ptr(k_scale), _ptr(v8),
                                            _ptr(v_scale), _ptr(k_idx8), _ptr(k_idx_scale), _ptr(cu_kv),
                                            _ptr(topk_per_seq), B, int(max_kv), _ptr(block_ids), _ptr(out),
                                            _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise MSAError(rc, "msa_sparse_attn_decode_mxfp8")
    _after(ws, stream, "msa_sparse_attn_decode_mxfp8")
    return block_ids, out


def _after(ws, stream, what):
    if check_status:
        rc = device_status(ws, stream)
        if rc:
            raise MSAError(rc, what)


def device_status(ws, stream=None) -> int:
    """Status word of the last call that used workspace ``ws`` (synchronises)."""
    return int(lib().msa_device_status(_ptr(ws), _stream(stream)))
