"""ctypes front of the fp64 C++ oracle of the MSA hot path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline leg use this module; the product path never imports it.  It shares
no code with the CUDA library.  See ``msa_oracle.cpp`` for the method and the
passages each function follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.cpp")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")


class Params(C.Structure):
    _fields_ = [("h_q", C.c_int), ("h_kv", C.c_int), ("d", C.c_int), ("d_idx", C.c_int),
                ("block_k", C.c_int), ("topk", C.c_int), ("causal", C.c_int),
                ("force_local", C.c_int), ("scale", C.c_double), ("threads", C.c_int), ("pool", C.c_int)]


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.POINTER(Params)
        vp = C.c_void_p
        _lib.msa_oracle_block_scores.argtypes = [P, vp, vp, C.c_int, C.c_int, C.c_longlong, vp, C.c_int, vp]
        _lib.msa_oracle_index_topk.argtypes = [P, vp, vp, C.c_int, C.c_int, C.c_longlong, vp, C.c_int, vp]
        _lib.msa_oracle_sparse_attn.argtypes = [P, vp, vp, vp, vp, C.c_int, C.c_int, C.c_longlong, vp,
                                                C.c_int, vp, vp]
        _lib.msa_oracle_dense_attn.argtypes = [P, vp, vp, vp, C.c_int, C.c_int, C.c_longlong, vp, C.c_int,
                                               vp, vp]
        _lib.msa_oracle_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, C.c_int, vp, C.c_int, C.c_int, vp, vp]
        for f in ("msa_oracle_block_scores", "msa_oracle_index_topk", "msa_oracle_sparse_attn",
                  "msa_oracle_dense_attn", "msa_oracle_decode"):
            getattr(_lib, f).restype = C.c_int
    return _lib


POOL_MAX, POOL_MEAN = 0, 1


def params(h_q, h_kv, d, d_idx, block_k, topk, causal=1, force_local=1, scale=0.0, threads=0,
           pool=POOL_MAX) -> Params:
    return Params(h_q, h_kv, d, d_idx, block_k, topk, int(causal), int(force_local), float(scale),
                  int(threads), int(pool))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _rows(rows: Optional[Sequence[int]], n: int):
    if rows is None:
        return None, n
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    return r, int(r.size)


def block_scores(P: Params, q_idx, k_idx, q_pos0: int = 0, rows=None) -> np.ndarray:
    """Eq. (6) pooled block scores M[rows, h_kv, nb] (-inf = not eligible)."""
    q_idx, k_idx = _u16(q_idx), _u16(k_idx)
    n_q, n_kv = q_idx.shape[0], k_idx.shape[0]
    r, nr = _rows(rows, n_q)
    nb = (n_kv + P.block_k - 1) // P.block_k
    out = np.empty((nr, P.h_kv, nb), dtype=np.float64)
    rc = lib().msa_oracle_block_scores(C.byref(P), _ptr(q_idx), _ptr(k_idx), n_q, n_kv, q_pos0,
                                       _ptr(r), nr, _ptr(out))
    if rc:
        raise ValueError("oracle block_scores: bad arguments (%d)" % rc)
    return out


def index_topk(P: Params, q_idx, k_idx, q_pos0: int = 0, rows=None) -> np.ndarray:
    """Index branch: block ids[rows, h_kv, topk], ascending, -1 padded."""
    q_idx, k_idx = _u16(q_idx), _u16(k_idx)
    n_q, n_kv = q_idx.shape[0], k_idx.shape[0]
    r, nr = _rows(rows, n_q)
    out = np.empty((nr, P.h_kv, P.topk), dtype=np.int32)
    rc = lib().msa_oracle_index_topk(C.byref(P), _ptr(q_idx), _ptr(k_idx), n_q, n_kv, q_pos0,
                                     _ptr(r), nr, _ptr(out))
    if rc:
        raise ValueError("oracle index_topk: bad arguments (%d)" % rc)
    return out


def sparse_attn(P: Params, q, k, v, ids, q_pos0: int = 0, rows=None, want_lse=False):
    """Main branch, eq. (8), over the given ids (one id list per listed row)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    n_q, n_kv = q.shape[0], k.shape[0]
    r, nr = _rows(rows, n_q)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    assert ids.shape == (nr, P.h_kv, P.topk), ids.shape
    o = np.empty((nr, P.h_q, P.d), dtype=np.float64)
    lse = np.empty((nr, P.h_q), dtype=np.float64) if want_lse else None
    rc = lib().msa_oracle_sparse_attn(C.byref(P), _ptr(q), _ptr(k), _ptr(v), _ptr(ids), n_q, n_kv,
                                      q_pos0, _ptr(r), nr, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle sparse_attn: bad arguments (%d)" % rc)
    return (o, lse) if want_lse else o


def dense_attn(P: Params, q, k, v, q_pos0: int = 0, rows=None, want_lse=False):
    """Dense GQA attention, eq. (1) (no block logic)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    n_q, n_kv = q.shape[0], k.shape[0]
    r, nr = _rows(rows, n_q)
    o = np.empty((nr, P.h_q, P.d), dtype=np.float64)
    lse = np.empty((nr, P.h_q), dtype=np.float64) if want_lse else None
    rc = lib().msa_oracle_dense_attn(C.byref(P), _ptr(q), _ptr(k), _ptr(v), n_q, n_kv, q_pos0, _ptr(r),
                                     nr, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle dense_attn: bad arguments (%d)" % rc)
    return (o, lse) if want_lse else o


def decode(P: Params, q, q_idx, k_cache, v_cache, k_idx_cache, cu_kv, seqs=None, dense=False):
    """One decode step per listed sequence: (ids[n_seq,h_kv,topk], o[n_seq,h_q,d])."""
    q, q_idx = _u16(q), _u16(q_idx)
    k_cache, v_cache, k_idx_cache = _u16(k_cache), _u16(v_cache), _u16(k_idx_cache)
    cu = np.ascontiguousarray(cu_kv, dtype=np.int64)
    batch = q.shape[0]
    s, ns = _rows(seqs, batch)
    ids = np.full((ns, P.h_kv, P.topk), -1, dtype=np.int32)
    o = np.empty((ns, P.h_q, P.d), dtype=np.float64)
    rc = lib().msa_oracle_decode(C.byref(P), _ptr(q), _ptr(q_idx), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(k_idx_cache), _ptr(cu), batch, _ptr(s), ns, int(dense), _ptr(ids),
                                 _ptr(o))
    if rc:
        raise ValueError("oracle decode: bad arguments (%d)" % rc)
    return ids, o


# ---------------------------------------------------------------------------
# Packed batches (cu_seqlens): each sequence is an independent problem, so the
# oracle of the batch is the single-sequence oracle on each sequence's rows.
# ---------------------------------------------------------------------------
def _seq_rows(cu, rows):
    """Per sequence: (s, lo, hi, local row indices or None for all rows, positions in `rows`)."""
    cu = np.asarray(cu, dtype=np.int64)
    out = []
    if rows is None:
        for s in range(len(cu) - 1):
            out.append((s, int(cu[s]), int(cu[s + 1]), None, None))
        return out
    rows = np.asarray(rows, dtype=np.int64)
    seq = np.searchsorted(cu, rows, side="right") - 1
    for s in np.unique(seq):
        sel = np.nonzero(seq == s)[0]
        out.append((int(s), int(cu[s]), int(cu[s + 1]), rows[sel] - cu[s], sel))
    return out


def index_topk_varlen(P: Params, q_idx, k_idx, cu_seqlens, topk_per_seq=None, rows=None) -> np.ndarray:
    """Block ids of a packed batch [rows or total, h_kv, topk]: each sequence
    selects with its own k (topk_per_seq, clamped to [1, topk]) and pads to
    topk with -1; ids are local to the sequence."""
    n = q_idx.shape[0] if rows is None else len(rows)
    out = np.full((n, P.h_kv, P.topk), -1, dtype=np.int32)
    for s, lo, hi, loc, pos in _seq_rows(cu_seqlens, rows):
        if hi <= lo:
            continue
        k = P.topk if topk_per_seq is None else int(min(max(int(topk_per_seq[s]), 1), P.topk))
        Ps = Params(*[getattr(P, f[0]) for f in P._fields_])
        Ps.topk = k
        ids = index_topk(Ps, q_idx[lo:hi], k_idx[lo:hi], 0, rows=loc)
        if pos is None:
            out[lo:hi, :, :k] = ids
        else:
            out[pos, :, :k] = ids
    return out


def sparse_attn_varlen(P: Params, q, k, v, ids, cu_seqlens, rows=None) -> np.ndarray:
    """Main branch of a packed batch over the given ids (one list per listed row)."""
    n = q.shape[0] if rows is None else len(rows)
    out = np.zeros((n, P.h_q, P.d), dtype=np.float64)
    for s, lo, hi, loc, pos in _seq_rows(cu_seqlens, rows):
        if hi <= lo:
            continue
        if pos is None:
            out[lo:hi] = sparse_attn(P, q[lo:hi], k[lo:hi], v[lo:hi], ids[lo:hi], 0)
        else:
            out[pos] = sparse_attn(P, q[lo:hi], k[lo:hi], v[lo:hi], ids[pos], 0, rows=loc)
    return out


# ---------------------------------------------------------------------------
# Index projections (titansim.online section 4.2: an index-query projection
# per GQA group, one index-key projection shared by all groups).
# ---------------------------------------------------------------------------
def _widen(bits) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def index_project(x, w_idx, h_kv: int, d_idx: int):
    """Q_idx[i, r, :] = x[i] . W_q^idx(r) and K_idx[i, 0, :] = x[i] . W_k^idx in float64, with the
    stacked weight w_idx [(h_kv + 1) d_idx, d_model] (rows r*d_idx..: W_q^idx(r); last d_idx rows: W_k^idx)."""
    xf, wf = _widen(x), _widen(w_idx)
    assert wf.shape == ((h_kv + 1) * d_idx, xf.shape[1]), wf.shape
    y = xf @ wf.T
    n = xf.shape[0]
    return y[:, :h_kv * d_idx].reshape(n, h_kv, d_idx), y[:, h_kv * d_idx:].reshape(n, 1, d_idx)


# ---------------------------------------------------------------------------
# MXFP8 (OCP Microscaling formats v1.0, E4M3 elements, E8M0 block scales):
# the format of the quantised KV cache (the zhichai.net summary: "MXFP8 KV
# cache").  Blocks of 32 consecutive elements along the last dimension share
# one scale 2^e.
# ---------------------------------------------------------------------------
MX_BLOCK = 32
E4M3_MAX = 448.0          # 1.75 * 2^8, the largest E4M3 normal
E4M3_EMAX = 8             # its exponent


def _e4m3_round(s: np.ndarray) -> np.ndarray:
    """Round float64 values to the E4M3 grid, nearest even, saturating at +-448."""
    a = np.abs(s)
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    quantum = np.where(a >= 2.0 ** -6, 2.0 ** (ex - 3), 2.0 ** -9)
    r = np.round(a / quantum) * quantum          # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, s)


def _e4m3_encode(r: np.ndarray) -> np.ndarray:
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << 7
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    normal = a >= 2.0 ** -6
    mant_n = np.where(normal, a / 2.0 ** ex * 8 - 8, 0).astype(np.int64)
    code_n = ((ex + 7) << 3) | mant_n
    code_s = (a / 2.0 ** -9).astype(np.int64)
    return sign | np.where(normal, code_n, code_s).astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3 byte -> float64 (no NaN codes are ever produced by the quantiser)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.where(b & 0x80, -mag, mag)


def quantize_mxfp8(x_bits):
    """bf16 bits [..., C] (C % 32 == 0) -> (E4M3 bytes [..., C], E8M0 bytes [..., C / 32]).

    Per block of 32: e = floor(log2(max |x|)) - 8, clamped to [-127, 127]
    (a block of zeros takes e = -127); elements are x / 2^e rounded to the
    E4M3 grid (nearest even, saturating at +-448); the scale byte is e + 127.
    """
    x = _widen(x_bits)
    sh = x.shape
    assert sh[-1] % MX_BLOCK == 0, sh
    xb = x.reshape(sh[:-1] + (sh[-1] // MX_BLOCK, MX_BLOCK))
    amax = np.abs(xb).max(axis=-1)
    _, ex = np.frexp(amax)                        # amax = m 2^ex, m in [0.5, 1)
    e = np.where(amax > 0, ex - 1 - E4M3_EMAX, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    scaled = xb / np.ldexp(1.0, e)[..., None]
    q = _e4m3_encode(_e4m3_round(scaled)).reshape(sh)
    return q, (e + 127).astype(np.uint8)


def dequantize_mxfp8(q, scales) -> np.ndarray:
    """E4M3 bytes [..., C] and E8M0 bytes [..., C / 32] -> float64 values."""
    v = e4m3_decode(q)
    sh = v.shape
    vb = v.reshape(sh[:-1] + (sh[-1] // MX_BLOCK, MX_BLOCK))
    sc = np.ldexp(1.0, np.asarray(scales, dtype=np.int64) - 127)
    return (vb * sc[..., None]).reshape(sh)
