"""Seeded synthetic inputs for the MiniMax Sparse Attention (MSA) hot path.

This module only draws numbers. It holds none of the method's arithmetic
(no scores, no pooling, no selection, no softmax), so the CPU oracle and the
CUDA path can both consume its output without sharing any code with each
other.

Workloads follow the problem as the MSA pages state it (titansim.online
summary, section 3.1 "109B MoE model configuration": 64 query heads, 4 KV
heads, head dim 128, block size B_k = 128, k = 16; m.163.com post, "Step 1
Index Attention": Q_idx in R^{n x h x d}, K_idx in R^{n x 1 x d}):

* Q, K, V are bf16 draws of N(0, 1).
* Q_idx and K_idx are integers drawn uniformly from {-3, ..., 3}, stored as
  bf16 (exact).  Integer index inputs make every index score an exact
  integer in fp32, so block ids are reproducible bit for bit.
* Needles: per GQA group, 8 index keys are overwritten with 4x the index
  query of a later query, at a position in an earlier (non-local) block.
  This mimics the multi-needle retrieval workloads that the m.163.com post
  runs ("实际测试结果"), which are not available here; the synthetic needles
  stand in for them.

All arrays are numpy ``uint16`` holding raw bf16 bit patterns (row-major,
last dimension innermost).  Random streams are numpy PCG64 generators keyed by
(seed, tensor id, chunk index) with a fixed chunk size, so the bytes do not
depend on the number of threads used to draw them.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Dict, List, Optional

import numpy as np

# Elements per independently seeded chunk.  Fixed: the bytes depend on it.
_CHUNK = 1 << 22

# Stream ids of the tensors (part of each chunk's seed key).
_T_Q, _T_K, _T_V, _T_QIDX, _T_KIDX, _T_NEEDLE, _T_LENS = range(7)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload of the MSA hot path."""
    name: str
    kind: str            # "prefill" or "decode"
    h_q: int
    h_kv: int
    d: int
    d_idx: int
    block_k: int
    topk: int
    seed: int
    n_q: int = 0         # prefill: query rows
    n_kv: int = 0        # prefill: key rows (n_q for a full prefill)
    batch: int = 0       # decode: sequences
    kv_min: int = 0      # decode: KV length range, inclusive
    kv_max: int = 0
    needles: int = 0     # planted needle keys per GQA group (per sequence in decode)

    @property
    def q_pos0(self) -> int:
        """Absolute position of query row 0 (chunked prefill: the last n_q rows)."""
        return self.n_kv - self.n_q


# The five workloads of the hot path, by what they are.
WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny_prefill_1k", "prefill", h_q=8, h_kv=2, d=64, d_idx=32, block_k=64,
                 topk=4, seed=0, n_q=1024, n_kv=1024, needles=0),
        Workload("prefill_32k", "prefill", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128,
                 topk=16, seed=1, n_q=32768, n_kv=32768, needles=8),
        Workload("prefill_128k", "prefill", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128,
                 topk=16, seed=2, n_q=131072, n_kv=131072, needles=8),
        Workload("decode_b64_64k_128k", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128,
                 topk=16, seed=3, batch=64, kv_min=65536, kv_max=131072, needles=8),
        Workload("chunked_prefill_1m", "prefill", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128,
                 topk=16, seed=4, n_q=8192, n_kv=1 << 20, needles=8),
        Workload("decode_b8_1m", "decode", h_q=64, h_kv=4, d=128, d_idx=64, block_k=128,
                 topk=16, seed=4, batch=8, kv_min=1 << 20, kv_max=1 << 20, needles=8),
    ]
}


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _rng(seed: int, tensor: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, chunk])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# bf16 bit patterns of the integers -3..3 (exact).
_INT_BF16 = f32_to_bf16_bits(np.arange(-3, 4, dtype=np.float32))


def _fill(shape, seed: int, tensor: int, kind: str) -> np.ndarray:
    """Draw a bf16 tensor chunk by chunk (chunks in parallel threads)."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16)
    nchunks = (total + _CHUNK - 1) // _CHUNK

    def work(c: int) -> None:
        lo = c * _CHUNK
        hi = min(total, lo + _CHUNK)
        g = _rng(seed, tensor, c)
        if kind == "normal":
            out[lo:hi] = f32_to_bf16_bits(g.standard_normal(hi - lo, dtype=np.float32))
        else:  # integers uniform in {-3..3}
            out[lo:hi] = _INT_BF16[g.integers(0, 7, size=hi - lo, dtype=np.int8)]

    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with _cf.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def _bf16_times4(bits: np.ndarray) -> np.ndarray:
    """4 * x for bf16 x in {-3..3}: exact, done in float32 and rounded back."""
    return f32_to_bf16_bits(bf16_bits_to_f32(bits) * np.float32(4.0))


def make_prefill(w: Workload, n_q: Optional[int] = None, n_kv: Optional[int] = None) -> dict:
    """Inputs of one (possibly chunked) causal prefill.

    Returns q [n_q,h_q,d], k, v [n_kv,h_kv,d], q_idx [n_q,h_kv,d_idx],
    k_idx [n_kv,1,d_idx] (uint16 bf16 bits), q_pos0, and the list of planted
    needles as (group, query_row, key_position) tuples.  ``n_q``/``n_kv``
    override the workload's sizes (the draw order and seeds are unchanged).
    """
    n_q = w.n_q if n_q is None else n_q
    n_kv = w.n_kv if n_kv is None else n_kv
    q_pos0 = n_kv - n_q
    s = w.seed
    out = {
        "q": _fill((n_q, w.h_q, w.d), s, _T_Q, "normal"),
        "k": _fill((n_kv, w.h_kv, w.d), s, _T_K, "normal"),
        "v": _fill((n_kv, w.h_kv, w.d), s, _T_V, "normal"),
        "q_idx": _fill((n_q, w.h_kv, w.d_idx), s, _T_QIDX, "int"),
        "k_idx": _fill((n_kv, 1, w.d_idx), s, _T_KIDX, "int"),
        "q_pos0": q_pos0,
    }
    out["needles"] = _plant_prefill(w, out, n_q, n_kv, q_pos0)
    return out


def _plant_prefill(w: Workload, t: dict, n_q: int, n_kv: int, q_pos0: int) -> List[tuple]:
    """Plant ``w.needles`` needle keys per group.

    For each group r: draw a query position p_q (absolute) uniformly from the
    query range restricted to p_q >= 2*B_k, then a key position p_k uniformly
    from [0, floor(p_q/B_k)*B_k - 1] (a block before the query's own block),
    and set K_idx[p_k] = 4 * Q_idx[p_q, r].  Later needles overwrite earlier
    ones at the same key position.
    """
    needles: List[tuple] = []
    if w.needles <= 0:
        return needles
    g = _rng(w.seed, _T_NEEDLE, 0)
    lo = max(q_pos0, 2 * w.block_k)
    if lo >= q_pos0 + n_q:
        return needles
    for r in range(w.h_kv):
        for _ in range(w.needles):
            pq = int(g.integers(lo, q_pos0 + n_q))
            hi = (pq // w.block_k) * w.block_k
            pk = int(g.integers(0, hi))
            t["k_idx"][pk, 0, :] = _bf16_times4(t["q_idx"][pq - q_pos0, r, :])
            needles.append((r, pq - q_pos0, pk))
    return needles


def make_decode(w: Workload, batch: Optional[int] = None, kv_min: Optional[int] = None,
                kv_max: Optional[int] = None) -> dict:
    """Inputs of one batched decode step with contiguous per-sequence caches.

    Returns q [B,h_q,d], q_idx [B,h_kv,d_idx], k_cache, v_cache [sum L,h_kv,d],
    k_idx_cache [sum L,1,d_idx] (uint16 bf16 bits), lens [B] and cu_kv [B+1]
    (int64), and the needles as (sequence, group, key_position_in_sequence).
    The decode query of sequence b sits at position lens[b]-1 and the caches
    include that position.
    """
    batch = w.batch if batch is None else batch
    kv_min = w.kv_min if kv_min is None else kv_min
    kv_max = w.kv_max if kv_max is None else kv_max
    s = w.seed
    gl = _rng(s, _T_LENS, 0)
    lens = gl.integers(kv_min, kv_max + 1, size=batch).astype(np.int64)
    cu = np.zeros(batch + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    total = int(cu[-1])
    out = {
        "q": _fill((batch, w.h_q, w.d), s, _T_Q, "normal"),
        "k_cache": _fill((total, w.h_kv, w.d), s, _T_K, "normal"),
        "v_cache": _fill((total, w.h_kv, w.d), s, _T_V, "normal"),
        "q_idx": _fill((batch, w.h_kv, w.d_idx), s, _T_QIDX, "int"),
        "k_idx_cache": _fill((total, 1, w.d_idx), s, _T_KIDX, "int"),
        "lens": lens,
        "cu_kv": cu,
    }
    needles: List[tuple] = []
    if w.needles > 0:
        g = _rng(s, _T_NEEDLE, 0)
        for b in range(batch):
            p = int(lens[b]) - 1
            hi = (p // w.block_k) * w.block_k
            if hi <= 0:
                continue
            for r in range(w.h_kv):
                for _ in range(w.needles):
                    pk = int(g.integers(0, hi))
                    out["k_idx_cache"][int(cu[b]) + pk, 0, :] = _bf16_times4(out["q_idx"][b, r, :])
                    needles.append((b, r, pk))
    out["needles"] = needles
    return out


def make_varlen_prefill(w: Workload, lens: Optional[List[int]] = None) -> dict:
    """A packed batch of independent causal prefills (cu_seqlens layout).

    ``w.batch`` sequences with lengths drawn uniformly from
    [w.kv_min, w.kv_max] (or the given ``lens``); sequence s is drawn like a
    full prefill of its own length with seed (w.seed, s) -- values, index
    integers and needles -- and the sequences are stored back to back.
    Returns q, k, v, q_idx, k_idx (packed, uint16 bf16 bits), lens,
    cu_seqlens (int32 [batch + 1]) and needles as (sequence, group,
    query_row, key_position) in sequence-local coordinates.
    """
    if lens is None:
        g = _rng(w.seed, _T_LENS, 0)
        lens = g.integers(w.kv_min, w.kv_max + 1, size=w.batch).tolist()
    parts = []
    needles = []
    for s, L in enumerate(lens):
        ws = Workload(**{**w.__dict__, "kind": "prefill", "seed": w.seed * 1000003 + s, "n_q": int(L),
                         "n_kv": int(L)})
        t = make_prefill(ws) if L > 0 else None
        if t is not None:
            needles += [(s, r, i, pk) for (r, i, pk) in t["needles"]]
        parts.append(t)
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    shapes = {"q": (w.h_q, w.d), "k": (w.h_kv, w.d), "v": (w.h_kv, w.d), "q_idx": (w.h_kv, w.d_idx),
              "k_idx": (1, w.d_idx)}
    out = {}
    for name, sh in shapes.items():
        chunks = [t[name] for t in parts if t is not None]
        out[name] = (np.concatenate(chunks, axis=0) if chunks else np.zeros((0,) + sh, dtype=np.uint16))
    out["lens"] = np.asarray(lens, dtype=np.int64)
    out["cu_seqlens"] = cu
    out["needles"] = needles
    return out


def make_index_projection(seed: int, n: int, d_model: int, h_kv: int, d_idx: int, integer: bool = False) -> dict:
    """Hidden states x [n, d_model] and the stacked index weights
    w_idx [(h_kv + 1) d_idx, d_model] (uint16 bf16 bits).

    Default: x ~ N(0, 1) and w ~ N(0, 1 / d_model) rounded to bf16.  With
    ``integer``: every row of x has 8 entries of +-1 at random columns (zeros
    elsewhere) and w is uniform on {-3..3}, so every projected value is an
    integer of magnitude <= 24 -- exact in fp32 and bf16, which makes the
    index ids downstream of the projection reproducible bit for bit.
    """
    n_out = (h_kv + 1) * d_idx
    g = _rng(seed, _T_QIDX, 7)
    if integer:
        x = np.zeros((n, d_model), dtype=np.float32)
        cols = np.argsort(g.random((n, d_model)), axis=1)[:, :8] if d_model <= 4096 else \
            np.stack([g.choice(d_model, 8, replace=False) for _ in range(n)])
        signs = g.choice(np.array([-1.0, 1.0], dtype=np.float32), size=(n, 8))
        np.put_along_axis(x, cols, signs, axis=1)
        w = g.integers(-3, 4, size=(n_out, d_model)).astype(np.float32)
    else:
        x = g.standard_normal((n, d_model), dtype=np.float32)
        w = g.standard_normal((n_out, d_model), dtype=np.float32) / np.float32(np.sqrt(d_model))
    return {"x": f32_to_bf16_bits(x), "w_idx": f32_to_bf16_bits(w)}
