"""Useful-work model of the MSA hot path (host logic, used by the bench).

* eq12_flops: the pages' complexity formula (titansim.online summary,
  section 5.2, eq. (12)): F_GQA(N) = 2 H_q d_h N^2 and
  F_MSA(N) = H_kv d_idx N^2 + 4 H_q d_h N k B_k.
* index_flops / main_flops: exact useful FLOPs of one prefill, counting only
  causally visible (query, key) pairs: 2 H_kv d_idx per visible pair for the
  index score, 4 H_q/H_kv d per (query, head, selected visible key) for the
  main branch (QK^T and PV, one multiply-add = 2 FLOPs each).
* decode_bytes: the bytes one decode step must read/write: the index-key cache
  of each sequence once (for all groups), the selected visible K/V rows, Q,
  Q_idx, O and the ids.
"""
from __future__ import annotations

import numpy as np


def eq12_flops(n: int, h_q: int, d_h: int, h_kv: int, d_idx: int, k: int, block_k: int):
    """(F_GQA, F_MSA) of eq. (12)."""
    f_gqa = 2.0 * h_q * d_h * n * n
    f_msa = 1.0 * h_kv * d_idx * n * n + 4.0 * h_q * d_h * n * k * block_k
    return f_gqa, f_msa


def visible_pairs(n_q: int, n_kv: int, q_pos0: int, causal: bool = True) -> int:
    """Number of (query, key) pairs with the key visible from the query."""
    if not causal:
        return n_q * n_kv
    p = np.arange(q_pos0, q_pos0 + n_q, dtype=np.int64)
    return int(np.minimum(p + 1, n_kv).sum())


def index_flops(n_q: int, n_kv: int, q_pos0: int, h_kv: int, d_idx: int, causal: bool = True) -> float:
    return 2.0 * h_kv * d_idx * visible_pairs(n_q, n_kv, q_pos0, causal)


def selected_keys(ids: np.ndarray, block_k: int, n_kv: int, q_pos0: int, causal: bool = True) -> int:
    """Sum over (query, group) of the visible keys in the selected blocks.

    ids: int32 [n_q, h_kv, topk] (-1 padding)."""
    n_q = ids.shape[0]
    p = (q_pos0 + np.arange(n_q, dtype=np.int64))[:, None, None]
    b = ids.astype(np.int64)
    lo = b * block_k
    hi = np.minimum(lo + block_k, n_kv)
    if causal:
        hi = np.minimum(hi, p + 1)
    cnt = np.where(b >= 0, np.maximum(hi - lo, 0), 0)
    return int(cnt.sum())


def main_flops(sel_keys: int, h_q: int, h_kv: int, d: int) -> float:
    return 4.0 * (h_q // h_kv) * d * sel_keys


def dense_main_flops(n_q: int, n_kv: int, q_pos0: int, h_q: int, d: int, causal: bool = True) -> float:
    return 4.0 * h_q * d * visible_pairs(n_q, n_kv, q_pos0, causal)


def decode_bytes(lens: np.ndarray, ids: np.ndarray, h_q: int, h_kv: int, d: int, d_idx: int, block_k: int,
                 dense: bool = False, mxfp8: bool = False) -> int:
    """Bytes one decode step must move (bf16 tensors, int32 ids).  With
    ``mxfp8`` the caches hold one E4M3 byte per element plus one E8M0 byte per
    32 elements."""
    lens = np.asarray(lens, dtype=np.int64)
    B = lens.size
    per = (1.0 + 1.0 / 32) if mxfp8 else 2.0                   # cache bytes per element
    total = 0
    if not dense:
        total += int(lens.sum() * d_idx * per)                  # index-key cache, once for all groups
        total += B * h_kv * d_idx * 2 + B * h_kv * ids.shape[2] * 4
        for b in range(B):
            sel = selected_keys(ids[b:b + 1], block_k, int(lens[b]), int(lens[b]) - 1)
            total += int(sel * d * per * 2)                      # K and V rows of the selected blocks
    else:
        total += int(lens.sum()) * h_kv * d * 2 * 2
    total += B * h_q * d * 2 * 2                                 # Q in, O out
    return total
