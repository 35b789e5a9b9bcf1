"""Helpers shared by the GPU parity tests (data movement only)."""
import numpy as np
import torch

import long_context_index_b200 as msa
import oracle


def dev(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits / int arrays -> CUDA tensor (bf16 for uint16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def params_pair(h_q, h_kv, d, d_idx, block_k, topk, causal=1, force_local=1, scale=0.0, pool=0):
    """The same problem as library parameters and as oracle parameters."""
    return (msa.Params.make(h_q, h_kv, d, d_idx, block_k, topk, causal, force_local, scale, pool),
            oracle.params(h_q, h_kv, d, d_idx, block_k, topk, causal, force_local, scale, pool=pool))


def assert_close(got: np.ndarray, ref: np.ndarray, atol=1e-2, rtol=1e-2, what=""):
    """Elementwise |got - ref| <= atol + rtol * |ref| (the parity tolerance)."""
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%s: %d / %d elements out of tolerance; max err %.4g; first %s got %s ref %s" % (
            what, int(bad.sum()), bad.size, float(err.max()), idx.tolist(),
            [float(got[tuple(i)]) for i in idx], [float(ref[tuple(i)]) for i in idx]))
