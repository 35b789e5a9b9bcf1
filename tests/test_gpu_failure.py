"""Failure handling on the GPU, without faulting or hanging it: a kernel
whose wait can never be satisfied must give up at its deadline, report
MSA_ERR_TIMEOUT through the workspace status word, and leave the context
usable for the next call."""
import numpy as np
import pytest
import torch

import long_context_index_b200 as msa
import oracle
from synth import WORKLOADS, make_prefill
from tests.gpu_util import dev, params_pair

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = msa.lib().msa_test_never_ready_wait(ws.data_ptr(), 256, 20_000_000, stream)   # 20 ms deadline
    assert rc == 0
    assert msa.device_status(ws) == -6   # MSA_ERR_TIMEOUT
    # The context still works: a normal call succeeds and matches the oracle.
    w = WORKLOADS["tiny_prefill_1k"]
    t = make_prefill(w)
    p, po = params_pair(w.h_q, w.h_kv, w.d, w.d_idx, w.block_k, w.topk)
    ids = msa.index_topk(p, dev(t["q_idx"]), dev(t["k_idx"]))
    torch.cuda.synchronize()
    rows = np.arange(0, w.n_q, 5, dtype=np.int32)
    assert np.array_equal(ids.cpu().numpy()[rows], oracle.index_topk(po, t["q_idx"], t["k_idx"], rows=rows))
    # (The index call checked its own workspace's status word: OK.)  A second
    # expiry on the same workspace is reported again.
    rc = msa.lib().msa_test_never_ready_wait(ws.data_ptr(), 256, 1_000_000, stream)
    assert rc == 0 and msa.device_status(ws) == -6


def test_hook_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    L = msa.lib()
    assert L.msa_test_never_ready_wait(ws.data_ptr(), 100, 1000, None) == -1
    assert L.msa_test_never_ready_wait(ws.data_ptr(), 256, 0, None) == -1
    assert L.msa_test_never_ready_wait(ws.data_ptr(), 256, 3_000_000_000, None) == -1
