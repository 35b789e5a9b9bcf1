"""Benchmark of the MSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over synthetic inputs resident in
HBM: the index branch and the main branch of a 128K-token causal prefill
(64 query heads, 4 KV heads, d = 128, d_idx = 64, B_k = 128, k = 16), then one
decode step of 64 sequences with KV lengths in [64K, 128K] (the same model
shape).  Tokens per step = 131072 prefill + 64 decode tokens.

Prints one JSON line (rank 0).  ``--gpus N`` runs N ranks, one per GPU: under
torchrun (WORLD_SIZE set) it must equal the world size; run directly with
N > 1 it relaunches itself under torchrun with N processes.  Each rank runs
its own independent problem of the same shape (weak scaling, no data-path
collective); the time is the max over ranks.  ``--impl reference`` times the
fp64 CPU oracle on bounded samples of the same workload on the host cores
instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, Workload, make_decode, make_prefill  # noqa: E402

METRIC = "MSA prefill & decode tokens/s at 128K ctx; % of B200 tensor / HBM roofline"
PREFILL = WORKLOADS["prefill_128k"]
DECODE = WORKLOADS["decode_b64_64k_128k"]


def cases(name):
    """The bench workload, a smaller instance of the same kernels for ncu
    captures ("small": 32K prefill and 8 decode sequences), the long-context
    pair ("long": the last 8192 queries of a 2^20-token chunked prefill and a
    batch of 8 sequences decoding at 2^20), a profiling pair small enough for
    multi-pass ncu captures ("prof": the last 4096 queries of a 65536-token
    context, about 1 GB of partials, and 8 sequences of 16K-32K tokens;
    "prof_decode": the same prefill and 64 sequences of 16K-32K tokens, whose
    200 MB of index keys exceed the L2 in 3.3 GB of caches), or a
    tiny pair that runs in seconds ("tiny": the 1K prefill and 4 short decode
    sequences)."""
    if name == "prof_decode":
        return (cases("prof")[0],
                Workload(**{**DECODE.__dict__, "kv_min": 16384, "kv_max": 32768, "name": "decode_b64_16k_32k"}))
    if name == "prof":
        return (Workload(**{**WORKLOADS["prefill_32k"].__dict__, "n_q": 4096, "n_kv": 65536,
                            "name": "chunked_prefill_64k_4k"}),
                Workload(**{**DECODE.__dict__, "batch": 8, "kv_min": 16384, "kv_max": 32768, "name": "decode_b8_32k"}))
    if name == "tiny":
        return WORKLOADS["tiny_prefill_1k"], Workload(**{**DECODE.__dict__, "batch": 4, "kv_min": 3000,
                                                           "kv_max": 9000, "name": "decode_b4_short"})
    if name == "small":
        return WORKLOADS["prefill_32k"], Workload(**{**DECODE.__dict__, "batch": 8, "name": "decode_b8"})
    if name == "long":
        return WORKLOADS["chunked_prefill_1m"], WORKLOADS["decode_b8_1m"]
    return PREFILL, DECODE


PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024

# DRAM bytes per call of the dominant unit at the bench workload, from ncu's
# dram__bytes_read.sum + dram__bytes_write.sum of its kernels on the 4096-query
# chunked prefill at 64K ("prof" case: 2.5436 GB), scaled by the query rows
# (x32; the traffic is the partial rows, one per query, head and selected
# block), on the kernel source with the given digest (a stale digest reports
# null).
TRAFFIC = {"attn_prefill": (2.5436e9 * 32, "61f508beef40", "attn_sparse.cu")}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def src_digest(name: str) -> str:
    path = os.path.join(ROOT, "long_context_index_b200", "csrc", name)
    return hashlib.sha1(open(path, "rb").read()).hexdigest()[:12]


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_smi_id(torch, dev: int) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def to_dev(torch, a, pin=False):
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    if pin:
        t = t.pin_memory()
    return t


def bf16(torch, t):
    return t.view(torch.bfloat16) if t.dtype == torch.int16 else t


def rank_workloads(case: str, rank: int):
    """The (prefill, decode) problems rank `rank` runs: the same shapes on
    every rank, each rank its own seed, so N ranks process N independent
    problems (weak scaling; no data crosses ranks)."""
    pre, dec = cases(case)
    off = 1000 * rank
    return (Workload(**{**pre.__dict__, "seed": pre.seed + off}),
            Workload(**{**dec.__dict__, "seed": dec.seed + off}))


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank time over all ranks (every rank calls this)."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args, rank, world, torch, dist):
    import long_context_index_b200 as msa
    from long_context_index_b200 import flops

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    wp, wd = rank_workloads(args.case, rank)
    tp = make_prefill(wp)
    td = make_decode(wd)
    pp = msa.Params.make(wp.h_q, wp.h_kv, wp.d, wp.d_idx, wp.block_k, wp.topk)
    pd = msa.Params.make(wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k, wd.topk)
    n = wp.n_q                 # prefill query rows
    n_kv = tp["k"].shape[0]    # prefill keys (n_kv > n: a chunk at the end of a longer context)
    q_pos0 = int(tp["q_pos0"])
    B = wd.batch
    max_kv = int(td["lens"].max())

    # Host (pinned) and device copies of every input.
    host = {k: to_dev(torch, tp[k], pin=True) for k in ("q", "k", "v", "q_idx", "k_idx")}
    hostd = {k: to_dev(torch, td[k], pin=True) for k in ("q", "q_idx", "cu_kv")}
    d_in = {k: bf16(torch, v.to(dev)) for k, v in host.items()}
    dd = {k: bf16(torch, to_dev(torch, td[k]).to(dev)) for k in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache",
                                                                  "cu_kv")}
    ids = torch.empty((n, wp.h_kv, wp.topk), dtype=torch.int32, device=dev)
    o = torch.empty((n, wp.h_q, wp.d), dtype=torch.bfloat16, device=dev)
    dids = torch.empty((B, wd.h_kv, wd.topk), dtype=torch.int32, device=dev)
    do = torch.empty((B, wd.h_q, wd.d), dtype=torch.bfloat16, device=dev)
    ws_i = torch.empty(msa.workspace_size(msa.OP_INDEX_TOPK, pp, n, n_kv), dtype=torch.uint8, device=dev)
    ws_p = torch.empty(max(256, msa.workspace_size(msa.OP_PREFILL, pp, n, n_kv)), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(msa.workspace_size(msa.OP_DECODE, pd, batch=B, max_kv=max_kv), dtype=torch.uint8,
                       device=dev)

    decode_form = msa.get_option(msa.OPT_DECODE_FUSED)   # the library's default form

    def step():
        msa.index_topk(pp, d_in["q_idx"], d_in["k_idx"], q_pos0, block_ids=ids, ws=ws_i)
        ev[1].record(stream)
        msa.sparse_attn_prefill(pp, d_in["q"], d_in["k"], d_in["v"], ids, q_pos0, out=o, ws=ws_p)
        ev[2].record(stream)
        msa.sparse_attn_decode(pd, dd["q"], dd["q_idx"], dd["k_cache"], dd["v_cache"], dd["k_idx_cache"],
                               dd["cu_kv"], max_kv, block_ids=dids, out=do, ws=ws_d)

    E = torch.cuda.Event
    ev = [E(enable_timing=True) for _ in range(4)]
    for _ in range(args.warmup):
        ev[0].record(stream)
        step()
        ev[3].record(stream)
    torch.cuda.synchronize()
    for wsx in (ws_i, ws_p, ws_d):
        rc = msa.device_status(wsx)
        if rc:
            raise RuntimeError("device status %d after warm-up" % rc)

    # ---- timed region: K steps, per-call CUDA events on the launching stream
    clk = ClockSampler(gpu_smi_id(torch, torch.cuda.current_device())) if rank == 0 else None
    time.sleep(0.3 if clk else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[E(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for s in range(args.steps):
        ev = evs[s]
        ev[0].record(stream)
        step()
        ev[3].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop() if clk else None
    t_total = evs[0][0].elapsed_time(evs[-1][3])
    t_idx = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_attn = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    t_dec = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    for wsx in (ws_i, ws_p, ws_d):
        rc = msa.device_status(wsx)
        if rc:
            raise RuntimeError("device status %d after the timed steps" % rc)
    if world > 1:
        t_total = max_over_ranks(t_total, dist, dev)
    ms_step = t_total / args.steps
    tokens_step = n + B
    value = tokens_step * world / (ms_step / 1e3)

    # ---- useful work of this step (from the ids of the last step)
    ids_h = ids.cpu().numpy()
    dids_h = dids.cpu().numpy()
    f_idx = flops.index_flops(n, n_kv, q_pos0, wp.h_kv, wp.d_idx)
    sel = flops.selected_keys(ids_h, wp.block_k, n_kv, q_pos0)
    f_main = flops.main_flops(sel, wp.h_q, wp.h_kv, wp.d)
    b_dec = flops.decode_bytes(td["lens"], dids_h, wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k)

    # ---- dense run (every causal block): the same call with no block ids
    # (prefill) / dense = 1 (decode), warmed up and timed over as many steps
    # as the sparse run, outside the sparse timed region
    t_dense_p = t_dense_d = None
    if not args.no_dense:
        def dense_step(ev_):
            ev_[0].record(stream)
            msa.sparse_attn_prefill(pp, d_in["q"], d_in["k"], d_in["v"], None, q_pos0, out=o, ws=ws_p)
            ev_[1].record(stream)
            msa.sparse_attn_decode(pd, dd["q"], None, dd["k_cache"], dd["v_cache"], None, dd["cu_kv"], max_kv,
                                   dense=True, out=do, ws=ws_d)
            ev_[2].record(stream)

        for _ in range(args.warmup):
            dense_step([E(enable_timing=True) for _ in range(3)])
        dev_ = [[E(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for s_ in range(args.steps):
            dense_step(dev_[s_])
        torch.cuda.synchronize()
        t_dense_p = statistics.median(e[0].elapsed_time(e[1]) for e in dev_)
        t_dense_d = statistics.median(e[1].elapsed_time(e[2]) for e in dev_)
        for wsx in (ws_p, ws_d):
            rc = msa.device_status(wsx)
            if rc:
                raise RuntimeError("device status %d after the dense runs" % rc)
    def median_ms(fn):
        """fn warmed up, then the median of as many timed calls as the step."""
        for _ in range(args.warmup):
            fn()
        evp = [(E(enable_timing=True), E(enable_timing=True)) for _ in range(args.steps)]
        for a_, b_ in evp:
            a_.record(stream)
            fn()
            b_.record(stream)
        torch.cuda.synchronize()
        return statistics.median(a_.elapsed_time(b_) for a_, b_ in evp)

    def fused_form(fn):
        """fn timed with the decode step in its one-launch form."""
        msa.set_option(msa.OPT_DECODE_FUSED, 1)
        try:
            return median_ms(fn)
        finally:
            msa.set_option(msa.OPT_DECODE_FUSED, decode_form)

    # ---- the decode step in its other form (one cooperative launch), for
    # the comparison that picks the library's default
    t_dec_fused = None
    if not decode_form:
        outs = [(torch.empty_like(dids), torch.empty_like(do)) for _ in range(2)]

        def dec_into(i):
            return lambda: msa.sparse_attn_decode(pd, dd["q"], dd["q_idx"], dd["k_cache"], dd["v_cache"],
                                                  dd["k_idx_cache"], dd["cu_kv"], max_kv, block_ids=outs[i][0],
                                                  out=outs[i][1], ws=ws_d)
        t_dec_fused = fused_form(dec_into(1))
        dec_into(0)()
        torch.cuda.synchronize()
        rc = msa.device_status(ws_d)
        if rc:
            raise RuntimeError("device status %d after the fused decode" % rc)
        if not (torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])):
            raise RuntimeError("the two decode forms disagree")
        del outs

    # ---- the same decode step over MXFP8 caches (quantised untimed, then
    # warmed up and timed over as many steps as the bf16 step)
    t_mx = b_mx = t_mx_fused = None
    if not args.no_mxfp8 and wd.d == 128:
        q8 = {k_: msa.quantize_mxfp8(dd[k_]) for k_ in ("k_cache", "v_cache", "k_idx_cache")}
        dids8 = torch.empty_like(dids)
        do8 = torch.empty_like(do)

        def mx_step():
            msa.sparse_attn_decode_mxfp8(pd, dd["q"], dd["q_idx"], q8["k_cache"][0], q8["k_cache"][1],
                                         q8["v_cache"][0], q8["v_cache"][1], q8["k_idx_cache"][0],
                                         q8["k_idx_cache"][1], dd["cu_kv"], max_kv, block_ids=dids8, out=do8,
                                         ws=ws_d)

        t_mx = median_ms(mx_step)
        if not decode_form:
            t_mx_fused = fused_form(mx_step)
        rc = msa.device_status(ws_d)
        if rc:
            raise RuntimeError("device status %d after the MXFP8 decode" % rc)
        b_mx = flops.decode_bytes(td["lens"], dids8.cpu().numpy(), wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k,
                                  mxfp8=True)
        del q8
    med_pre = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    med_dec = statistics.median(e[2].elapsed_time(e[3]) for e in evs)

    # ---- end to end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and its results back; the
    # copies are pipelined with the kernels: inputs and outputs are double
    # buffered, uploads run on one copy stream and downloads on another, so
    # step t + 1's upload and step t - 1's download overlap step t's kernels.
    e2e_value = None
    h2d = sum(t.numel() * t.element_size() for t in list(host.values()) + list(hostd.values()))
    d2h = 0
    if not args.no_e2e:
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        sets = []
        for _ in range(2):
            sets.append({
                "in": {k_: torch.empty_like(v_) for k_, v_ in d_in.items()},
                "ind": {k_: torch.empty_like(dd[k_]) for k_ in hostd},
                "ids": torch.empty_like(ids), "o": torch.empty_like(o),
                "dids": torch.empty_like(dids), "do": torch.empty_like(do),
                "h_o": torch.empty((n, wp.h_q, wp.d), dtype=torch.int16).pin_memory(),
                "h_ids": torch.empty((n, wp.h_kv, wp.topk), dtype=torch.int32).pin_memory(),
                "h_do": torch.empty((B, wd.h_q, wd.d), dtype=torch.int16).pin_memory(),
                "h_dids": torch.empty((B, wd.h_kv, wd.topk), dtype=torch.int32).pin_memory(),
                "uploaded": E(), "computed": E(), "downloaded": E(),
            })
        d2h = sum(sets[0][k_].numel() * sets[0][k_].element_size() for k_ in ("h_o", "h_ids", "h_do", "h_dids"))

        def run_pipeline(n_steps, first_ev=None, last_ev=None):
            if first_ev is not None:
                first_ev.record(up)
            for i in range(n_steps):
                st_ = sets[i % 2]
                with torch.cuda.stream(up):
                    up.wait_event(st_["computed"])          # step i - 2 no longer reads these inputs
                    for k_, t_ in host.items():
                        st_["in"][k_].view(torch.int16).copy_(t_, non_blocking=True)
                    for k_, t_ in hostd.items():
                        st_["ind"][k_].view(t_.dtype).copy_(t_, non_blocking=True)
                    st_["uploaded"].record(up)
                stream.wait_event(st_["uploaded"])
                stream.wait_event(st_["downloaded"])       # step i - 2's results are on the host
                x_, xd_ = st_["in"], st_["ind"]
                msa.index_topk(pp, x_["q_idx"], x_["k_idx"], q_pos0, block_ids=st_["ids"], ws=ws_i)
                msa.sparse_attn_prefill(pp, x_["q"], x_["k"], x_["v"], st_["ids"], q_pos0, out=st_["o"], ws=ws_p)
                msa.sparse_attn_decode(pd, xd_["q"], xd_["q_idx"], dd["k_cache"], dd["v_cache"], dd["k_idx_cache"],
                                       xd_["cu_kv"], max_kv, block_ids=st_["dids"], out=st_["do"], ws=ws_d)
                st_["computed"].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(st_["computed"])
                    st_["h_o"].copy_(st_["o"].view(torch.int16), non_blocking=True)
                    st_["h_ids"].copy_(st_["ids"], non_blocking=True)
                    st_["h_do"].copy_(st_["do"].view(torch.int16), non_blocking=True)
                    st_["h_dids"].copy_(st_["dids"], non_blocking=True)
                    st_["downloaded"].record(down)
            if last_ev is not None:
                stream.wait_stream(down)
                last_ev.record(stream)

        for st_ in sets:                                    # the events start out completed
            for k_ in ("uploaded", "computed", "downloaded"):
                st_[k_].record(stream)
        run_pipeline(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = E(enable_timing=True), E(enable_timing=True)
        run_pipeline(args.steps, a, b)
        torch.cuda.synchronize()
        t_e2e = a.elapsed_time(b)
        if world > 1:
            t_e2e = max_over_ranks(t_e2e, dist, dev)
        e2e_value = tokens_step * world / (t_e2e / args.steps / 1e3)
        for wsx in (ws_i, ws_p, ws_d):
            rc = msa.device_status(wsx)
            if rc:
                raise RuntimeError("device status %d after the end-to-end steps" % rc)
        del sets

    peaks, peak_src = load_peaks()
    next_rows = None if args.no_extras else measure_next_rows(
        msa, torch, args, stream, median_ms, peaks, d_in, dd, wp, wd, td, n, n_kv, q_pos0, max_kv, ids, o, dids,
        do, ws_d)
    kern = {
        "index_topk_prefill": {"ms": t_idx, "bound": "tensor", "work": f_idx, "unit": "TFLOP/s",
                               "achieved": f_idx / (t_idx / 1e3) / 1e12, "peak": peaks["bf16_tflops"]},
        "attn_prefill": {"ms": t_attn, "bound": "tensor", "work": f_main, "unit": "TFLOP/s",
                         "achieved": f_main / (t_attn / 1e3) / 1e12, "peak": peaks["bf16_tflops"]},
        "decode_step": {"ms": t_dec, "bound": "hbm", "work": b_dec, "unit": "GB/s",
                        "achieved": b_dec / (t_dec / 1e3) / 1e9, "peak": peaks["hbm_gbs"]},
    }
    for k_, v_ in kern.items():
        v_["frac"] = v_["achieved"] / v_["peak"]
    dom = max(kern, key=lambda k_: kern[k_]["ms"])
    dk = kern[dom]
    traffic = None
    if args.case == "full" and dom in TRAFFIC and TRAFFIC[dom][1] == src_digest(TRAFFIC[dom][2]):
        traffic = TRAFFIC[dom][0]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; integer index inputs with planted needles)",
        "config": {"workload": "%s + %s" % (wp.name, wd.name),
                   "seq_len": n_kv, "prefill_rows": n, "decode_batch": B,
                   "h_q": wp.h_q, "h_kv": wp.h_kv, "d": wp.d, "d_idx": wp.d_idx, "block_k": wp.block_k,
                   "topk": wp.topk, "tokens_per_step": tokens_step,
                   "l2": "inputs larger than L2 (%.1f GB prefill inputs; %.1f GB decode caches), no flush"
                         % (sum(t_.numel() * t_.element_size() for t_ in host.values()) / 1e9,
                            sum(dd[k_].numel() * dd[k_].element_size() for k_ in ("k_cache", "v_cache", "k_idx_cache")) / 1e9)},
        "prefill": {"ms": t_idx + t_attn, "tokens_per_s": n * world / ((t_idx + t_attn) / 1e3),
                    "index_ms": t_idx, "attn_ms": t_attn, "useful_tflop": (f_idx + f_main) / 1e12,
                    "tensor_frac": (f_idx + f_main) / ((t_idx + t_attn) / 1e3) / 1e12 / peaks["bf16_tflops"]},
        "decode": {"ms": t_dec, "tokens_per_s": B * world / (t_dec / 1e3), "bytes": b_dec,
                   "hbm_frac": b_dec / (t_dec / 1e3) / 1e9 / peaks["hbm_gbs"],
                   "form": "one fused launch" if decode_form else "index-scan and attention launches",
                   "fused_form_ms": t_dec_fused, "mxfp8_fused_form_ms": t_mx_fused},
        "decode_mxfp8": None if t_mx is None else {
            "ms": t_mx, "tokens_per_s": B * world / (t_mx / 1e3), "bytes": b_mx,
            "hbm_frac": b_mx / (t_mx / 1e3) / 1e9 / peaks["hbm_gbs"], "stat": "median per step",
            "note": "the same decode step over MXFP8 (E4M3 + E8M0 per 32) K, V and index-key caches"},
        "next_rows": next_rows,
        "dense": None if t_dense_p is None else {
            "prefill_ms": t_dense_p, "decode_ms": t_dense_d, "steps": args.steps, "warmup": args.warmup,
            "stat": "median per step; sparse medians %.3f ms prefill, %.4f ms decode" % (med_pre, med_dec),
            "kernels": "prefill: query-outer tcgen05 flash kernel over every causal block (a block-major pass "
                       "would write one partial per (query, block)); decode: split-KV kernel over every block",
            "prefill_sparse_speedup": t_dense_p / med_pre, "decode_sparse_speedup": t_dense_d / med_dec},
        "roofline": {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                     "unit": dk["unit"], "frac": dk["frac"], "traffic": traffic,
                     "peak_source": peak_src + (" burst" if dk["bound"] == "tensor" else "")},
        "kernels": {k_: {kk: vv for kk, vv in v_.items() if kk != "work"} for k_, v_ in kern.items()},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "prefill inputs and outputs cross PCIe every step (double-buffered, uploads and downloads "
                        "on their own streams, overlapping the kernels); decode KV caches stay resident"},
        # Per step: index top-k (1); sparse prefill: schedule count, tile
        # sums, tile scans and fill (4), block-major attention (1), partial merge
        # (1); decode: persistent index scan with the merge folded in and
        # persistent attention with the combine folded in (2), or the two
        # in one fused launch (1).
        "gpu_launches": (7 + (1 if decode_form else 2)) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.case == "full":
        line["cpu_baseline"] = cpu_baseline(tp, td, wp, wd)
    return line


def measure_next_rows(msa, torch, args, stream, median_ms, peaks, d_in, dd, wp, wd, td, n, n_kv, q_pos0, max_kv,
                      ids, o, dids, do, ws_d):
    """The entry points beyond the prefill + decode step, each timed like the
    step (warm-up, then the median of as many calls) on inputs of the bench's
    shapes, with its useful work against the measured peak:

    * index_project: Q_idx and K_idx from hidden states x [n, 8192] (the
      hidden width h_q d of the model shape) and the stacked weight
      [(h_kv + 1) d_idx, 8192]; x and the weight are seeded normals drawn on
      the device.
    * index_topk_mean_pool: the index branch of the prefill with block mean
      pooling instead of max pooling.
    * prefill_varlen: index branch + main branch of the prefill's rows cut into
      a packed batch of independent sequences (seeded lengths in
      [8192, 24576], the last one cut to fit); the rows are the prefill's own
      synthetic inputs, so only the sequence boundaries are new.
    * decode_adaptive_k: the decode step with a seeded per-sequence k in
      [4, topk]."""
    from long_context_index_b200 import flops
    dev = d_in["q"].device
    out = {}

    def entry(ms, work, bound, note):
        unit, peak = ("TFLOP/s", peaks["bf16_tflops"]) if bound == "tensor" else ("GB/s", peaks["hbm_gbs"])
        ach = work / (ms / 1e3) / (1e12 if bound == "tensor" else 1e9)
        return {"ms": ms, "bound": bound, "achieved": ach, "unit": unit, "peak": peak, "frac": ach / peak,
                "note": note}

    # index projections
    d_model = wp.h_q * wp.d
    pp = msa.Params.make(wp.h_q, wp.h_kv, wp.d, wp.d_idx, wp.block_k, wp.topk)
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)
    x = torch.randn((n, d_model), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    w = (torch.randn(((wp.h_kv + 1) * wp.d_idx, d_model), generator=gen, device=dev, dtype=torch.float32)
         / d_model ** 0.5).to(torch.bfloat16)
    qi = torch.empty((n, wp.h_kv, wp.d_idx), dtype=torch.bfloat16, device=dev)
    ki = torch.empty((n, 1, wp.d_idx), dtype=torch.bfloat16, device=dev)
    ws_j = torch.empty(max(256, msa.workspace_size(msa.OP_INDEX_PROJECT, pp, n)), dtype=torch.uint8, device=dev)
    t = median_ms(lambda: msa.index_project(pp, x, w, q_idx=qi, k_idx=ki, ws=ws_j))
    n_out = (wp.h_kv + 1) * wp.d_idx
    f = 2.0 * n * d_model * n_out
    b = (n * d_model + n_out * d_model + n * n_out) * 2
    # Whichever of the two floors is longer bounds the kernel.
    bound = "tensor" if f / (peaks["bf16_tflops"] * 1e12) >= b / (peaks["hbm_gbs"] * 1e9) else "hbm"
    out["index_project"] = entry(t, f if bound == "tensor" else b, bound,
                                 "x [%d, %d] -> Q_idx, K_idx: %.3f TFLOP, %.2f GB" % (n, d_model, f / 1e12, b / 1e9))
    out["index_project"]["hbm_frac"] = b / (t / 1e3) / 1e9 / peaks["hbm_gbs"]
    del x, w, qi, ki, ws_j

    # mean pooling
    pm = msa.Params.make(wp.h_q, wp.h_kv, wp.d, wp.d_idx, wp.block_k, wp.topk, pool=msa.POOL_MEAN)
    ws_m = torch.empty(msa.workspace_size(msa.OP_INDEX_TOPK, pm, n, n_kv), dtype=torch.uint8, device=dev)
    ids_m = torch.empty_like(ids)
    t = median_ms(lambda: msa.index_topk(pm, d_in["q_idx"], d_in["k_idx"], q_pos0, block_ids=ids_m, ws=ws_m))
    out["index_topk_mean_pool"] = entry(t, flops.index_flops(n, n_kv, q_pos0, wp.h_kv, wp.d_idx), "tensor",
                                        "the prefill's index branch, block mean instead of max")
    del ws_m, ids_m

    # packed batch of independent prefills over the prefill's rows
    if q_pos0 == 0:
        g = np.random.default_rng(5)
        lens = []
        while sum(lens) < n:
            lens.append(int(min(g.integers(8192, 24577), n - sum(lens))))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev)
        ws_vi = torch.empty(msa.workspace_size(msa.OP_INDEX_TOPK_VARLEN, pp, n, batch=len(lens)), dtype=torch.uint8,
                            device=dev)
        ws_vp = torch.empty(msa.workspace_size(msa.OP_PREFILL_VARLEN, pp, n, batch=len(lens)), dtype=torch.uint8,
                            device=dev)
        ids_v = torch.empty_like(ids)
        o_v = torch.empty_like(o)

        def varlen_step():
            msa.index_topk_varlen(pp, d_in["q_idx"], d_in["k_idx"], cu, block_ids=ids_v, ws=ws_vi)
            msa.sparse_attn_prefill_varlen(pp, d_in["q"], d_in["k"], d_in["v"], cu, ids_v, out=o_v, ws=ws_vp)
        t = median_ms(varlen_step)
        ids_h = ids_v.cpu().numpy()
        f_i = f_m = 0.0
        row = 0
        for L in lens:
            f_i += flops.index_flops(L, L, 0, wp.h_kv, wp.d_idx)
            f_m += flops.main_flops(flops.selected_keys(ids_h[row:row + L], wp.block_k, L, 0), wp.h_q, wp.h_kv,
                                    wp.d)
            row += L
        out["prefill_varlen"] = entry(t, f_i + f_m, "tensor", "%d sequences of %s tokens (%d rows)"
                                      % (len(lens), "/".join(map(str, lens)), n))
        out["prefill_varlen"]["tokens_per_s"] = n / (t / 1e3)
        del ws_vi, ws_vp, ids_v, o_v

    # adaptive k in decode
    pd = msa.Params.make(wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k, wd.topk)
    ks = np.random.default_rng(7).integers(4, wd.topk + 1, size=wd.batch).astype(np.int32)
    kt = torch.from_numpy(ks).to(dev)
    dids_a = torch.empty_like(dids)
    do_a = torch.empty_like(do)
    t = median_ms(lambda: msa.sparse_attn_decode(pd, dd["q"], dd["q_idx"], dd["k_cache"], dd["v_cache"],
                                                 dd["k_idx_cache"], dd["cu_kv"], max_kv, block_ids=dids_a, out=do_a,
                                                 ws=ws_d, topk_per_seq=kt))
    bts = flops.decode_bytes(td["lens"], dids_a.cpu().numpy(), wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k)
    out["decode_adaptive_k"] = entry(t, bts, "hbm", "per-sequence k in [4, %d], mean %.1f" % (wd.topk, ks.mean()))
    return out


# ---------------------------------------------------------------------------
# the fp64 oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(tp, td, wp, wd, rows, seqs, threads):
    import oracle
    po = oracle.params(wp.h_q, wp.h_kv, wp.d, wp.d_idx, wp.block_k, wp.topk, threads=threads)
    t0 = time.perf_counter()
    ids = oracle.index_topk(po, tp["q_idx"], tp["k_idx"], rows=rows)
    oracle.sparse_attn(po, tp["q"], tp["k"], tp["v"], ids, rows=rows)
    pd = oracle.params(wd.h_q, wd.h_kv, wd.d, wd.d_idx, wd.block_k, wd.topk, threads=threads)
    oracle.decode(pd, td["q"], td["q_idx"], td["k_cache"], td["v_cache"], td["k_idx_cache"], td["cu_kv"], seqs=seqs)
    return time.perf_counter() - t0


def cpu_baseline(tp, td, wp, wd, rows_n=2048, seqs_n=32):
    threads = os.cpu_count() or 1
    rows = np.linspace(0, wp.n_q - 1, rows_n).astype(np.int32)
    seqs = np.arange(seqs_n, dtype=np.int32)
    t = oracle_sample(tp, td, wp, wd, rows, seqs, threads)
    return {"value": (rows_n + seqs_n) / t, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d prefill rows evenly spaced over the 128K prefill (index + main branch) and %d decode "
                      "sequences, fp64, %.1f s" % (rows_n, seqs_n, t)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    case = getattr(args, "case", "full") if args is not None else "full"
    PREFILL, DECODE = cases(case)
    tp = make_prefill(PREFILL)
    td = make_decode(DECODE)
    threads = os.cpu_count() or 1
    rows_n, seqs_n = 24, 2
    rng = np.random.default_rng(0)

    def one():
        rows = np.sort(rng.integers(0, PREFILL.n_q, rows_n)).astype(np.int32)
        seqs = np.sort(rng.choice(DECODE.batch, seqs_n, replace=False)).astype(np.int32)
        return oracle_sample(tp, td, PREFILL, DECODE, rows, seqs, threads)

    for _ in range(args.warmup):
        one()
    times = [one() for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = (rows_n + seqs_n) / t
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "%s + %s" % (PREFILL.name, DECODE.name), "seq_len": PREFILL.n_kv,
                   "decode_batch": DECODE.batch},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": "per step %d random rows of the %s prefill (index + main branch) and %d "
                                   "decode sequences" % (rows_n, PREFILL.name, seqs_n)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def relaunch_command(argv, n_gpus: int, port: int):
    """The torchrun command that runs this bench with one process per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n_gpus),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", choices=["full", "small", "long", "prof", "prof_decode", "tiny"], default="full")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-mxfp8", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the projection, mean-pool, packed-batch and adaptive-k measurements")
    args = ap.parse_args(argv)
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # Run directly with N > 1: one process per GPU under torchrun.
        return subprocess.call(relaunch_command(argv, args.gpus, free_port()))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.stderr.write("bench.py: --gpus %d but WORLD_SIZE=%d\n" % (args.gpus, world))
        return 2
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world, torch, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
