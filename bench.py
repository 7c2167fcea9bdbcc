#!/usr/bin/env python
"""Benchmark: exact attention forward + backward on B200 through libfa.so's C ABI.

One step = one pass of the whole hot path over one batch: fa_fwd (tiled forward with online softmax) followed by
fa_bwd (preprocess, recomputing backward, dQ conversion).  The headline workload is the long-context causal case the
throughput target is stated on (B=1, H=16, N=16384, d=128, bf16: the largest single-GPU configuration).  Every other
workload shape (tiny, GPT-2-small, BERT-large with key lengths, 4K / 8K long context, 64K block-sparse) is measured in
the same run under "configs", together with the packed-batch, decode and head-dim-256 paths and the standard
(materialising) attention baseline on the GPT-2 shape.  FLOPs are algorithmic: forward 4*d per visible (query, key)
pair, backward 2.5x forward (five GEMM-shaped products per visible tile pair), step 3.5x forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--no-extras] [--no-cpu-baseline] [--no-e2e]

Multi-GPU (torchrun, one process per GPU): each rank runs its own independent batch of the same shape (attention
heads are independent, so there is no data-path collective: weak scaling); value = all ranks' FLOPs / max time.
--impl reference times the fp64 CPU oracle (the reference arm of this repository) on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd / fwd+bwd TFLOP/s on 1 B200 and % of dense BF16 tensor peak"
DEFAULT_WORKLOAD = "lc16k"
WORKLOAD_NAMES = {
    "gpt2": "gpt2-small-shaped causal self-attention fwd+bwd B8 H12 N1024 d64 bf16",
    "tiny": "tiny exact attention fwd+bwd B1 H2 N256 d64 bf16",
    "bert": "bert-large-shaped attention with key lengths fwd+bwd B16 H16 N512 d64 bf16",
    "lc4k": "long-context causal fwd+bwd B1 H16 N4096 d128 bf16",
    "lc8k": "long-context causal fwd+bwd B1 H16 N8192 d128 bf16",
    "lc16k": "long-context causal fwd+bwd B1 H16 N16384 d128 bf16",
    "bs64k": "block-sparse fwd+bwd B1 H8 N65536 d64 fp16, 128x128 tile mask band4+butterfly+2% random",
    "lc8k_d256": "long-context causal fwd+bwd at head dim 256 B1 H16 N8192 d256 bf16",
}
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
# workloads reported with HBM bandwidth next to TFLOP/s (short sequences: near or below the ridge point)
HBM_REPORTED = ("tiny", "bert")


# ---------------------------------------------------------------------------------------------- FLOP accounting
def visible_pairs(B, H, N, causal, key_lens=None, block_mask=None, tile=128):
    """Number of (query, key) pairs the method must compute (integer, exact)."""
    import numpy as np
    if block_mask is None and key_lens is None:
        return B * H * (N * (N + 1) // 2 if causal else N * N)
    if block_mask is None and not causal:
        return H * N * int(np.sum(np.minimum(np.asarray(key_lens, dtype=np.int64), N)))
    nT = -(-N // tile)
    if key_lens is None and not causal:  # kept tiles times their (possibly ragged) extents
        ext = np.minimum(N - np.arange(nT) * tile, tile).astype(np.int64)
        return B * H * int(ext @ np.asarray(block_mask, dtype=np.int64) @ ext)
    # general: count per tile (rows x visible keys)
    total = 0
    lens = [N] * B if key_lens is None else [min(int(x), N) for x in key_lens]
    for b in range(B):
        for i in range(nT):
            r0, r1 = i * tile, min(N, (i + 1) * tile)
            for j in range(nT):
                if block_mask is not None and not block_mask[i, j]:
                    continue
                c0, c1 = j * tile, min(N, (j + 1) * tile, lens[b])
                if c1 <= c0:
                    continue
                for r in range(r0, r1):
                    hi = min(c1, r + 1) if causal else c1
                    total += max(0, hi - c0)
    return total * H


def row_visible_keys(w, sel_r):
    """Visible keys of each selected query row (integer array), for the sampled-row CPU baseline."""
    import numpy as np
    r = np.asarray(sel_r, dtype=np.int64)
    if w.key_lens or w.blocksparse:
        raise ValueError("row sampling is used on the dense long-context workloads only")
    return np.minimum(r + 1, w.N) if w.causal else np.full_like(r, w.N)


# The sources of the kernels the DRAM-traffic record covers (the d <= 128 forward and backward launches of the
# long-context workload): their headers and the launch code.  Changes elsewhere (the d = 256 kernels, the block-mask
# list builder, the allocation-free entry, the C header's comments) leave the record valid.
TRAFFIC_SOURCES = ("fa_common.cuh", "ptx.cuh", "fa_fwd.cuh", "fa_bwd.cuh", "fa_lib.cu")


def kernel_src_hash():
    """sha256 (first 16 hex digits) over TRAFFIC_SOURCES, file name + contents, in that order."""
    import hashlib
    files = [os.path.join(ROOT, "exact_io_aware_48_b200", "csrc", f) for f in TRAFFIC_SOURCES]
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel):
    """Per-launch DRAM bytes of `kernel` from the committed ncu record, or None if absent or if the kernel sources
    changed since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "kernel_traffic.json")) as f:
            rec = json.load(f)
        if rec.get("src_hash") != kernel_src_hash():
            return None
        e = rec[workload][kernel]
        return int(e["read"]) + int(e["write"])
    except Exception:
        return None


def recorded_standard_traffic():
    """The ncu DRAM totals of one standard (materialising) forward and one tiled forward on the GPT-2 shape."""
    try:
        with open(os.path.join(ROOT, "profiles", "standard_traffic_gpt2.json")) as f:
            return json.load(f)
    except Exception:
        return None


def fwd_flops(d, pairs):
    return 4.0 * d * pairs


def algorithmic_bwd_bytes(w):
    """Minimum DRAM bytes of one bwd_kernel launch: Q, K, V, dO read, dK, dV written (16-bit), LSE2 and D rows
    (fp32) read.  The fp32 dQ partial sums are reduced in L2 and counted separately."""
    e = 2
    return 6 * w.B * w.H * w.N * w.d * e + 2 * 4 * w.B * w.H * w.nT * 128


def algorithmic_pass_bytes(w):
    """Minimum HBM bytes of a whole forward call (Q, K, V read, O written, LSE written) and of a whole backward call
    (Q, K, V, O, dO read, dQ, dK, dV written, LSE read, D written and read)."""
    e = 2
    t = w.B * w.H * w.N * w.d * e
    rows = w.B * w.H * w.N
    return 4 * t + 4 * rows, 8 * t + 12 * rows


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), \
            float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period_s=0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": names}


# ---------------------------------------------------------------------------------------------- GPU arm
class Problem:
    """Device-resident inputs, outputs and workspace for one attention workload; step() = forward + backward through
    fa_fwd / fa_bwd (fa_fwd_blocksparse and fa_bwd with the tile mask for the block-sparse workload)."""

    def __init__(self, w, seed_offset=0, device="cuda"):
        import torch
        from exact_io_aware_48_b200 import _lib
        self.w = w
        self.lib = _lib
        w.seed += seed_offset  # independent problem per rank
        q, k, v, do = w.tensors()
        w.seed -= seed_offset
        self.host = [t.pin_memory() for t in (q, k, v, do)]
        self.q, self.k, self.v, self.do = [t.to(device) for t in self.host]
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.H, w.N), device=device, dtype=torch.float32)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.mask = w.block_mask()
        self.bm = None if self.mask is None else torch.as_tensor(self.mask, dtype=torch.uint8, device=device)
        self.ws_bytes = _lib.fa_bwd_workspace_size(w.B, w.H, w.N, w.d, self.bm is not None)
        self.ws = torch.empty(self.ws_bytes, device=device, dtype=torch.uint8)
        self.fws_bytes = _lib.fa_blocksparse_workspace_size(w.N) if self.bm is not None else 0
        self.fws = torch.empty(max(self.fws_bytes, 1), device=device, dtype=torch.uint8)
        self.dt = _lib.FA_BF16 if w.dtype == "bf16" else _lib.FA_FP16
        self.pairs = visible_pairs(w.B, w.H, w.N, w.causal, w.key_lens_array(), self.mask)
        self.fwd_flops = fwd_flops(w.d, self.pairs)
        self.kl = None
        if w.key_lens:
            self.kl = torch.as_tensor(w.key_lens_array(), dtype=torch.int32, device=device)

    def fwd(self, stream):
        w, L = self.w, self.lib
        if self.bm is None:
            rc = L.fa_fwd(self.q, self.k, self.v, self.o, self.lse, w.B, w.H, w.N, w.d, w.scale, w.causal, self.kl,
                          self.dt, stream)
        else:
            rc = L.fa_fwd_blocksparse(self.q, self.k, self.v, self.o, self.lse, w.B, w.H, w.N, w.d, w.scale,
                                      w.causal, self.kl, self.bm, self.fws, self.fws_bytes, self.dt, stream)
        if rc:
            raise RuntimeError(f"forward: {L.fa_status_string(rc)}")

    def bwd(self, stream):
        w, L = self.w, self.lib
        rc = L.fa_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, self.dq, self.dk, self.dv, w.B, w.H, w.N,
                      w.d, w.scale, w.causal, self.kl, self.bm, self.ws, self.ws_bytes, self.dt, stream)
        if rc:
            raise RuntimeError(f"fa_bwd: {L.fa_status_string(rc)}")

    def step(self, stream):
        self.fwd(stream)
        self.bwd(stream)


def aggregate(local_ms, step_flops, steps, world, device):
    """Whole-job throughput: every rank ran `steps` steps of `step_flops` each; the job time is the max of the
    ranks' device times (one all-reduce MAX when world > 1).  Returns (TFLOP/s, max ms)."""
    total_ms = float(local_ms)
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([total_ms], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    return world * step_flops * steps / (total_ms / 1e3) / 1e12, total_ms


def time_loop(fn, steps, stream, flush, kernel_events=None):
    """Device time (ms) of each call of fn, L2 flushed before each (flush not timed).  kernel_events: optional
    (kernel_id, lib) whose launches are bracketed by per-step events; returns (step_ms list, kernel_ms list)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)] \
        if kernel_events else None
    if kev:  # torch creates the CUDA event lazily on first record: create them before handing them to the library
        for a, b in kev:
            a.record(stream)
            b.record(stream)
        stream.synchronize()
    with torch.cuda.stream(stream):
        for s in range(steps):
            flush.zero_()
            if kev:
                kernel_events[1].fa_set_kernel_events(kernel_events[0], kev[s][0], kev[s][1])
            ev[s][0].record(stream)
            fn(stream)
            ev[s][1].record(stream)
    if kev:
        kernel_events[1].fa_set_kernel_events(kernel_events[0], None, None)
    stream.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    k_ms = [a.elapsed_time(b) for a, b in kev] if kev else None
    return step_ms, k_ms


def check_status(lib, stream, where):
    status = lib.fa_last_device_status(stream)
    if status:
        raise RuntimeError(f"{where}: device status {lib.fa_status_string(status)}")


def measure_config(name, stream, flush, peak, hbm, p=None, reps=20):
    """Forward and backward of one workload, each timed alone (median of `reps` calls, L2 flushed before each):
    call-level ms and TFLOP/s, the main kernels' own ms (events around their launches), fractions of the dense bf16
    peak, and HBM GB/s by algorithmic bytes for the short-sequence workloads.  Block-sparse: TFLOP/s count kept-tile
    pairs and the mask-to-list conversion is timed on its own."""
    import torch
    from exact_io_aware_48_b200 import _lib, inputs
    w = inputs.workloads()[name]
    own = p is None
    if own:
        p = Problem(w)
    for _ in range(5):  # warm-up steps
        p.step(stream)
    f_ms, fk = time_loop(p.fwd, reps, stream, flush, (_lib.FA_KERNEL_FWD, _lib))
    b_ms, bk = time_loop(p.bwd, reps, stream, flush, (_lib.FA_KERNEL_BWD_MAIN, _lib))
    check_status(_lib, stream, name)
    f, b = statistics.median(f_ms), statistics.median(b_ms)
    fkm, bkm = statistics.median(fk), statistics.median(bk)
    ff = p.fwd_flops
    out = {"workload": WORKLOAD_NAMES[name], "visible_pairs": int(p.pairs),
           "fwd_ms": round(f, 4), "bwd_ms": round(b, 4), "fwd_bwd_ms": round(f + b, 4),
           "fwd_tflops": round(ff / f / 1e9, 1), "bwd_tflops": round(2.5 * ff / b / 1e9, 1),
           "fwd_bwd_tflops": round(3.5 * ff / (f + b) / 1e9, 1),
           "fwd_frac": round(ff / f / 1e9 / peak, 4), "bwd_frac": round(2.5 * ff / b / 1e9 / peak, 4),
           "fwd_kernel_ms": round(fkm, 4), "bwd_main_kernel_ms": round(bkm, 4),
           "fwd_kernel_tflops": round(ff / fkm / 1e9, 1), "bwd_main_kernel_tflops": round(2.5 * ff / bkm / 1e9, 1)}
    if name in HBM_REPORTED:
        fb, bb = algorithmic_pass_bytes(w)
        out.update({"fwd_us": round(f * 1e3, 2), "bwd_us": round(b * 1e3, 2),
                    "fwd_hbm_gbs": round(fb / f / 1e6, 1), "bwd_hbm_gbs": round(bb / b / 1e6, 1),
                    "fwd_hbm_frac": round(fb / f / 1e6 / hbm, 4), "bwd_hbm_frac": round(bb / b / 1e6 / hbm, 4),
                    "algorithmic_bytes": {"fwd": fb, "bwd": bb}})
    if p.bm is not None:
        nT = w.nT
        rp, ci, cp, ri = (torch.empty(n, device="cuda", dtype=torch.int32) for n in (nT + 1, nT * nT, nT + 1, nT * nT))

        def lists(st):
            rc = _lib.fa_blockmask_lists(p.bm, nT, rp, ci, cp, ri, st)
            if rc:
                raise RuntimeError(f"fa_blockmask_lists: {_lib.fa_status_string(rc)}")
        for _ in range(3):
            lists(stream)
        l_ms, _ = time_loop(lists, reps, stream, flush)
        lm = statistics.median(l_ms)
        out.update({"kept_tiles": int(p.mask.sum()), "tiles": nT * nT, "mask_lists_ms": round(lm, 4),
                    "flop_convention": "kept-tile pairs (kept tiles x 128 x 128 x H); fwd_ms and bwd_ms include "
                                       "the mask-to-list conversion, which mask_lists_ms times alone"})
    if own:
        del p
        torch.cuda.empty_cache()
    return out


def measure_varlen(stream, flush, peak):
    """Packed variable-length batch (BERT-large shape: B16 H16 d64 bf16, non-causal, the BERT workload's sequence
    lengths U[128, 512]) through fa_fwd_varlen / fa_bwd_varlen, next to the same sequences padded to N = 512 with
    key lengths (the dense entry points).  TFLOP/s count the same visible pairs (sum over sequences of len^2) for
    both; the padded run also spends time on the padding rows' queries."""
    import numpy as np
    import torch
    from exact_io_aware_48_b200 import _lib, inputs
    w = inputs.workloads()["bert"]
    lens = [int(x) for x in w.key_lens_array()]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, H, d, B = int(cu[-1]), w.H, w.d, w.B
    q, k, v, do = (inputs.gaussian((total, H, d), w.seed * 1000 + 50 + t, "bf16").cuda() for t in range(4))
    o = torch.empty_like(q)
    lse = torch.empty((H, total), device="cuda", dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    cud = torch.as_tensor(cu).cuda()
    mx = max(lens)
    ws_bytes = _lib.fa_bwd_varlen_workspace_size(B, H, mx, d)
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    scale = 1.0 / math.sqrt(d)

    def fwd(st):
        rc = _lib.fa_fwd_varlen(q, k, v, o, lse, cud, cud, B, H, mx, mx, total, total, d, scale, False, _lib.FA_BF16,
                                st)
        if rc:
            raise RuntimeError(f"fa_fwd_varlen: {_lib.fa_status_string(rc)}")

    def bwd(st):
        rc = _lib.fa_bwd_varlen(q, k, v, o, do, lse, dq, dk, dv, cud, cud, B, H, mx, mx, total, total, d, scale, False,
                                ws, ws_bytes, _lib.FA_BF16, st)
        if rc:
            raise RuntimeError(f"fa_bwd_varlen: {_lib.fa_status_string(rc)}")

    pairs = H * sum(n * n for n in lens)
    flops = fwd_flops(d, pairs)
    for _ in range(3):
        fwd(stream)
        bwd(stream)
    f_ms, _ = time_loop(fwd, 20, stream, flush)
    b_ms, _ = time_loop(bwd, 20, stream, flush)
    f, b = statistics.median(f_ms), statistics.median(b_ms)
    check_status(_lib, stream, "packed-batch kernels")
    padded = Problem(w)  # the same shape padded to N with key lengths
    for _ in range(3):
        padded.step(stream)
    pf_ms, _ = time_loop(padded.fwd, 20, stream, flush)
    pb_ms, _ = time_loop(padded.bwd, 20, stream, flush)
    pf, pb = statistics.median(pf_ms), statistics.median(pb_ms)
    out = {"workload": f"packed BERT-large shape B{B} H{H} d{d} bf16, lengths U[128,512], total {total} tokens",
           "fwd_ms": round(f, 4), "bwd_ms": round(b, 4),
           "fwd_tflops": round(flops / f / 1e9, 1), "bwd_tflops": round(2.5 * flops / b / 1e9, 1),
           "fwd_bwd_tflops": round(3.5 * flops / (f + b) / 1e9, 1),
           "padded_key_lens_fwd_bwd_ms": round(pf + pb, 4), "padded_key_lens_fwd_bwd_tflops":
           round(3.5 * flops / (pf + pb) / 1e9, 1)}
    del padded
    return out


def measure_decode(stream, flush, hbm_gbs):
    """Split-K/V decode (inference with a full K/V cache): B8 H16, one new query per sequence against 16384 cached
    keys, d128 bf16, causal (aligned with the end of the keys).  Bound by reading the cache: algorithmic bytes are
    K and V (2*B*H*Nk*d*2) plus Q and O; reported as GB/s and as a fraction of the measured HBM copy bandwidth."""
    import torch
    from exact_io_aware_48_b200 import _lib, inputs
    B, H, Nq, Nk, d = 8, 16, 1, 16384, 128
    q = inputs.gaussian((B, H, Nq, d), 500, "bf16").cuda()
    k = inputs.gaussian((B, H, Nk, d), 501, "bf16").cuda()
    v = inputs.gaussian((B, H, Nk, d), 502, "bf16").cuda()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device="cuda", dtype=torch.float32)
    ws_bytes = _lib.fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, 0)
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    scale = 1.0 / math.sqrt(d)

    def step(st):
        rc = _lib.fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, True, None, 0, ws, ws_bytes, _lib.FA_BF16,
                                 st)
        if rc:
            raise RuntimeError(f"fa_fwd_splitkv: {_lib.fa_status_string(rc)}")

    for _ in range(3):
        step(stream)
    ms, _ = time_loop(step, 20, stream, flush)
    check_status(_lib, stream, "split-K/V forward")
    t = statistics.median(ms)
    nbytes = 2 * B * H * Nk * d * 2 + 2 * B * H * Nq * d * 2
    gbs = nbytes / t / 1e6
    return {"workload": f"decode B{B} H{H} Nq{Nq} Nk{Nk} d{d} bf16 causal, split-K/V", "ms": round(t, 4),
            "bytes": nbytes, "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm_gbs, 4) if hbm_gbs else None}


def measure_d256(stream, flush, peak, hbm):
    """Head dim 256 (its own forward and backward kernels) on the long-context causal shape at twice the head dim,
    B1 H16 N8192 bf16, through fa_fwd / fa_bwd.  TFLOP/s by the algorithmic convention (4*d per visible pair
    forward, 2.5x backward)."""
    return measure_config("lc8k_d256", stream, flush, peak, hbm)


def measure_standard(stream, flush, reps=5):
    """The slide deck's suggested experiment ("Run it": a toy that materialises the attention matrix against the
    tiled streaming version) on the GPT-2 shape: eager PyTorch standard attention -- S = scale*QK^T written to HBM,
    masked, softmax, P V, backward through autograd (P and dS also materialised) -- timed next to fa_fwd/fa_bwd on
    the same inputs.  Measurement only: nothing here is on the library's path.  The DRAM-byte ratio is the one an
    ncu capture of the same comparison recorded (profiles/standard_traffic_gpt2.json)."""
    import torch
    from exact_io_aware_48_b200 import inputs
    w = inputs.workloads()["gpt2"]
    p = Problem(w)
    q = p.q.detach().clone().requires_grad_(True)
    k = p.k.detach().clone().requires_grad_(True)
    v = p.v.detach().clone().requires_grad_(True)
    mask = torch.ones(w.N, w.N, device="cuda", dtype=torch.bool).tril() if w.causal else None

    def std_fwd(_s=None):
        s = torch.matmul(q, k.transpose(-1, -2)) * w.scale
        if mask is not None:
            s = s.masked_fill(~mask, float("-inf"))
        return torch.matmul(torch.softmax(s.float(), dim=-1).to(q.dtype), v)

    def std_step(_s=None):
        o = std_fwd()
        o.backward(p.do)
        q.grad = k.grad = v.grad = None

    with torch.cuda.stream(stream):
        for _ in range(3):
            std_step()
            p.step(stream)
    stream.synchronize()
    res = {}
    for name, fn in (("standard_fwd", lambda s: std_fwd()), ("standard_fwd_bwd", std_step),
                     ("tiled_fwd", p.fwd), ("tiled_fwd_bwd", p.step)):
        with torch.cuda.stream(stream):
            ms, _ = time_loop(fn, reps, stream, flush)
        res[name] = statistics.median(ms)
    with torch.no_grad():
        o_std = std_fwd().detach()
    p.fwd(stream)
    stream.synchronize()
    err = float((o_std.float() - p.o.float()).abs().max())
    out = {"workload": WORKLOAD_NAMES["gpt2"], "standard": "eager PyTorch, S and P materialised in HBM",
           "ms": {k2: round(v2, 4) for k2, v2 in res.items()}, "standard_fwd_ms": round(res["standard_fwd"], 4),
           "speedup_fwd": round(res["standard_fwd"] / res["tiled_fwd"], 2),
           "speedup_fwd_bwd": round(res["standard_fwd_bwd"] / res["tiled_fwd_bwd"], 2),
           "max_abs_diff_O": err, "l2": "flushed before every timed call"}
    tr = recorded_standard_traffic()
    if tr:
        out["dram_bytes_recorded"] = {"standard_fwd": tr["standard_fwd_dram_bytes"],
                                      "tiled_fwd": tr["tiled_fwd_dram_bytes"],
                                      "ratio": round(tr["standard_fwd_dram_bytes"] / tr["tiled_fwd_dram_bytes"], 1),
                                      "source": "ncu dram__bytes_read.sum + dram__bytes_write.sum (recorded)"}
    del p
    return out


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from exact_io_aware_48_b200 import _lib, inputs
    from datetime import timedelta

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    _lib.load()
    peak, peak_sus, hbm, peak_src = peaks()
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    w = inputs.workloads()[args.workload]
    p = Problem(w, seed_offset=rank)
    for _ in range(args.warmup):
        p.step(stream)
    stream.synchronize()
    if _lib.fa_last_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error during warm-up")

    # ------------------------------------------------------------------ timed region: K steps, device-timed
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms, kern_ms = time_loop(p.step, args.steps, stream, flush, (_lib.FA_KERNEL_BWD_MAIN, _lib))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if _lib.fa_last_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error in timed region")
    step_flops = 3.5 * p.fwd_flops
    value, total_ms = aggregate(float(sum(step_ms)), step_flops, args.steps, world, "cuda")
    ms_per_step = total_ms / args.steps

    # roofline of the dominant kernel (bwd main: 2.5x forward FLOPs per launch), timed live by events around its
    # launches inside the timed steps
    kmean = float(np.mean(kern_ms))
    achieved = 2.5 * p.fwd_flops / (kmean / 1e3) / 1e12
    kname = f"bwd_kernel<{w.d},{w.dtype}>"
    roofline = {"kernel": kname, "bound": "tensor", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops (burst)", "kernel_ms": round(kmean, 4),
                "traffic": recorded_traffic(w.name, kname), "traffic_unit": "bytes per launch (ncu DRAM read+write)",
                "algorithmic_bytes": algorithmic_bwd_bytes(w)}
    # ------------------------------------------------------------------ end to end through the C ABI, host buffers
    e2e = run_e2e(p, stream, args, world, chunks=args.e2e_chunks) if args.e2e else None

    configs = extra = None
    if args.extras and rank == 0:
        configs = {args.workload: measure_config(args.workload, stream, flush, peak, hbm, p=p)}
    del p
    torch.cuda.empty_cache()
    if args.extras and rank == 0:
        for name in ("tiny", "gpt2", "bert", "lc4k", "lc8k", "lc16k", "bs64k"):
            if name not in configs:
                configs[name] = measure_config(name, stream, flush, peak, hbm)
        extra = {"varlen": measure_varlen(stream, flush, peak), "decode": measure_decode(stream, flush, hbm),
                 "d256": measure_d256(stream, flush, peak, hbm), "standard_vs_tiled": measure_standard(stream, flush)}
    cpu = cpu_baseline(w) if rank == 0 and world == 1 and args.cpu_baseline else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES.get(w.name, w.name),
                       "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "global_batch": w.B * world,
                       "seq_len": w.N, "parallelism": f"dp{world} (independent heads per rank, no collective)",
                       "l2": "flushed (256 MiB write, untimed) before every timed step",
                       "flop_convention": "fwd 4*d*visible pairs; bwd 2.5x; step 3.5x"},
            "frac_of_peak": {"step": round(value / world / peak, 4), "peak_tflops": peak, "peak_source": peak_src,
                             "datasheet_dense_bf16_tflops": 2250.0,
                             "step_of_datasheet": round(value / world / 2250.0, 4)},
            "roofline": roofline,
            "e2e": e2e,
            "gpu_launches": 4 * args.steps,
            "clocks": clk.summary(),
            "configs": configs,
            "paths": extra,
            "cpu_baseline": cpu,
        }
        if configs and args.workload in configs:
            c = configs[args.workload]
            line["fwd_tflops"], line["bwd_tflops"] = c["fwd_tflops"], c["bwd_tflops"]
            line["frac_of_peak"].update({"fwd": c["fwd_frac"], "bwd": c["bwd_frac"]})
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(p, stream, args, world, chunks=4):
    """Same metric through the public C ABI with host buffers: per step, copy q, k, v, dO from pinned host memory,
    run the forward and backward, copy O, LSE, dQ, dK, dV back to pinned host memory; device-timed.

    Heads are independent, so a caller with host data can overlap the copies with the compute: the batch is cut
    into `chunks` groups of batch entries (or of heads when B = 1), each group's inputs go up on one stream, its
    fa_fwd / fa_bwd calls run on the compute stream as soon as its inputs have landed, and its outputs come back on a
    third stream while the next group computes.  Every byte of the step still crosses PCIe inside the timed region.
    The serial form (all inputs, then compute, then all outputs) is timed too and reported beside it."""
    import torch
    w, L = p.w, p.lib
    outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (p.o, p.lse, p.dq, p.dk, p.dv)]
    h2d = sum(t.numel() * t.element_size() for t in p.host)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    dev_in, dev_out = (p.q, p.k, p.v, p.do), (p.o, p.lse, p.dq, p.dk, p.dv)
    if w.B >= chunks and w.B % chunks == 0:
        axis = 0
    elif w.B == 1 and w.H % chunks == 0:
        axis = 1
    else:
        axis, chunks = 0, 1
    Bc, Hc = (w.B // chunks, w.H) if axis == 0 else (w.B, w.H // chunks)

    def part(t, c):  # group c of a [B, H, ...] tensor: contiguous, 16-byte aligned
        n = t.shape[axis] // chunks
        return t.narrow(axis, c * n, n)

    def compute(c, st):
        q, k, v, do = (part(t, c) for t in dev_in)
        o, lse, dq, dk, dv = (part(t, c) for t in dev_out)
        kl = p.kl if (p.kl is None or axis == 1) else p.kl[c * Bc:(c + 1) * Bc]
        if p.bm is None:
            rc = L.fa_fwd(q, k, v, o, lse, Bc, Hc, w.N, w.d, w.scale, w.causal, kl, p.dt, st)
        else:
            rc = L.fa_fwd_blocksparse(q, k, v, o, lse, Bc, Hc, w.N, w.d, w.scale, w.causal, kl, p.bm, p.fws,
                                      p.fws_bytes, p.dt, st)
        if rc:
            raise RuntimeError(f"forward: {L.fa_status_string(rc)}")
        rc = L.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, Bc, Hc, w.N, w.d, w.scale, w.causal, kl, p.bm, p.ws,
                      p.ws_bytes, p.dt, st)
        if rc:
            raise RuntimeError(f"fa_bwd: {L.fa_status_string(rc)}")

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    state = {"comp": [None] * chunks, "out": [None] * chunks}

    def step():
        ins = []
        for c in range(chunks):
            if state["comp"][c] is not None:
                s_in.wait_event(state["comp"][c])  # the previous step's compute has read this group's inputs
            with torch.cuda.stream(s_in):
                for dst, src in zip(dev_in, p.host):
                    part(dst, c).copy_(part(src, c), non_blocking=True)
            e = ev()
            e.record(s_in)
            ins.append(e)
        for c in range(chunks):
            stream.wait_event(ins[c])
            if state["out"][c] is not None:
                stream.wait_event(state["out"][c])  # the previous step's outputs of this group have left
            compute(c, stream)
            e = ev()
            e.record(stream)
            state["comp"][c] = e
            s_out.wait_event(e)
            with torch.cuda.stream(s_out):
                for dst, src in zip(outs, dev_out):
                    part(dst, c).copy_(part(src, c), non_blocking=True)
            e2 = ev()
            e2.record(s_out)
            state["out"][c] = e2

    def serial_step(s):
        for dst, src in zip(dev_in, p.host):
            dst.copy_(src, non_blocking=True)
        p.step(s)
        for dst, src in zip(outs, dev_out):
            dst.copy_(src, non_blocking=True)

    n = max(5, args.steps // 4)

    def timed(run):
        for _ in range(2):
            run()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(s_in)
        s_in.wait_event(ev0)
        for _ in range(n):
            run()
        for s_ in (s_in, stream):
            e = ev()
            e.record(s_)
            s_out.wait_event(e)
        ev1.record(s_out)
        torch.cuda.synchronize()
        return ev0.elapsed_time(ev1) / n

    def serial():
        with torch.cuda.stream(s_in):
            serial_step(s_in)

    def copies():  # the step's PCIe traffic alone, both directions at once: the bound for the overlapped step
        with torch.cuda.stream(s_in):
            for dst, src in zip(dev_in, p.host):
                dst.copy_(src, non_blocking=True)
        with torch.cuda.stream(s_out):
            for dst, src in zip(outs, dev_out):
                dst.copy_(src, non_blocking=True)

    ms_serial = timed(serial)
    ms_copies = timed(copies)
    ref = [t.clone() for t in outs]  # the unchunked step's results
    ms = timed(step)
    check_status(L, stream, "end-to-end steps")
    for name, a, b in zip(("O", "LSE", "dQ", "dK", "dV"), ref, outs):  # chunking must not change the results
        if name == "dQ":  # fp32 reductions in run-dependent order: one 16-bit unit in the last place at most
            ok = float((a.float() - b.float()).abs().max()) <= 2.0 ** -7 * max(float(a.float().abs().max()), 1e-3)
        else:
            ok = torch.equal(a, b)
        if not ok:
            raise RuntimeError(f"end-to-end: {name} of the overlapped steps differs from the unchunked step")
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms, ms_serial, ms_copies], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, ms_serial, ms_copies = float(t[0].item()), float(t[1].item()), float(t[2].item())
    val = world * 3.5 * p.fwd_flops / (ms / 1e3) / 1e12
    return {"value": round(val, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "overlap": f"{chunks} groups of {'batch entries' if axis == 0 else 'heads'}, "
            "copies in, compute and copies out on three streams",
            "serial_ms_per_step": round(ms_serial, 4),
            "serial_value": round(world * 3.5 * p.fwd_flops / (ms_serial / 1e3) / 1e12, 3),
            "copies_only_ms_per_step": round(ms_copies, 4),
            "copies_only_gbs": {"h2d": round(h2d / (ms_copies / 1e3) / 1e9, 1),
                                "d2h": round(d2h / (ms_copies / 1e3) / 1e9, 1)}}


# ---------------------------------------------------------------------------------------------- CPU oracle
def host_cpu():
    """CPU model and core counts of this host."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except AttributeError:
        avail = os.cpu_count()
    return {"model": model, "nproc": avail, "logical_cpus": os.cpu_count()}


class OracleRows:
    """The fp64 oracle on sampled query rows of a workload: per row, the row's forward (O, LSE) and its dQ (which
    recomputes the row's forward).  Credited with the algorithmic FLOPs of that work: 4*d per visible pair for the
    forward and 6*d for the dQ share of the backward (recomputed scores, dP, dQ; the backward's full 10*d adds dV and
    dK), so rate = credited FLOPs / seconds and the full step's extrapolated time = 3.5 * 4*d * all pairs / rate."""

    def __init__(self, w):
        import oracle
        from exact_io_aware_48_b200 import inputs
        oracle.build()
        self.w = w
        self.inputs = inputs
        self.oracle = oracle
        self.q, self.k, self.v, self.do = (inputs.to_f64(t) for t in w.tensors())

    def run(self, nrows, seed):
        w = self.w
        sb, sr = self.inputs.sample_rows(seed, w.B * w.H, w.N, nrows)
        t0 = time.perf_counter()
        self.oracle.attn_fwd_rows(self.q, self.k, self.v, w.scale, sb, sr, causal=w.causal)
        self.oracle.attn_bwd_rows(self.q, self.k, self.v, self.do, w.scale, sb, sr, causal=w.causal)
        dt = time.perf_counter() - t0
        return dt, 10.0 * w.d * float(row_visible_keys(w, sr).sum())


def cpu_baseline(w, target_s=10.0):
    """The oracle as it stands on this host's cores, on a bounded sample of the timed workload (sampled query rows,
    rate extrapolated to the full step), plus the tiny workload's full fwd+bwd on one core and on all cores."""
    import oracle
    from exact_io_aware_48_b200 import inputs
    oracle.build()
    cores = oracle.num_threads()
    rows = OracleRows(w)
    secs, flops, n, nrows = 0.0, 0.0, 0, 256
    while secs < target_s and n < 64:
        dt, f = rows.run(nrows, 5000 + n)
        secs += dt
        flops += f
        n += 1
    rate = flops / secs
    full_flops = 3.5 * fwd_flops(w.d, visible_pairs(w.B, w.H, w.N, w.causal, w.key_lens_array(), w.block_mask()))
    tiny = inputs.workloads()["tiny"]
    tq, tk, tv, tdo = (inputs.to_f64(t) for t in tiny.tensors())
    tiny_flops = 3.5 * fwd_flops(tiny.d, visible_pairs(tiny.B, tiny.H, tiny.N, tiny.causal))

    def tiny_rate(threads, reps=5):
        oracle.set_num_threads(threads)
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.attn_bwd(tq, tk, tv, tdo, tiny.scale, causal=tiny.causal)
        return reps * tiny_flops / (time.perf_counter() - t0) / 1e12

    tiny_1 = tiny_rate(1)
    tiny_all = tiny_rate(cores)
    oracle.set_num_threads(cores)
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} x {nrows} seeded query rows of the timed workload: each row's forward and dQ (fp64 C "
                      f"oracle, OpenMP over rows), {secs:.1f} s; rate extrapolated to the full step",
            "extrapolated_full_step_s": round(full_flops / rate, 1), "extrapolated": True,
            "host": host_cpu(),
            "tiny_full_fwd_bwd": {"workload": WORKLOAD_NAMES["tiny"], "tflops_1_core": round(tiny_1, 6),
                                  f"tflops_{cores}_cores": round(tiny_all, 6)}}


def run_reference(args):
    from exact_io_aware_48_b200 import inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = inputs.workloads()[args.workload]
    rows = OracleRows(w)
    nrows = 256  # each step: 256 seeded query rows of the workload (bounded sample)
    for s in range(args.warmup):
        rows.run(nrows, 9000 + s)
    secs, flops = 0.0, 0.0
    for s in range(args.steps):
        dt, f = rows.run(nrows, 9500 + s)
        secs += dt
        flops += f
    val = flops / secs / 1e12
    ms = secs / args.steps * 1e3
    cores = rows.oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES.get(w.name, w.name),
                       "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "global_batch": w.B,
                       "seq_len": w.N, "parallelism": "host cores (OpenMP)"},
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{nrows} seeded query rows per step: each row's forward and dQ, fp64; rate "
                                       "extrapolated to the full step", "host": host_cpu()},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_standard(args):
    """Prints the standard-vs-tiled comparison alone (the default run includes it under paths.standard_vs_tiled)."""
    import torch
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    line = {"mode": "standard-attention baseline", **measure_standard(stream, flush, reps=max(5, args.steps // 2))}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--standard", action="store_true",
                    help="time eager standard (materialising) attention next to the tiled kernels and exit")
    ap.add_argument("--no-extras", "--no-targets", dest="extras", action="store_false",
                    help="skip the other workloads and paths (configs, paths keys)")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-chunks", type=int, default=4,
                    help="groups of batch entries (or heads when B = 1) whose copies overlap the compute in e2e")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOAD_NAMES),
                    help="timed workload (default: the 16K long-context causal d128 case; others are for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.standard:
        run_standard(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
