#!/usr/bin/env python3
"""Benchmark of the HGRN2 hot path on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one training pass of the chunkwise recurrence over one batch: the
forward that keeps the chunk states (hgrn2_fwd_train) and the backward that
reads them (hgrn2_bwd_saved, gradients of q, log f and i) on the training workload B=8, H=16, T=2048, d_k=d_v=128, bf16 token tensors,
fp32 state, forget-gate lower bound 0.95, dO ~ N(0,1).  Inputs (268 MB of
token tensors per step, more than the 126 MB L2) are resident in HBM before
the timed region.  Under torchrun each rank runs its own batch on its own GPU
(data-parallel replicas, no collective on the data path): weak scaling.

The same JSON line also carries the decode step (B=256, H=16, 1000 in-place
steps of the fp32 state), the training pair on packed documents of varied
length (16,384 tokens, H=16), the training pair with 64-wide heads (H=32), the two
forward-only workloads (forward layer, long sequence), the scalar-decay variant,
end-to-end numbers through host buffers, the
roofline of the dominant call, SM clocks sampled during the timed region, and
the CPU oracle timed on a bounded sample (rank 0, one GPU only).
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "HGRN2 fwd+bwd tokens/s (H=16,d=128,T=2048) & % bf16 tensor peak; step GB/s"

# Algorithmic counts per token per head (d_k = d_v = d = 128, chunk C = 64 for accounting,
# causal half of the intra-chunk products, bf16 token tensors, state recompute not counted):
D = 128
C_ACC = 64
FWD_FLOPS = C_ACC * (D + D) + 4 * D * D           # 81,920
BWD_FLOPS = C_ACC * (3 * D + 2 * D) + 8 * D * D   # 172,032
FWD_BYTES = 2 * (D + D + D + D)                   # read q, log f, i; write o = 1,024
BWD_BYTES = 2 * (4 * D + 3 * D)                   # read q, log f, i, dO; write dq, dlog f, di = 1,792
STEP_BYTES_PER_BH = 2 * D * D * 4 + 2 * (4 * D)   # decode: S read+write fp32, q/log f/i/o bf16 = 132,096
# decode-step backward: S and dS read, dS_prev written (fp32); q, log f, i, dO read and dq, dlog f,
# di written (bf16) = 198,400
STEP_BWD_BYTES_PER_BH = 3 * D * D * 4 + 2 * (7 * D)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK / MASTER_*).  The data
    path has no collective: the process group only carries the barriers and the max over ranks
    of the device times.  backend "gloo" (CPU) is for tests of this host logic."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: the whole job is done when every rank is."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(tokens_per_rank_step: int, steps: int, ms: float, world: int) -> float:
    """Tokens per second of the whole job: every rank processes its own batch (weak scaling)."""
    return world * tokens_per_rank_step * steps / (ms / 1e3)


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch."""
    return 1003 + rank


def traffic_record(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    src_hash = csrc_hash()
    for line in open(p):
        if line.startswith("#") or "|" not in line:
            continue
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == kernel and cells[1] == src_hash:
            try:
                return float(cells[3])
            except ValueError:
                return None
    return None


def csrc_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_attention_hgrn2_b200", "csrc")
    for fn in sorted(os.listdir(d)):
        if fn.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(d, fn), "rb").read())
    return h.hexdigest()[:12]


# ------------------------------------------------------------------------------------------ ours
def run_ours(args, world, rank, local):
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I

    L.load_library()
    w = I.TRAIN
    B, T, H, dk, dv, chunk = w.B, w.T, w.H, w.dk, w.dv, w.chunk
    inp = I.make_workload(w, seed=rank_seed(rank))
    dev = torch.device("cuda", local)
    q, lf, x, dO = (inp[k].to(dev) for k in ("q", "log_f", "i", "dO"))
    ws_f = torch.empty(max(L.workspace_size(B, T, H, dk, dv, chunk, w.dtype, False), 16), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(max(L.workspace_size(B, T, H, dk, dv, chunk, w.dtype, True), 16), dtype=torch.uint8, device=dev)
    o = torch.empty_like(x)
    sv = L.new_saved(q)   # chunk states kept by the training forward for the backward

    def step():
        L.fwd(q, lf, x, chunk=chunk, out=o, workspace=ws_f, saved=sv)
        return L.bwd(q, lf, x, dO, chunk=chunk, workspace=ws_b, saved=sv)

    def fwd_call():
        L.fwd(q, lf, x, chunk=chunk, out=o, workspace=ws_f, saved=sv)

    def bwd_call():
        L.bwd(q, lf, x, dO, chunk=chunk, workspace=ws_b, saved=sv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # estimate the step time, to keep the GPU busy for ~50 ms before the timed region
    w0 = time.perf_counter()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n_spin = max(1, int(0.05 / max((time.perf_counter() - w0) / 3, 1e-6)))
    stream = torch.cuda.current_stream()
    K = args.steps
    step_est_ms = 1e3 * (time.perf_counter() - w0) / 3
    # the K-step timed region is repeated until about 100 ms of steps have been timed (at most
    # 25 regions); the reported time is the median region, with the spread beside it
    reps = max(1, min(25, int(np.ceil(100.0 / max(K * step_est_ms, 1e-3)))))
    gate = 2_000_000   # cycles of a device-side sleep that holds the queue while the host fills it
    region_ms = []
    with ClockSampler(local) as clk:
        time.sleep(0.1)              # nvidia-smi starting up
        for _ in range(n_spin):      # clocks back up after that idle period
            step()
        launches0 = L.counters()[2]  # synchronises
        for _ in range(reps):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            barrier(world)
            torch.cuda.synchronize()
            # timed region: only the two bracketing events, so nothing but the calls runs between
            # them; the sleep ahead of t0 lets the host queue the K steps before the GPU reaches them
            torch.cuda._sleep(gate)
            t0.record(stream)
            for _ in range(K):
                step()
            t1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            region_ms.append(t0.elapsed_time(t1))
        launches = (L.counters()[2] - launches0) // reps
        # per-call durations, same data and clocks: K forward calls, then K backward calls
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        torch.cuda._sleep(gate)
        ev[0].record(stream)
        for _ in range(K):
            fwd_call()
        ev[1].record(stream)
        for _ in range(K):
            bwd_call()
        ev[2].record(stream)
        torch.cuda.synchronize()
    ms_local = statistics.median(region_ms)
    ms = max_over_ranks(ms_local, world)
    fwd_ms = ev[0].elapsed_time(ev[1]) / K
    bwd_ms = ev[1].elapsed_time(ev[2]) / K
    ms_per_step = ms / K
    tokens_per_step = B * T
    value = whole_job_value(tokens_per_step, K, ms, world)

    pk = peaks()
    th = B * T * H   # token-heads per step
    if bwd_ms >= fwd_ms:
        dom, dom_ms, dom_bytes = "hgrn2_bwd_saved", bwd_ms, BWD_BYTES * th
    else:
        dom, dom_ms, dom_bytes = "hgrn2_fwd_train", fwd_ms, FWD_BYTES * th
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    tr = traffic_record(dom)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                "traffic": tr, "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_launch": dom_bytes, "avg_launch_ms": round(dom_ms, 4),
                "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4)}
    flops_step = (FWD_FLOPS + BWD_FLOPS) * th
    bytes_step = (FWD_BYTES + BWD_BYTES) * th
    tensor_frac = flops_step / (ms_per_step / 1e3) / (pk["bf16_tflops_sustained"] * 1e12)
    step_roof = {"achieved_gbs": round(bytes_step / (ms_per_step / 1e3) / 1e9, 1),
                 "hbm_frac": round(bytes_step / (ms_per_step / 1e3) / 1e9 / pk["hbm_gbs"], 4),
                 "algorithmic_tflops": round(flops_step / (ms_per_step / 1e3) / 1e12, 2),
                 "bf16_peak_frac": round(tensor_frac, 4),
                 "bf16_peak_tflops": pk["bf16_tflops_sustained"]}

    clocks = clk.summary()
    timed = {"regions": reps, "steps_per_region": K,
             "ms_per_step_median": round(ms_local / K, 5),
             "ms_per_step_min": round(min(region_ms) / K, 5), "ms_per_step_max": round(max(region_ms) / K, 5),
             "spread": round((max(region_ms) - min(region_ms)) / ms_local, 4),
             "timed_ms_total": round(sum(region_ms), 2)}
    if clocks.get("sm_mhz"):
        # time x median SM clock: comparable across runs at different clocks
        timed["ms_x_sm_ghz_per_step"] = round(ms_local / K * clocks["sm_mhz"] / 1e3, 5)
    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
           "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": w.name, "B": B, "T": T, "H": H, "d_k": dk, "d_v": dv, "chunk": chunk,
                      "tensor_core_chunk": 128,
                      "chunk_note": "chunk is the call's argument (the exact route's chunk); the tensor-core "
                                    "kernels that run this workload tile by 128 tokens",
                      "lb": w.lb, "global_batch": B * world, "seq_len": T,
                      "parallelism": f"dp{world} (independent replicas, no collective)",
                      "calls": "hgrn2_fwd_train + hgrn2_bwd_saved",
                      "l2": "no flush: 268 MB of token inputs per step > 126 MB L2"},
           "roofline": roofline, "step_roofline": step_roof, "gpu_launches": launches,
           "timed_regions": timed, "clocks": clocks}

    if not args.no_e2e:
        out["e2e"] = run_e2e(args, q, lf, x, dO, o, ws_f, ws_b, sv, w, world)
    if not args.no_decode:
        out["decode_step"] = run_decode(args, dev, pk)
    if not args.no_varlen:
        out["varlen"] = run_varlen(args, dev, pk, rank)
    if not args.no_lb0:
        from linear_attention_hgrn2_b200 import inputs as I
        out["lower_bound_zero"] = run_head_dim(args, dev, pk, rank, I.TRAIN_LB0, 19, ref_ms=ms_per_step)
    if not args.no_d64:
        from linear_attention_hgrn2_b200 import inputs as I
        out["head_dim_64"] = run_head_dim(args, dev, pk, rank, I.TRAIN_D64, 9)
    if not args.no_d256:
        from linear_attention_hgrn2_b200 import inputs as I
        out["head_dim_256"] = run_head_dim(args, dev, pk, rank, I.TRAIN_D256, 17)
    if not args.no_long_train:
        from linear_attention_hgrn2_b200 import inputs as I
        out["long_sequence_train"] = run_head_dim(args, dev, pk, rank, I.TRAIN_LONG, 23)
    if not args.no_fwd_configs:
        out["forward_configs"] = run_fwd_configs(args, dev, pk, rank)
    if not args.no_scalar:
        out["scalar_decay"] = run_scalar(args, dev, pk, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(inp, w, budget_s=args.cpu_seconds)
        out["cpu_baseline_other_workloads"] = cpu_baseline_others(budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_e2e(args, q, lf, x, dO, o, ws_f, ws_b, sv, w, world):
    """Same step through host buffers: every step's inputs go host -> device from pinned memory and
    all its outputs (o, dq, d log f, di) come back device -> host, inside the timed region.

    The copies are pipelined as a training input pipeline would be: the upload of step k+1 (one
    stream), the compute of step k (the current stream) and the download of step k-1 (a third
    stream) overlap, with two device buffer sets.  The timed region includes the pipeline's fill
    (the first upload) and drain (the last download)."""
    import linear_attention_hgrn2_b200 as L
    hin = [t.cpu().pin_memory() for t in (q, lf, x, dO)]
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, q, q, x)]
    din = [[q, lf, x, dO], [torch.empty_like(t) for t in (q, lf, x, dO)]]
    dout_o = [o, torch.empty_like(o)]
    K = max(3, min(args.steps, 32))   # the pipeline's fill and drain are timed once per run
    comp = torch.cuda.current_stream()
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    first = [True, True]

    def upload(k):
        sl = k % 2
        with torch.cuda.stream(s_up):
            if not first[sl]:
                s_up.wait_event(comp_done[sl])      # step k-2 has finished reading this buffer set
            for d, h in zip(din[sl], hin):
                d.copy_(h, non_blocking=True)
            up_done[sl].record(s_up)

    def compute_and_download(k):
        sl = k % 2
        comp.wait_event(up_done[sl])
        if not first[sl]:
            comp.wait_event(down_done[sl])          # step k-2's outputs have left this buffer set
        qq, ll, xx, dd = din[sl]
        L.fwd(qq, ll, xx, chunk=w.chunk, out=dout_o[sl], workspace=ws_f, saved=sv)
        dq, dlf, di, _ = L.bwd(qq, ll, xx, dd, chunk=w.chunk, workspace=ws_b, saved=sv)
        comp_done[sl].record(comp)
        first[sl] = False
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[sl])
            for h, d in zip(hout, (dout_o[sl], dq, dlf, di)):
                d.record_stream(s_down)
                h.copy_(d, non_blocking=True)
            down_done[sl].record(s_down)

    def run(nsteps):
        upload(0)
        for k in range(nsteps):
            if k + 1 < nsteps:
                upload(k + 1)
            compute_and_download(k)
        comp.wait_stream(s_down)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_up.wait_event(a)
    run(K)
    b.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world)
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return {"value": round(whole_job_value(w.B * w.T, K, ms, world), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
            "ms_per_step": round(ms / K, 3),
            "pipeline": "upload k+1 | compute k | download k-1 on three streams; fill and drain timed"}


def run_decode(args, dev, pk):
    """Decode workload: B=256, H=16, d=128, 1000 consecutive in-place steps (one timed sequence)."""
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I
    cfg = I.DECODE
    steps = cfg["steps"]
    d = I.make_decode(cfg["B"], cfg["H"], cfg["dk"], cfg["dv"], steps, cfg["dtype"], cfg["lb"],
                      seed=1005, device=str(dev))
    S = d["S"]
    o = torch.empty((cfg["B"], cfg["H"], cfg["dv"]), dtype=cfg["dtype"], device=dev)
    for t in range(5):
        L.step(d["q"][t], d["log_f"][t], d["i"][t], S, out=o)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for t in range(steps):
        L.step(d["q"][t], d["log_f"][t], d["i"][t], S, out=o)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # the same steps with the lower-bounded gate formed in the kernel from the raw logits
    for t in range(5):
        L.step_lb(d["q"][t], d["g"][t], d["i"][t], cfg["lb"], S, out=o)
    torch.cuda.synchronize()
    a.record()
    for t in range(steps):
        L.step_lb(d["q"][t], d["g"][t], d["i"][t], cfg["lb"], S, out=o)
    b.record()
    torch.cuda.synchronize()
    ms_lb = a.elapsed_time(b) / steps
    # the step backward, from the last token to the first, dS carried in place (truncated BPTT
    # through decode steps); one state buffer stands for the per-step states (268 MB > L2)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1006)
    dO = torch.randn((steps,) + tuple(o.shape), generator=gen, device=dev).to(cfg["dtype"])
    dS = torch.randn(tuple(S.shape), generator=gen, device=dev)
    for t in range(5):
        L.step_bwd(d["q"][t], d["log_f"][t], d["i"][t], S, dO[t], dS, dS_out=dS)
    torch.cuda.synchronize()
    a.record()
    for t in reversed(range(steps)):
        L.step_bwd(d["q"][t], d["log_f"][t], d["i"][t], S, dO[t], dS, dS_out=dS)
    b.record()
    torch.cuda.synchronize()
    ms_bwd = a.elapsed_time(b) / steps
    nbh = cfg["B"] * cfg["H"]
    gbs_bwd = STEP_BWD_BYTES_PER_BH * nbh / (ms_bwd / 1e3) / 1e9
    del dO, dS
    gbs = STEP_BYTES_PER_BH * nbh / (ms / 1e3) / 1e9
    gbs_lb = STEP_BYTES_PER_BH * nbh / (ms_lb / 1e3) / 1e9
    res = {"workload": cfg["name"], "ms_per_step": round(ms, 5), "tokens_per_s": round(cfg["B"] / (ms / 1e3), 1),
           "achieved_gbs": round(gbs, 1), "peak_gbs": pk["hbm_gbs"], "frac": round(gbs / pk["hbm_gbs"], 4),
           "bytes_per_step": STEP_BYTES_PER_BH * nbh, "steps": steps,
           "l2": "state 268 MB > 126 MB L2, streaming loads/stores",
           "lower_bound_gate": {"call": "hgrn2_step_lb (f = lb + (1-lb) sigmoid(g) in the kernel)",
                                "ms_per_step": round(ms_lb, 5), "achieved_gbs": round(gbs_lb, 1),
                                "frac": round(gbs_lb / pk["hbm_gbs"], 4)},
           "backward": {"call": "hgrn2_step_bwd (dS in place, last token to first)",
                        "ms_per_step": round(ms_bwd, 5), "bytes_per_step": STEP_BWD_BYTES_PER_BH * nbh,
                        "achieved_gbs": round(gbs_bwd, 1), "frac": round(gbs_bwd / pk["hbm_gbs"], 4)}}
    del d, S
    torch.cuda.empty_cache()
    return res


def run_varlen(args, dev, pk, rank):
    """Packed documents: the training pair (hgrn2_fwd_varlen with saved states, then
    hgrn2_bwd_varlen) over 16,384 tokens cut into documents of exponential length."""
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I
    cfg = I.VARLEN
    lens = I.document_lengths(cfg["total_T"], cfg["mean_len"], seed=rank_seed(rank) + 7)
    inp = I.make_varlen(lens, cfg["H"], cfg["dk"], cfg["dv"], cfg["dtype"], cfg["lb"], seed=rank_seed(rank) + 8,
                        with_dO=True)
    q, lf, x, dO, cu = (inp[k].to(dev) for k in ("q", "log_f", "i", "dO", "cu_seqlens"))
    sv = L.new_saved_varlen(q, cu)
    o = torch.empty_like(x)
    chunk = cfg["chunk"]

    def fwd_call():
        L.fwd_varlen(q, lf, x, cu, chunk=chunk, out=o, saved=sv)

    def bwd_call():
        L.bwd_varlen(q, lf, x, dO, cu, chunk=chunk, saved=sv)

    for _ in range(max(args.warmup, 3)):
        fwd_call()
        bwd_call()
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    torch.cuda._sleep(2_000_000)
    ev[0].record()
    for _ in range(K):
        fwd_call()
        bwd_call()
    ev[1].record()
    for _ in range(K):
        fwd_call()
    ev[2].record()
    for _ in range(K):
        bwd_call()
    ev[3].record()
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / K
    fwd_ms = ev[1].elapsed_time(ev[2]) / K
    bwd_ms = ev[2].elapsed_time(ev[3]) / K
    th = cfg["total_T"] * cfg["H"]
    gbs_b = BWD_BYTES * th / (bwd_ms / 1e3) / 1e9
    res = {"workload": cfg["name"], "documents": len(lens), "min_len": min(lens), "max_len": max(lens),
           "tokens_per_s": round(cfg["total_T"] / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
           "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
           "bwd_achieved_gbs": round(gbs_b, 1), "bwd_frac": round(gbs_b / pk["hbm_gbs"], 4),
           "calls": "hgrn2_fwd_varlen (saved states) + hgrn2_bwd_varlen", "steps": K}
    del inp, q, lf, x, dO, sv, o
    torch.cuda.empty_cache()
    return res


def run_head_dim(args, dev, pk, rank, w, seed_off, ref_ms=None):
    """The training pair on a variant of the training workload: 64-wide heads (B=8, H=32, T=2048),
    256-wide heads (B=8, H=8, T=2048, run as 128-wide blocks), the first layer's forget-gate
    lower bound lb = 0 (the same shapes; with ref_ms, the headline step's time, for the ratio), or
    the long sequence's shape (B=1, H=8, T=32768: 8 (b,h), both calls in sequence segments).
    Exact-route passes over the timed steps are counted on the device."""
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I
    inp = I.make_workload(w, seed=rank_seed(rank) + seed_off)
    q, lf, x, dO = (inp[k].to(dev) for k in ("q", "log_f", "i", "dO"))
    sv = L.new_saved(q)
    o = torch.empty_like(x)

    def fwd_call():
        L.fwd(q, lf, x, chunk=w.chunk, out=o, saved=sv)

    def bwd_call():
        L.bwd(q, lf, x, dO, chunk=w.chunk, saved=sv)

    for _ in range(max(args.warmup, 3)):
        fwd_call()
        bwd_call()
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    L.counters(reset=True)
    torch.cuda._sleep(2_000_000)
    ev[0].record()
    for _ in range(K):
        fwd_call()
        bwd_call()
    ev[1].record()
    for _ in range(K):
        fwd_call()
    ev[2].record()
    for _ in range(K):
        bwd_call()
    ev[3].record()
    torch.cuda.synchronize()
    cnt = L.counters(reset=True)
    ms = ev[0].elapsed_time(ev[1]) / K
    fwd_ms = ev[1].elapsed_time(ev[2]) / K
    bwd_ms = ev[2].elapsed_time(ev[3]) / K
    th = w.B * w.T * w.H
    bwd_bytes = 2 * 7 * w.dk * th   # read q, log f, i, dO; write dq, dlog f, di (bf16)
    gbs_b = bwd_bytes / (bwd_ms / 1e3) / 1e9
    res = {"workload": w.name, "tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
           "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4), "bwd_achieved_gbs": round(gbs_b, 1),
           "bwd_frac": round(gbs_b / pk["hbm_gbs"], 4), "calls": "hgrn2_fwd_train + hgrn2_bwd_saved", "steps": K,
           "lb": w.lb, "exact_route_passes": int(cnt[0]), "tensor_core_chunk_passes": int(cnt[1])}
    if ref_ms:
        res["step_time_vs_headline"] = round(ms / ref_ms, 4)
    if w.dk > 128 or w.dv > 128:
        res["route"] = ("128-wide half-head blocks on the tensor cores, read in place; each block pair adds its "
                        "share of the outputs by TMA reduce-add into zeroed outputs; bwd_frac counts the algorithmic "
                        "bytes of the wide head only")
    del inp, q, lf, x, dO, sv, o
    torch.cuda.empty_cache()
    return res


def run_fwd_configs(args, dev, pk, rank):
    """The two forward-only workloads: the forward layer (B=4, H=8, T=2048, lb=0.5) and the long
    sequence (B=1, H=8, T=32768, lb=0.9, h0 in, hT out).  With 32 and 8 (b,h) pairs they run the
    segmented forward: every segment from a zero state, then the carried states added to the
    segments' first chunks by a fix-up that sums the entering states itself (2 launches: the
    forward layer's 4 segments per pair, the long sequence's 18)."""
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I
    res = {}
    for w in (I.FWD_LAYER, I.LONG):
        inp = I.make_workload(w, seed=rank_seed(rank) + 11)
        q, lf, x = (inp[k].to(dev) for k in ("q", "log_f", "i"))
        h0 = inp["h0"].to(dev) if "h0" in inp else None
        o = torch.empty_like(x)
        ws = torch.empty(max(L.workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.dtype, False), 16),
                         dtype=torch.uint8, device=dev)

        def call():
            return L.fwd(q, lf, x, h0, want_hT=w.want_hT, chunk=w.chunk, out=o, workspace=ws)

        for _ in range(max(args.warmup, 3)):
            call()
        torch.cuda.synchronize()
        K = args.steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        L.counters(reset=True)
        torch.cuda._sleep(2_000_000)
        a.record()
        for _ in range(K):
            call()
        b.record()
        torch.cuda.synchronize()
        launches = L.counters(reset=True)[2] // K
        ms = a.elapsed_time(b) / K
        th = w.B * w.T * w.H
        nbytes = FWD_BYTES * th + (2 * w.B * w.H * w.dk * w.dv * 4 if w.want_hT else 0)
        gbs = nbytes / (ms / 1e3) / 1e9
        res[w.name] = {"tokens_per_s": round(w.B * w.T / (ms / 1e3), 1), "ms_per_call": round(ms, 4),
                       "launches_per_call": launches, "achieved_gbs": round(gbs, 1),
                       "frac": round(gbs / pk["hbm_gbs"], 4), "calls": K}
        del inp, q, lf, x, o, ws, h0
        torch.cuda.empty_cache()
    return res


def run_scalar(args, dev, pk, rank):
    """The scalar-decay variant (one decay per head and token, explicit key) at the training
    workload's shape: hgrn2_scalar_fwd + hgrn2_scalar_bwd."""
    import linear_attention_hgrn2_b200 as L
    from linear_attention_hgrn2_b200 import inputs as I
    w = I.SCALAR_TRAIN
    inp = I.make_scalar_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.lb, seed=rank_seed(rank) + 13, with_dO=True)
    g = {k: t.to(dev) for k, t in inp.items()}
    sv = L.new_scalar_saved(g["q"])   # the training pair: chunk states kept by the forward

    def fwd_call():
        L.scalar_fwd(g["q"], g["k"], g["v"], g["log_g"], saved=sv)

    def bwd_call():
        L.scalar_bwd(g["q"], g["k"], g["v"], g["log_g"], g["dO"], saved=sv)

    for _ in range(2):
        fwd_call()
        bwd_call()
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for _ in range(K):
        fwd_call()
    ev[1].record()
    for _ in range(K):
        bwd_call()
    ev[2].record()
    torch.cuda.synchronize()
    fwd_ms = ev[0].elapsed_time(ev[1]) / K
    bwd_ms = ev[1].elapsed_time(ev[2]) / K
    # algorithmic bytes per token-head (bf16): forward reads q, k, v, log g and writes o; backward
    # reads q, k, v, log g, dO and writes dq, dk, dv, d log g
    dk, dv = w.dk, w.dv
    step_bytes = 2 * (2 * dk + dv + 1 + dv) + 2 * (2 * dk + 2 * dv + 1 + 2 * dk + dv + 1)
    th = w.B * w.T * w.H
    res = {"workload": w.name, "tokens_per_s": round(w.B * w.T / ((fwd_ms + bwd_ms) / 1e3), 1),
           "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
           "route": "tensor cores (forward keeps chunk states; backward: reverse sweep over them)",
           "step_hbm": {"achieved_gbs": round(step_bytes * th / ((fwd_ms + bwd_ms) / 1e3) / 1e9, 1),
                        "peak_gbs": pk["hbm_gbs"],
                        "frac": round(step_bytes * th / ((fwd_ms + bwd_ms) / 1e3) / 1e9 / pk["hbm_gbs"], 4),
                        "bytes_per_token_head": step_bytes},
           "calls": "hgrn2_scalar_fwd_train + hgrn2_scalar_bwd_saved", "steps": K}
    del g, inp, sv
    torch.cuda.empty_cache()
    return res


def cpu_baseline(inp, w, budget_s=15.0):
    """The oracle (unchanged) on the host cores: fwd+bwd of whole (batch, head) sequences of the workload.

    A first run over `cores` sequences sizes the sample to about `budget_s` seconds of wall time
    (capped at the whole workload)."""
    import oracle
    cores = oracle.num_threads()
    f64 = lambda t: t.to(torch.float64).numpy()

    def run(nbatch):
        sl = lambda t: f64(t[:nbatch].contiguous())
        qq, ll, xx, gg = (sl(inp[k]) for k in ("q", "log_f", "i", "dO"))
        t0 = time.perf_counter()
        oracle.fwd(qq, ll, xx)
        oracle.bwd(qq, ll, xx, gg)
        return time.perf_counter() - t0

    dt1 = run(1)                                  # one batch row = H whole sequences
    nb = max(1, min(w.B, int(budget_s / max(dt1, 1e-3))))
    dt = run(nb) if nb > 1 else dt1
    n = nb * w.H
    tok = nb * w.T                                # tokens of all H heads
    whole = "the whole workload" if nb == w.B else f"{nb} of {w.B} batch rows"
    return {"value": round(tok / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fwd+bwd of {n} whole (batch,head) sequences ({whole}; T={w.T}, d=128), "
                      f"fp64 C oracle, OpenMP over (batch,head); {dt:.2f} s wall",
            "seconds": round(dt, 3)}


def cpu_baseline_others(budget_s=15.0):
    """The oracle (unchanged) on the host cores for the other workloads, each on a bounded sample:
    the forward layer (fwd, B=4, H=8, T=2048) and the long sequence (fwd, B=1, H=8, T=32768,
    h0 in, hT out), whole (batch, head) sequences; the decode workload (B=256, H=16), its first
    decode steps.  Each leg is sized from a first short run to about budget_s / 3 seconds."""
    import oracle
    from linear_attention_hgrn2_b200 import inputs as I
    cores = oracle.num_threads()
    f64 = lambda t: t.to(torch.float64).numpy()
    out = {}
    for w in (I.FWD_LAYER, I.LONG):
        inp = I.make_workload(w, seed=1011)
        def run(nb, nh):
            sl = lambda t: f64(t[:nb, :, :nh].contiguous())
            h0 = f64(inp["h0"][:nb, :nh].contiguous()) if "h0" in inp else None
            t0 = time.perf_counter()
            oracle.fwd(sl(inp["q"]), sl(inp["log_f"]), sl(inp["i"]), h0)
            return time.perf_counter() - t0
        nh = min(w.H, cores)
        dt1 = run(1, nh)
        nb = max(1, min(w.B, int(budget_s / 3 / max(dt1, 1e-3))))
        dt = run(nb, nh) if nb > 1 else dt1
        seqs = nb * nh
        out[w.name] = {"value": round(seqs * w.T / w.H / dt, 2), "unit": "tokens/s", "cores": cores,
                       "kind": "oracle", "seconds": round(dt, 3),
                       "sample": f"fwd of {seqs} whole (batch,head) sequences of {w.B * w.H} (T={w.T}); "
                                 f"tokens/s counts a token as all H heads"}
    cfg = I.DECODE
    S0 = f64(I.decode_state(cfg["B"], cfg["H"], cfg["dk"], cfg["dv"], 1005, cfg["S_sigma"]))
    def steps(n):   # only the oracle's own calls are timed, not the drawing of the tokens
        S, dt = S0, 0.0
        for t in range(n):
            tok = I.decode_token(cfg["B"], cfg["H"], cfg["dk"], cfg["dv"], cfg["dtype"], cfg["lb"], 1005, t)
            a = [f64(tok[k]) for k in ("q", "log_f", "i")]
            t0 = time.perf_counter()
            _, S = oracle.step(*a, S)
            dt += time.perf_counter() - t0
        return dt
    dt1 = steps(2) / 2
    n = max(2, min(cfg["steps"], int(budget_s / 3 / max(dt1, 1e-3))))
    dt = steps(n)
    out[cfg["name"]] = {"value": round(cfg["B"] * n / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                        "ms_per_step": round(dt / n * 1e3, 2), "seconds": round(dt, 3),
                        "sample": f"the first {n} of {cfg['steps']} decode steps, all {cfg['B']}x{cfg['H']} "
                                  f"(batch,head) states (the oracle's calls only)"}
    return out


# ------------------------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The oracle as the reference arm: same metric and config, bounded samples per step, host cores."""
    if rank != 0:
        return
    import oracle
    from linear_attention_hgrn2_b200 import inputs as I
    w = I.TRAIN
    inp = I.make_workload(w, seed=1003)
    f64 = lambda t: t.to(torch.float64).numpy()
    cores = oracle.num_threads()
    heads = max(1, min(w.H, cores))
    sl = lambda t: f64(t[:1, :, :heads].contiguous())
    qq, ll, xx, gg = (sl(inp[k]) for k in ("q", "log_f", "i", "dO"))

    def one():
        oracle.fwd(qq, ll, xx)
        oracle.bwd(qq, ll, xx, gg)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    tok = args.steps * heads * w.T / w.H
    value = tok / dt
    sample = (f"each step: fwd+bwd of {heads} whole (batch,head) sequences (T={w.T}, d=128) of the workload "
              f"on the fp64 C oracle")
    out = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk, "d_v": w.dv,
                      "chunk": w.chunk, "lb": w.lb, "global_batch": w.B, "seq_len": w.T,
                      "parallelism": "host cores (OpenMP over batch,head)"},
           "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-d64", action="store_true")
    ap.add_argument("--no-lb0", action="store_true")
    ap.add_argument("--no-d256", action="store_true")
    ap.add_argument("--no-fwd-configs", action="store_true")
    ap.add_argument("--no-long-train", action="store_true")
    ap.add_argument("--no-scalar", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
