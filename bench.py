#!/usr/bin/env python3
"""Benchmark: causal bf16 attention forward + backward through the C ABI.

One step = one pass of the whole path over one batch: fa_fwd (fused tiled
forward, online softmax, lse) then the backward (row pass, fused recompute
kernel, dQ conversion).  Default workload: B=2, H=16, N=8192, d=128, causal,
no dropout -- the long-context configuration the TFLOPS target is stated for
(N >= 8192, d = 128).  FLOPs follow the attention convention:
4*B*H*N^2*d forward, halved when causal, and 2.5x that backward.

Multi-GPU (torchrun): every rank runs its own copy of the workload (its own
B*H heads; heads are independent, so there is no collective on the data
path) and the job's value is the total FLOPs of all ranks over the slowest
rank's time ("weak" scaling).

``--impl reference`` times the fp64 CPU oracle (the only other
implementation of this path) on the host cores instead, on a bounded sample
of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd and fwd+bwd TFLOPS (bf16, causal) and % of B200 BF16 tensor peak"
DATASHEET_BF16_TFLOPS = 2250.0
LONG_REGION_MS = 1000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# --------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------- traffic record

def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("bwd_sm100.cuh", "fwd_sm100.cuh", "sm100.cuh", "dropout_hash.cuh", "fa_api.cu"):
        with open(os.path.join(ROOT, "io_aware_exact_25_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


# ------------------------------------------------------- oracle (CPU)

def oracle_step(x, w, n_rows: int, mask=None):
    """fp64 oracle forward + full backward on the causal prefix of length
    n_rows of head (b=0, h=0): an exact sub-problem of the workload (causal
    rows < n_rows see only keys < n_rows), with the top-left corner of the
    block mask if there is one.  Returns (seconds, FLOPs)."""
    import oracle
    from io_aware_exact_25_b200.inputs import visible_block_fraction
    q, k, v, do = (x[n][:1, :1, :n_rows].contiguous() for n in ("q", "k", "v", "do"))
    bm = None
    frac = 0.5 if w.causal else 1.0
    if mask is not None:
        nt = (n_rows + 127) // 128
        sub = mask[:1, :nt, :nt].contiguous()
        bm = sub.numpy()
        frac = visible_block_fraction(sub, w.causal)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed, block_mask=bm)
    oracle.backward_q(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed, block_mask=bm)
    oracle.backward_kv(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed, block_mask=bm)
    dt = time.perf_counter() - t0
    f = 4.0 * n_rows * n_rows * w.d * frac
    return dt, 3.5 * f


def varlen_oracle_step(x, w, n_rows: int):
    """fp64 oracle forward + full backward of head 0 of the first sequence of
    a packed variable-length batch, its first n_rows tokens (an exact
    sub-problem under the causal mask).  Returns (seconds, FLOPs)."""
    import oracle
    L0 = min(w.lens[0], n_rows)
    q, k, v, do = (x[n][:L0, :1].transpose(0, 1).unsqueeze(0).contiguous() for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    oracle.backward_q(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    oracle.backward_kv(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    dt = time.perf_counter() - t0
    return dt, 3.5 * 4.0 * L0 * L0 * w.d * (0.5 if w.causal else 1.0)


def oracle_full(x, w):
    """fp64 oracle forward + full backward on every head and row of the
    workload.  Returns (seconds, FLOPs by the attention convention)."""
    import oracle
    q, k, v, do = (x[n] for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    oracle.backward_q(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    oracle.backward_kv(q, k, v, do, w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed)
    return time.perf_counter() - t0, w.fwd_flops() + w.bwd_flops()


def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from io_aware_exact_25_b200.inputs import workload_inputs
    import oracle
    x = workload_inputs(w)
    n_rows = min(args.ref_rows, w.lens[0] if w.lens else w.N)
    full = args.ref_full and not w.lens
    if w.lens:
        step = lambda: varlen_oracle_step(x, w, n_rows)
    else:
        step = (lambda: oracle_full(x, w)) if full else (lambda: oracle_step(x, w, n_rows))
    for _ in range(args.warmup):
        step()
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, f = step()
        tot_t += dt
        tot_f += f
    value = tot_f / tot_t / 1e12
    sample = (f"per step: fwd+bwd of the whole workload ({w.B * w.H} heads x {w.N} rows)" if full else
              f"per step: fwd+bwd of the {'causal ' if w.causal else ''}prefix N={n_rows} of head (0,0)"
              + (" (sequence 0 of the packed batch)" if w.lens else ""))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if not full:
        # the prefix is an exact sub-problem whose work grows as n^2; the whole
        # workload is B*H heads of length N
        lens = w.lens or (w.N,) * w.B
        line["extrapolated_full_problem_s"] = (tot_t / args.steps) * w.H * sum((L / n_rows) ** 2 for L in lens)
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, mask_kind=None, frac=None):
    if w.lens:
        T = sum(w.lens)
        tensor_mib = T * w.H * w.d * 2 / 2 ** 20
        return {"workload": f"{w.name}: {w.B} sequences of {min(w.lens)}-{max(w.lens)} tokens (total {T}) packed "
                            f"token-major, H={w.H} d={w.d} {'causal' if w.causal else 'non-causal'} "
                            f"dropout={w.p_drop} bf16",
                "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "dropout_p": w.p_drop,
                "lens": list(w.lens), "total_tokens": T,
                "l2": f"inputs larger than L2 (Q, K, V, dO: 4 x {tensor_mib:.0f} MiB per step > 126 MB L2)",
                "parallelism": "replicas: each GPU runs its own batch, no collective"}
    tensor_mib = w.B * w.H * w.N * w.d * 2 / 2 ** 20
    cfg = {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} "
                       f"{'causal' if w.causal else 'non-causal'} dropout={w.p_drop} bf16",
           "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "dropout_p": w.p_drop,
           "l2": (f"inputs larger than L2 (Q, K, V, dO: 4 x {tensor_mib:.0f} MiB per step > 126 MB L2)"
                  if 4 * tensor_mib > 126 else
                  f"inputs ({4 * tensor_mib:.0f} MiB) fit in L2: no flush between steps"),
           "parallelism": "replicas: each GPU runs its own B*H heads, no collective"}
    if mask_kind:
        cfg["block_mask"] = mask_kind
        cfg["visible_block_fraction"] = frac
        cfg["workload"] += f" block-sparse {mask_kind} ({100 * frac:.1f}% of dense non-causal work)"
    return cfg


# ------------------------------------------------------------ our arm

def pipelined_e2e(dev, stream, x, d_in0, d_out0, compute, steps, barrier):
    """End to end through the public API: every step copies its inputs from
    pinned host memory to the device, runs ``compute(inputs, outputs,
    stream)`` and copies every result back.  Uploads, compute and downloads
    run on three streams over two sets of device buffers, so step k+1's
    upload and step k-1's download overlap step k's compute (the PCIe link is
    full duplex).  Returns (ms for ``steps`` steps, H2D and D2H bytes a step)."""
    import torch
    h_in = {n: x[n].pin_memory() for n in d_in0}
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    nbuf = 2
    d_in = [d_in0] + [{n: torch.empty_like(t) for n, t in d_in0.items()} for _ in range(nbuf - 1)]
    d_out = [d_out0] + [{n: torch.empty_like(t) for n, t in d_out0.items()} for _ in range(nbuf - 1)]
    h_out = [{n: torch.empty_like(t, device="cpu").pin_memory() for n, t in d_out0.items()} for _ in range(nbuf)]
    d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_cmp = stream
    ev_up, ev_cmp, ev_dn = ([torch.cuda.Event() for _ in range(nbuf)] for _ in range(3))
    for evs, st in ((ev_up, s_up), (ev_cmp, s_cmp), (ev_dn, s_dn)):
        for e in evs:
            e.record(st)

    def step(kstep):
        bi = kstep % nbuf
        din, dout, hout = d_in[bi], d_out[bi], h_out[bi]
        s_up.wait_event(ev_cmp[bi])  # step k-2 finished reading these inputs
        with torch.cuda.stream(s_up):
            for n, h in h_in.items():
                din[n].copy_(h, non_blocking=True)
        ev_up[bi].record(s_up)
        s_cmp.wait_event(ev_up[bi])
        s_cmp.wait_event(ev_dn[bi])  # step k-2's results are on the host
        compute(din, dout, s_cmp)
        ev_cmp[bi].record(s_cmp)
        s_dn.wait_event(ev_cmp[bi])
        with torch.cuda.stream(s_dn):
            for n, t in dout.items():
                hout[n].copy_(t, non_blocking=True)
        ev_dn[bi].record(s_dn)

    for kstep in range(3):
        step(kstep)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for kstep in range(steps):
        step(kstep)
    e1.record(s_dn)  # the last download follows every upload and every compute
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1), h2d, d2h


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)

    from io_aware_exact_25_b200 import binding
    from io_aware_exact_25_b200.inputs import workload_inputs
    lib = binding.load()

    x = workload_inputs(w)
    B, H, N, d = w.B, w.H, w.N, w.d
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    mask_cpu, mask, frac = None, None, None
    if args.block_mask:
        from io_aware_exact_25_b200.inputs import block_mask, visible_block_fraction
        mask_cpu = block_mask(args.block_mask, H, N, seed=w.seed)
        mask = mask_cpu.to(dev)
        frac = visible_block_fraction(mask_cpu, w.causal)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = binding.bwd_workspace_size(B, H, N, d)
    work = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    causal = int(w.causal)
    P = binding._ptr

    def check(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {binding.strerror(rc)}")

    splits = args.splitkv if args.splitkv > 0 else (lib.fa_splitkv_suggest(B, H, N, d) if args.splitkv < 0 else 1)
    split_ws_bytes = int(lib.fa_fwd_splitkv_workspace_size(B, H, N, d, splits)) if splits > 1 else 0
    split_ws = torch.empty(max(split_ws_bytes, 16), dtype=torch.uint8, device=dev)

    def fwd():
        if mask is not None:
            check(lib.fa_fwd_blocksparse(P(q), P(k), P(v), P(o), P(lse), None, B, H, N, d, w.scale, causal, w.p_drop,
                                         w.seed, P(mask), H, s), "fa_fwd_blocksparse")
        elif splits > 1:
            check(lib.fa_fwd_splitkv(P(q), P(k), P(v), P(o), P(lse), B, H, N, d, w.scale, causal, w.p_drop, w.seed,
                                     splits, P(split_ws), split_ws_bytes, s), "fa_fwd_splitkv")
        else:
            check(lib.fa_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, N, d, w.scale, causal, w.p_drop, w.seed, s),
                  "fa_fwd")

    def bwd_prepare():
        check(lib.fa_bwd_prepare(P(o), P(do), P(lse), B, H, N, d, P(work), wsb, s), "fa_bwd_prepare")

    def bwd_recompute():
        if mask is not None:
            check(lib.fa_bwd_recompute_blocksparse(P(q), P(k), P(v), P(do), P(dk), P(dv), B, H, N, d, w.scale, causal,
                                                   w.p_drop, w.seed, P(mask), H, P(work), wsb, s),
                  "fa_bwd_recompute_blocksparse")
            return
        check(lib.fa_bwd_recompute(P(q), P(k), P(v), P(do), P(dk), P(dv), B, H, N, d, w.scale, causal,
                                   w.p_drop, w.seed, P(work), wsb, s), "fa_bwd_recompute")

    def bwd_finalize():
        check(lib.fa_bwd_finalize(P(dq), B, H, N, d, w.scale, P(work), wsb, s), "fa_bwd_finalize")

    stages = [("fwd_kernel", fwd), ("bwd_pre_kernel", bwd_prepare), ("bwd_kernel", bwd_recompute),
              ("bwd_post_kernel", bwd_finalize)]

    def barrier():
        if ws > 1:
            dist.barrier()

    # warm-up (untimed)
    for _ in range(args.warmup):
        for _, fn in stages:
            fn()
    torch.cuda.synchronize(dev)
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error during warm-up")

    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    time.sleep(0.3)

    # device-timed region: events between the stage launches on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for st in range(args.steps):
        ev[st][0].record(stream)
        for i, (name, fn) in enumerate(stages):
            if args.nvtx:
                torch.cuda.nvtx.range_push(name)
            fn()
            if args.nvtx:
                torch.cuda.nvtx.range_pop()
            ev[st][i + 1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    per_stage_ms = [sum(ev[st][i].elapsed_time(ev[st][i + 1]) for st in range(args.steps)) / args.steps
                    for i in range(len(stages))]
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error in the timed region")

    if args.no_extras:
        if rank == 0:
            ffp = w.fwd_flops() if frac is None else 4.0 * B * H * N * N * d * frac
            print(json.dumps({"profiling_run": True, "workload": w.name, "splitkv": splits,
                              "block_mask": args.block_mask,
                              "fwd_tflops": ffp / (per_stage_ms[0] * 1e-3) / 1e12,
                              "ms_per_step": elapsed_ms / args.steps,
                              "stage_ms": dict(zip([n for n, _ in stages], per_stage_ms))}), flush=True)
        if ws > 1:
            dist.destroy_process_group()
        return 0

    # end to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs binding.fwd + binding.bwd and
    # copies every result back.  Uploads, compute and downloads run on three
    # streams over two sets of device buffers, so step k+1's upload and step
    # k-1's download overlap step k's compute (the PCIe link is full duplex).
    def compute(din, dout, st):
        binding.fwd(din["q"], din["k"], din["v"], causal=w.causal, scale=w.scale, dropout_p=w.p_drop, seed=w.seed,
                    o=dout["o"], lse=dout["lse"], block_mask=mask, stream=st)
        binding.bwd(din["q"], din["k"], din["v"], dout["o"], din["do"], dout["lse"], causal=w.causal, scale=w.scale,
                    dropout_p=w.p_drop, seed=w.seed, dq=dout["dq"], dk=dout["dk"], dv=dout["dv"], workspace=work,
                    block_mask=mask, stream=st)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = pipelined_e2e(dev, stream, x, {"q": q, "k": k, "v": v, "do": do},
                                     {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}, compute, e2e_steps, barrier)
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error in the end-to-end run")

    # every replica checks its own outputs with identities that hold at any
    # size (sum_j dK_j = 0 and, without dropout, sum_j dV_j = sum_i dO_i, in
    # fp32 sums of the bf16 outputs; everything finite), then the job takes
    # the slowest rank's times and the AND of the checks
    ok = bool(torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()
              and torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all())
    if mask is None:
        sdk = dk.float().sum(dim=2)
        ok = ok and bool((sdk.abs() <= 1e-2 * dk.float().abs().sum(dim=2) + 1e-2).all())
        if w.p_drop == 0.0:
            sdv, sdo = dv.float().sum(dim=2), do.float().sum(dim=2)
            ok = ok and bool(((sdv - sdo).abs() <= 1e-2 * dv.float().abs().sum(dim=2) + 1e-2).all())
    from io_aware_exact_25_b200.replicas import replica_summary
    summ = replica_summary(elapsed_ms, e2e_ms, per_stage_ms, ok, device=dev)
    elapsed_ms, e2e_ms, per_stage_ms = summ["elapsed_ms"], summ["e2e_ms"], summ["stage_ms"]
    if not summ["all_ok"]:
        raise RuntimeError("a replica's outputs failed their checks")

    if rank == 0:
        ff, fb = w.fwd_flops(), w.bwd_flops()
        if frac is not None:
            # block-sparse: FLOPs of the visible blocks only (diagonal blocks
            # count half under the causal mask)
            ff = 4.0 * B * H * N * N * d * frac
            fb = 2.5 * ff
        ms_step = elapsed_ms / args.steps
        value = ws * (ff + fb) / (ms_step * 1e-3) / 1e12
        fwd_ms = per_stage_ms[0]
        bwd_ms = sum(per_stage_ms[1:])
        peaks, peak_kind = load_peaks()
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        # a timed region under a second runs at burst clocks; a seconds-long
        # loop settles under the power cap at the sustained figure
        long_region = elapsed_ms >= LONG_REGION_MS
        roof_peak = sustained if long_region else burst
        roof_peak_name = "bf16_tflops_sustained" if long_region else "bf16_tflops (burst)"
        # dominant kernel: the largest share of the step
        names = [n for n, _ in stages]
        dom = max(range(len(stages)), key=lambda i: per_stage_ms[i])
        dom_flops = {0: ff, 2: fb}.get(dom)
        tensor_bytes = B * H * N * d * 2
        row_bytes = B * H * N * 4
        # algorithmic HBM bytes per launch: each input read once, each output
        # written once (the fp32 dQ accumulator's one read+write round trip is
        # listed separately)
        alg_bytes = {0: 4 * tensor_bytes + row_bytes, 2: 6 * tensor_bytes + 2 * row_bytes}.get(dom)
        if dom_flops is not None:
            achieved = dom_flops / (per_stage_ms[dom] * 1e-3) / 1e12
            traffic = recorded_traffic(names[dom], w.name) if mask is None else None
            roof = {"bound": "tensor", "kernel": names[dom], "achieved": achieved, "peak": roof_peak,
                    "unit": "TFLOP/s", "frac": achieved / roof_peak,
                    "peak_note": f"{roof_peak_name} of {peak_kind} MEASURED_PEAKS.json: the timed region is "
                                 f"{elapsed_ms:.1f} ms ({'>=' if long_region else '<'} {LONG_REGION_MS / 1e3:g} s)",
                    "timed_region_ms": elapsed_ms,
                    "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
                    "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS,
                    "traffic": traffic,
                    "traffic_source": (f"dram__bytes_read.sum + dram__bytes_write.sum of one launch, committed "
                                       f"ncu summary profiles/{names[dom]}_{w.name}.md (same kernel sources)"
                                       if traffic is not None else None),
                    "algorithmic_flops_per_launch": dom_flops,
                    "hbm": {"algorithmic_bytes_per_launch": alg_bytes,
                            "algorithmic_gbs": alg_bytes / (per_stage_ms[dom] * 1e-3) / 1e9,
                            "dram_gbs_at_event_time": (traffic / (per_stage_ms[dom] * 1e-3) / 1e9
                                                       if traffic is not None else None),
                            "peak_gbs": hbm_peak,
                            "dq_accumulator_round_trip_bytes": 2 * B * H * N * d * 4 if dom == 2 else 0,
                            "materialised_s_bytes": 2 * B * H * N * N * 4}}
        else:
            roof = {"bound": "hbm", "kernel": names[dom], "achieved": None, "peak": None, "unit": "GB/s",
                    "frac": None, "traffic": None}
        # oracle baseline on the host cores (bounded sample of the same workload)
        import oracle
        cpu_rows = min(args.cpu_rows, N)
        cpu_dt, cpu_f, reps = 0.0, 0.0, 0
        while reps < 20 and (reps == 0 or cpu_dt < args.cpu_seconds):
            dt_, f_ = oracle_step(x, w, cpu_rows, mask_cpu)
            cpu_dt, cpu_f, reps = cpu_dt + dt_, cpu_f + f_, reps + 1
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, args.block_mask, frac),
            "fwd_tflops": ws * ff / (fwd_ms * 1e-3) / 1e12,
            "fwd_bwd_tflops": value,
            "frac_of_peak": {
                "fwd_vs_burst": (ff / (fwd_ms * 1e-3) / 1e12) / burst,
                "fwd_bwd_vs_burst": (value / ws) / burst,
                "fwd_vs_datasheet": (ff / (fwd_ms * 1e-3) / 1e12) / DATASHEET_BF16_TFLOPS,
                "fwd_bwd_vs_datasheet": (value / ws) / DATASHEET_BF16_TFLOPS,
                "fwd_vs_sustained": (ff / (fwd_ms * 1e-3) / 1e12) / sustained,
                "fwd_bwd_vs_sustained": (value / ws) / sustained,
                "peaks": f"{peak_kind}: burst {burst}, sustained {sustained}, datasheet {DATASHEET_BF16_TFLOPS}"},
            "stage_ms": dict(zip(names, per_stage_ms)),
            "roofline": roof,
            "cpu_baseline": {"value": cpu_f / cpu_dt / 1e12, "unit": "TFLOPS", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"{reps} x fp64 fwd+bwd of the {'causal ' if w.causal else ''}prefix N={cpu_rows} of head (0,0)"
                                       f"{' with its block mask corner' if mask is not None else ''} "
                                       f"({cpu_dt:.1f} s)"},
            "e2e": {"value": ws * (ff + fb) * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "binding.fwd/binding.bwd (C ABI) with pinned host buffers; uploads, compute and "
                           "downloads on three streams over two device buffer sets"},
            "gpu_launches": args.steps * (len(stages) + (1 if splits > 1 else 0)),
            "splitkv": splits,
            "replica_checks": {"ranks": ws, "all_ok": summ["all_ok"],
                               "checks": "finite outputs; sum_j dK_j = 0; sum_j dV_j = sum_i dO_i without dropout"},
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ours_varlen(args, w):
    """One step = fa_fwd_varlen + fa_bwd_varlen over a packed variable-length
    batch; FLOPs summed over the sequences (Workload.fwd_flops)."""
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    from io_aware_exact_25_b200 import binding
    from io_aware_exact_25_b200.inputs import workload_inputs
    lib = binding.load()
    x = workload_inputs(w)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    cu = x["cu_seqlens"].to(dev)
    T, H, d = q.shape
    B, maxs = w.B, w.N
    o = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = int(lib.fa_bwd_varlen_workspace_size(B, H, maxs, d))
    work = torch.empty(wsb, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev).cuda_stream
    P = binding._ptr
    S4 = binding._tok_strides(q, k, v, o)
    S8 = binding._tok_strides(q, k, v, o, do, dq, dk, dv)
    causal = int(w.causal)

    def check(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {binding.strerror(rc)}")

    def fwd():
        check(lib.fa_fwd_varlen(P(q), P(k), P(v), P(o), P(lse), S4, P(cu), None, B, H, maxs, T, d, w.scale, causal,
                                w.p_drop, w.seed, s), "fa_fwd_varlen")

    def bwd():
        check(lib.fa_bwd_varlen(P(q), P(k), P(v), P(o), P(do), P(lse), P(dq), P(dk), P(dv), S8, P(cu), None, B, H,
                                maxs, T, d, w.scale, causal, w.p_drop, w.seed, P(work), wsb, s), "fa_bwd_varlen")

    # fa_bwd_varlen launches bwd_pre_kernel, bwd_kernel and bwd_post_kernel
    stages = [("fwd_kernel", fwd), ("bwd_pre_kernel + bwd_kernel + bwd_post_kernel", bwd)]
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        for _, fn in stages:
            fn()
    torch.cuda.synchronize(dev)
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error during warm-up")
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for st in range(args.steps):
        ev[st][0].record(stream)
        for i, (name, fn) in enumerate(stages):
            if args.nvtx:
                torch.cuda.nvtx.range_push(name)
            fn()
            if args.nvtx:
                torch.cuda.nvtx.range_pop()
            ev[st][i + 1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    stage_ms = [sum(ev[st][i].elapsed_time(ev[st][i + 1]) for st in range(args.steps)) / args.steps
                for i in range(len(stages))]
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error in the timed region")
    ok = bool(torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()
              and torch.isfinite(dv.float()).all())
    # per sequence and head: sum_j dK_j = 0 and, without dropout, sum_j dV_j = sum_i dO_i
    seg = torch.repeat_interleave(torch.arange(B, device=dev), torch.tensor(w.lens, device=dev))

    def seg_sum(t):
        return torch.zeros((B, H, d), dtype=torch.float32, device=dev).index_add_(0, seg, t.float())

    ok = ok and bool((seg_sum(dk).abs() <= 1e-2 * seg_sum(dk.abs()) + 1e-2).all())
    if w.p_drop == 0.0:
        ok = ok and bool(((seg_sum(dv) - seg_sum(do)).abs() <= 1e-2 * seg_sum(dv.abs()) + 1e-2).all())
    # end to end through the public API, inputs from and results to pinned
    # host memory (the same three-stream pipeline as the dense path)
    def compute(din, dout, st):
        binding.fwd_varlen(din["q"], din["k"], din["v"], cu, maxs, causal=w.causal, scale=w.scale,
                           dropout_p=w.p_drop, seed=w.seed, o=dout["o"], lse=dout["lse"], stream=st)
        binding.bwd_varlen(din["q"], din["k"], din["v"], dout["o"], din["do"], dout["lse"], cu, maxs,
                           causal=w.causal, scale=w.scale, dropout_p=w.p_drop, seed=w.seed, dq=dout["dq"],
                           dk=dout["dk"], dv=dout["dv"], workspace=work, stream=st)

    def barrier():
        if ws > 1:
            dist.barrier()

    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = pipelined_e2e(dev, stream, x, {"q": q, "k": k, "v": v, "do": do},
                                     {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}, compute, e2e_steps, barrier)
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error in the end-to-end run")
    from io_aware_exact_25_b200.replicas import replica_summary
    summ = replica_summary(elapsed_ms, e2e_ms, stage_ms, ok, device=dev)
    if not summ["all_ok"]:
        raise RuntimeError("a replica's outputs failed their checks")
    if rank == 0:
        ff, fb = w.fwd_flops(), w.bwd_flops()
        ms_step = summ["elapsed_ms"] / args.steps
        value = ws * (ff + fb) / (ms_step * 1e-3) / 1e12
        peaks, peak_kind = load_peaks()
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        long_region = summ["elapsed_ms"] >= LONG_REGION_MS
        roof_peak = sustained if long_region else burst
        fwd_ms, bwd_ms = summ["stage_ms"]
        dom = 0 if fwd_ms > bwd_ms else 1
        dom_flops = ff if dom == 0 else fb
        achieved = dom_flops / ((fwd_ms if dom == 0 else bwd_ms) * 1e-3) / 1e12
        # the CPU baseline: the oracle on the first sequence of the batch, head 0
        import oracle
        L0 = min(w.lens[0], args.cpu_rows)
        cpu_dt, cpu_f = varlen_oracle_step(x, w, L0)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w),
            "fwd_tflops": ws * ff / (fwd_ms * 1e-3) / 1e12, "fwd_bwd_tflops": value,
            "frac_of_peak": {"fwd_vs_burst": (ff / (fwd_ms * 1e-3) / 1e12) / burst,
                             "fwd_bwd_vs_burst": (value / ws) / burst,
                             "fwd_bwd_vs_datasheet": (value / ws) / DATASHEET_BF16_TFLOPS,
                             "peaks": f"{peak_kind}: burst {burst}, sustained {sustained}"},
            "stage_ms": dict(zip([n for n, _ in stages], summ["stage_ms"])),
            "roofline": {"bound": "tensor", "kernel": stages[dom][0], "achieved": achieved, "peak": roof_peak,
                         "unit": "TFLOP/s", "frac": achieved / roof_peak,
                         "peak_note": f"{'bf16_tflops_sustained' if long_region else 'bf16_tflops (burst)'} of "
                                      f"{peak_kind}: the timed region is {summ['elapsed_ms']:.1f} ms",
                         "traffic": None, "algorithmic_flops_per_launch": dom_flops},
            "cpu_baseline": {"value": cpu_f / cpu_dt / 1e12, "unit": "TFLOPS", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"fp64 fwd+bwd of sequence 0 (first {L0} tokens), head 0 ({cpu_dt:.1f} s)"},
            "e2e": {"value": ws * (ff + fb) * e2e_steps / (summ["e2e_ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "binding.fwd_varlen/binding.bwd_varlen (C ABI) with pinned host buffers; uploads, "
                           "compute and downloads on three streams over two device buffer sets"},
            "gpu_launches": args.steps * (1 + 3),
            "replica_checks": {"ranks": ws, "all_ok": summ["all_ok"],
                               "checks": "finite outputs; per sequence and head sum_j dK_j = 0 and "
                                         "sum_j dV_j = sum_i dO_i"},
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


NVLINK_GBS = 770.0  # measured peer copy per direction on this machine's B200s (nominal 900)


def run_seqpar_emulated(args, w):
    """``--seqpar W``: the sequence-parallel path of io_aware_exact_25_b200.seqpar
    with its W ranks played in turn on one GPU ("FlashAttention for Efficient
    Training", section 5.3).  Rank r holds the key window key_windows(N, W,
    causal)[r]; a step is, per rank, fa_fwd_partial over its window (and, with
    the summed exchange, fa_weight_partial on its piece) and
    fa_bwd_recompute_range over it, plus the work every rank repeats on the
    whole sequence -- fa_merge_partials (of all pieces, or the one-piece
    conversion of the sum), fa_bwd_prepare, fa_bwd_finalize -- timed once.
    The ranks share one backward workspace, so the dQ accumulator ends up
    holding the sum the NCCL all-reduce would form, and a torch sum of the
    weighted pieces stands in for the forward's all-reduce: the outputs are
    the whole problem's.  Every launch is timed with CUDA events; a rank's
    time is its own launches plus the repeated ones.  The exchanges do not
    happen on one GPU: their bytes are counted and converted to a time at
    the measured NVLink copy rate, as a model, not a measurement (the stand-in
    sum's own time is reported beside it and counted in no rank)."""
    import torch

    ws, rank, local = dist_env()
    if ws > 1:
        raise SystemExit("--seqpar plays every rank on one GPU: run it without torchrun")
    if w.lens:
        raise SystemExit("--seqpar takes a dense workload")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from io_aware_exact_25_b200 import binding
    from io_aware_exact_25_b200.inputs import workload_inputs
    from io_aware_exact_25_b200.seqpar import key_windows, tile_work

    W = args.seqpar
    x = workload_inputs(w)
    B, H, N, d = w.B, w.H, w.N, w.d
    # "work": the causal split that balances the ranks; "even": equal tile counts
    windows = key_windows(N, W, w.causal and args.seqpar_split == "work")
    q, do = x["q"].to(dev), x["do"].to(dev)
    kw = [x["k"][:, :, a:b].contiguous().to(dev) for a, b in windows]
    vw = [x["v"][:, :, a:b].contiguous().to(dev) for a, b in windows]
    part_o = torch.empty((W, B, H, N, d), dtype=torch.float32, device=dev)
    part_lse = torch.empty((W, B, H, N), dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq = torch.empty_like(q)
    dk = [torch.empty_like(t) for t in kw]
    dv = [torch.empty_like(t) for t in vw]
    work = torch.empty(binding.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kwargs = dict(causal=w.causal, scale=w.scale, dropout_p=w.p_drop, seed=w.seed)

    # (name, rank / None for the work every rank repeats / "exchange", launch)
    launches = []
    for r, (a, b) in enumerate(windows):
        launches.append(("fa_fwd_partial", r, lambda r=r, a=a: binding.fwd_partial(
            q, kw[r], vw[r], a, part_o=part_o[r], part_lse=part_lse[r], **kwargs)))
    if args.seqpar_exchange == "sum":
        # part_lse stacked is what the lse all-gather delivers; the torch sum
        # stands in for the all-reduce of the weighted pieces (not a rank's
        # kernel time: the exchange)
        lse_w = torch.empty_like(lse)
        o_sum = torch.empty((B, H, N, d), dtype=torch.float32, device=dev)
        for r in range(W):
            launches.append(("fa_weight_partial", r, lambda r=r: binding.weight_partial(
                part_o[r], part_lse, r, lse=lse_w)))
        launches.append(("all-reduce stand-in", "exchange", lambda: torch.sum(part_o, dim=0, out=o_sum)))
        launches.append(("fa_merge_partials", None, lambda: binding.merge_partials(
            o_sum.unsqueeze(0), lse_w.unsqueeze(0), o=o, lse=lse)))
    else:
        launches.append(("fa_merge_partials", None, lambda: binding.merge_partials(part_o, part_lse, o=o, lse=lse)))
    launches.append(("fa_bwd_prepare", None, lambda: binding.bwd_prepare(o, do, lse, work)))
    for r, (a, b) in enumerate(windows):
        if b > a:
            launches.append(("fa_bwd_recompute_range", r, lambda r=r, a=a: binding.bwd_recompute_range(
                q, kw[r], vw[r], do, a, work, dk=dk[r], dv=dv[r], **kwargs)))
    launches.append(("fa_bwd_finalize", None, lambda: binding.bwd_finalize(dq, work, w.scale)))

    for _ in range(args.warmup):
        for _, _, fn in launches:
            fn()
    torch.cuda.synchronize(dev)
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error during warm-up")

    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)] for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for st in range(args.steps):
        ev[st][0].record(stream)
        for i, (_, _, fn) in enumerate(launches):
            fn()
            ev[st][i + 1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if binding.device_error(stream) != 0:
        raise RuntimeError("kernel reported a device error in the timed region")
    ms = [sum(ev[st][i].elapsed_time(ev[st][i + 1]) for st in range(args.steps)) / args.steps
          for i in range(len(launches))]
    step_ms = sum(ev[st][0].elapsed_time(ev[st][-1]) for st in range(args.steps)) / args.steps

    # the whole problem's identities hold for the assembled outputs
    dk_all, dv_all = torch.cat(dk, dim=2).float(), torch.cat(dv, dim=2).float()
    ok = bool(torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()
              and torch.isfinite(dk_all).all() and torch.isfinite(dv_all).all())
    ok = ok and bool((dk_all.sum(dim=2).abs() <= 1e-2 * dk_all.abs().sum(dim=2) + 1e-2).all())
    if w.p_drop == 0.0:
        sdo = do.float().sum(dim=2)
        ok = ok and bool(((dv_all.sum(dim=2) - sdo).abs() <= 1e-2 * dv_all.abs().sum(dim=2) + 1e-2).all())
    if not ok:
        raise RuntimeError("the assembled outputs failed their checks")

    shared_ms = sum(m for (_, r, _), m in zip(launches, ms) if r is None)
    stand_in_ms = sum(m for (_, r, _), m in zip(launches, ms) if r == "exchange")
    rank_ms = [shared_ms + sum(m for (_, rr, _), m in zip(launches, ms) if rr == r) for r in range(W)]
    nt = (N + 127) // 128
    tw = tile_work(nt, w.causal)
    rank_steps = [sum(tw[a // 128:(b + 127) // 128]) for a, b in windows]
    ff, fb = w.fwd_flops(), w.bwd_flops()
    # per rank, received: the forward's other pieces (fp32 O and lse) for the
    # gather, or their lse plus a ring all-reduce of the fp32 weighted piece
    # (2 (W-1)/W of it) for the sum; the backward's ring all-reduce of the
    # fp32 dQ accumulator
    ring = 2 * (W - 1) / W
    if args.seqpar_exchange == "sum":
        fwd_bytes = int((W - 1) * B * H * N * 4 + ring * B * H * N * d * 4)
    else:
        fwd_bytes = (W - 1) * B * H * N * (d + 1) * 4
    bwd_bytes = int(ring * B * H * N * d * 4)
    model_ms = (fwd_bytes + bwd_bytes) / (NVLINK_GBS * 1e9) * 1e3
    peaks, peak_kind = load_peaks()
    by_name = {}
    for (name, _, _), m in zip(launches, ms):
        by_name[name] = by_name.get(name, 0.0) + m
    line = {
        "metric": METRIC, "value": (ff + fb) / (step_ms * 1e-3) / 1e12, "unit": "TFLOPS", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w), parallelism=f"sequence parallel over {W} key windows, the ranks "
                                                       f"played in turn on one GPU"),
        "seqpar": {
            "world": W, "split": args.seqpar_split, "exchange": args.seqpar_exchange, "windows": windows,
            "rank_work_steps": rank_steps,
            "rank_ms": rank_ms, "max_rank_ms": max(rank_ms), "mean_rank_ms": sum(rank_ms) / W,
            "balance_max_over_mean": max(rank_ms) / (sum(rank_ms) / W),
            "repeated_per_rank_ms": shared_ms, "launch_ms_by_entry_point": by_name,
            "rank_compute_tflops": (ff + fb) / (max(rank_ms) * 1e-3) / 1e12,
            "rank_compute_note": "whole-problem FLOPs over the slowest rank's kernel time: what W GPUs would "
                                 "reach if the exchanges were free (a projection from one GPU)",
            "exchange_bytes_per_rank": {"forward": fwd_bytes, "backward_dq_all_reduce": bwd_bytes},
            "all_reduce_stand_in_ms": stand_in_ms,
            "exchange_model_ms": model_ms,
            "exchange_model_note": f"bytes / {NVLINK_GBS:g} GB/s measured NVLink peer copy; not measured here "
                                   f"(one GPU)"},
        "e2e": None, "cpu_baseline": None,
        "gpu_launches": args.steps * sum(1 for _, r, _ in launches if r != "exchange"),
        "peaks": f"{peak_kind} MEASURED_PEAKS.json",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long8k_causal")
    ap.add_argument("--cpu-rows", type=int, default=8192,
                    help="causal prefix length of the oracle baseline sample")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="repeat the oracle baseline sample until it has run this long (at most 20 times)")
    ap.add_argument("--splitkv", type=int, default=0,
                    help="forward with fa_fwd_splitkv: number of splits (-1: suggested, 0: plain kernel)")
    ap.add_argument("--block-mask", default=None,
                    help="block-sparse run with this synthetic block mask, e.g. 'local:4,global:2' or "
                         "'random:0.25' (io_aware_exact_25_b200.inputs.block_mask)")
    ap.add_argument("--seqpar", type=int, default=0,
                    help="time the sequence-parallel path of this many ranks, played in turn on one GPU")
    ap.add_argument("--seqpar-split", choices=["work", "even"], default="work",
                    help="--seqpar key windows: balanced by causal work, or equal tile counts")
    ap.add_argument("--seqpar-exchange", choices=["sum", "gather"], default="sum",
                    help="--seqpar forward exchange: weighted pieces summed, or whole pieces gathered and merged")
    ap.add_argument("--nvtx", action="store_true",
                    help="wrap each stage launch of the timed region in an NVTX range (for profiler timelines)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the end-to-end and CPU-baseline legs (profiling runs)")
    ap.add_argument("--ref-rows", type=int, default=1024,
                    help="causal prefix length per step of the reference (oracle) arm")
    ap.add_argument("--ref-full", action="store_true",
                    help="reference arm: time the oracle on the whole workload (small workloads only)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.block_mask and args.splitkv:
        ap.error("--block-mask and --splitkv are separate forward variants")
    from io_aware_exact_25_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.seqpar:
        if args.seqpar < 1 or args.block_mask or args.splitkv:
            ap.error("--seqpar takes a rank count >= 1 and no other forward variant")
        return run_seqpar_emulated(args, w)
    if w.lens:
        return run_ours_varlen(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
