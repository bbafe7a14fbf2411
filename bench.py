#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200: one step = forward + backward of the
long-context causal workload (B=2, H=16, N=8192, d=128, bf16), all four library kernels.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  The metric is attention fwd+bwd TFLOP/s with the FLOP count
4*B*H*N^2*d (halved for causal) for the forward and 2.5x that for the backward, and its fraction
of the measured dense-bf16 tensor peak.  Multi-GPU runs (torchrun) give every rank its own batch
of heads (heads are independent: no collective on the data path) and report the whole-job
throughput over the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on the same metric (a bounded sample of the same
workload per step) -- the only other place this file runs the oracle is the ``cpu_baseline`` leg.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import attn_inputs as ai  # noqa: E402

METRIC = "attention fwd/bwd TFLOP/s bf16 at N=8K d=128 causal; % of B200 BF16 peak"
WORKLOAD = dict(B=2, H=16, N=8192, d=128, causal=True)
WORKLOAD_NAME = "long-context causal fwd+bwd, B=2 H=16 N=8192 d=128 bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


class L2Flush:
    """Empties the 126 MB L2 between timed steps, outside the timed events: a 256 MiB buffer is
    written (nothing the next step reads stays cached), then a second 256 MiB buffer is read, so
    that the dirty lines of the write are written back here and not during the next timed
    kernel (which would otherwise pay up to 126 MB of write-back traffic)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def pass_bytes(B, H, Hkv, N, d, forward: bool) -> int:
    """Compulsory HBM bytes of one pass: each input read once and each output written once.
    Forward: Q, K, V in, O (bf16) and L (fp32) out.  Backward main kernel: Q, dO, K, V, L, D in,
    dQ, dK, dV out (the fp32 dQ accumulator's traffic is not counted: it is the kernel's own)."""
    q = B * H * N * d * 2
    kv = B * Hkv * N * d * 2
    rows = B * H * N * 4
    if forward:
        return q + 2 * kv + q + rows
    return 2 * q + 2 * kv + 2 * rows + q + 2 * kv


def binding_roofline(work: float, nbytes: int, avg_ms: float, peaks: dict, peak_src: str) -> dict:
    """Roofline of one attention kernel launch: `work` FLOP and `nbytes` compulsory HBM bytes in
    `avg_ms`.  The binding roof is the one with the longer ideal time -- the FLOPs at the tensor
    peak or the bytes at the copy bandwidth (short sequences are HBM bound, long ones tensor
    bound); the other is reported beside it."""
    t_tensor = work / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    tensor = {"bound": "tensor", "achieved": work / (avg_ms * 1e-3) / 1e12,
              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
              "peak_source": f"{peak_src} bf16_tflops (burst)"}
    tensor["frac"] = tensor["achieved"] / tensor["peak"]
    tensor["frac_of_sustained"] = tensor["achieved"] / peaks.get("bf16_tflops_sustained",
                                                                 tensor["peak"])
    hbm = {"bound": "hbm", "achieved": nbytes / (avg_ms * 1e-3) / 1e9,
           "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs",
           "algorithmic_bytes": nbytes}
    hbm["frac"] = hbm["achieved"] / hbm["peak"]
    roof, other = (hbm, tensor) if t_hbm > t_tensor else (tensor, hbm)
    roof["other_roof"] = {k: other[k] for k in ("bound", "achieved", "unit", "frac")}
    return roof


def flops(B, H, N, d, causal):
    fwd = 4.0 * B * H * N * N * d * (0.5 if causal else 1.0)
    return fwd, 2.5 * fwd


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="fattn", choices=["fattn", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="head chunks of fa_fwd_bwd_host in the end-to-end leg")
    ap.add_argument("--shape", default=None,
                    help="B,H,N,d,causal override (profiling runs on a smaller case)")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="key/value heads per batch (grouped-query attention; default: H)")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per workload: the GPT-2-small and BERT-large shapes and the 30 "
                         "points of the B*H*N = 131072 sweep (fwd+bwd, bf16)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the FP8 (e4m3) forward on the workload instead of the bf16 step")
    ap.add_argument("--decode", default=None,
                    help="B,H,H_kv,Nq,Nk,d[,splits]: time the split-key forward (decoding) instead "
                         "of the headline step; reports HBM throughput")
    args = ap.parse_args(argv)
    global WORKLOAD_NAME
    if args.shape:
        B, H, N, d, c = (int(x) for x in args.shape.split(","))
        WORKLOAD.update(B=B, H=H, N=N, d=d, causal=bool(c))
        WORKLOAD_NAME = f"shape override B={B} H={H} N={N} d={d} causal={bool(c)} (profiling)"
    if args.kv_heads is not None and args.kv_heads != WORKLOAD["H"]:
        if args.kv_heads < 1 or WORKLOAD["H"] % args.kv_heads:
            ap.error("--kv-heads must divide H")
        WORKLOAD["H_kv"] = args.kv_heads
        WORKLOAD_NAME += (f", grouped-query attention: {WORKLOAD['H']} query heads on "
                          f"{args.kv_heads} key/value heads")
    return args


# ---------------------------------------------------------------------------------- ranks
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(backend):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def rank_seed(rank: int) -> int:
    """Every rank draws its own batch (weak scaling: per-GPU work fixed as N grows)."""
    return 1000 + rank


def reduce_max(x: float, device=None) -> float:
    """Max over ranks (timing is the slowest rank's device time)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms while running.

    start() returns once the first sample has been written, so that sampling is live before the
    timed region begins; begin() / end() mark the timed region on the host clock (call them right
    after the synchronize on each side), and stop() keeps the samples whose timestamps fall inside
    it.  A region shorter than the sampling interval may hold none: then the samples nearest to
    it on either side are kept and the result says so ("window": "nearest")."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self, wait_s: float = 5.0):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t_end = time.time() + wait_s
        while time.time() < t_end and self.proc.poll() is None:
            self.out.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(s: str):
        import datetime
        try:
            return datetime.datetime.strptime(s, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append((self._stamp(parts[0]), parts[1:]))
        os.unlink(self.path)
        window = "timed region"
        if self.t0 is not None and self.t1 is not None and all(t is not None for t, _ in rows):
            inside = [r for t, r in rows if self.t0 <= t <= self.t1]
            if not inside:
                before = [r for t, r in rows if t < self.t0][-1:]
                after = [r for t, r in rows if t > self.t1][:1]
                inside = before + after
                window = "nearest"
            rows = inside
        else:
            rows = [r for _, r in rows]
            window = "whole run"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None, "window": window}


# ---------------------------------------------------------------------------------- oracle leg
def oracle_sample(rows: int, seed: int = 0):
    """fp64 oracle fwd+bwd on one head of the workload restricted to its first `rows` positions
    (a causal prefix: a shorter instance of the same computation).  Returns (seconds, flops)."""
    from oracle import attention_backward, attention_forward
    d = WORKLOAD["d"]
    x = ai.make_inputs(1, 1, rows, d, seed=seed)
    f = {k: ai.bf16_bits_to_f64(v) for k, v in x.items()}
    s = ai.default_scale(d)
    t0 = time.perf_counter()
    O, L = attention_forward(f["q"], f["k"], f["v"], True, s)
    attention_backward(f["q"], f["k"], f["v"], O, L, f["do"], True, s)
    dt = time.perf_counter() - t0
    ff, fb = flops(1, 1, rows, d, True)
    return dt, ff + fb


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline():
    dt, fl = oracle_sample(WORKLOAD["N"])
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, forward+backward of 1 of the {WORKLOAD['B'] * WORKLOAD['H']}"
                      f" heads (N=8192, d=128, causal) in {dt:.1f} s; algorithmic FLOPs"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    # size one step so the whole --warmup + --steps run stays within about three minutes
    t_cal, _ = oracle_sample(1024)
    rows = 1024
    for r in (8192, 4096, 2048):
        est = t_cal * (r / 1024) ** 2
        if est * (args.steps + args.warmup) <= 180:
            rows = r
            break
    for _ in range(args.warmup):
        oracle_sample(rows)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(rows)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, **WORKLOAD,
                   "reference_sample": f"1 head, first {rows} positions per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(),
                         "kind": "oracle",
                         "sample": f"fp64 numpy oracle fwd+bwd, 1 head x {rows} positions "
                                   "(causal prefix of the workload) per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------- GPU arm
def kernel_traffic(kernel_name: str, workload: dict):
    """DRAM bytes per launch of `kernel_name` on `workload` from a committed ncu capture, if one
    was taken for that kernel and workload on the current source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f).get("records", [])
    except (OSError, ValueError, AttributeError):
        return None
    for rec in recs:
        if rec.get("kernel") != kernel_name or rec.get("workload") != workload:
            continue
        if rec.get("csrc_sha256") != csrc_code_hash():
            return None
        return rec.get("bytes_per_launch")
    return None


def csrc_code_hash() -> str:
    """sha256 of the CUDA sources with comments removed and whitespace collapsed: a traffic
    record stays valid across comment edits and goes stale with any change to the code."""
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "exact_io_aware_43_b200", "csrc")
    for fn in sorted(os.listdir(d)):
        with open(os.path.join(d, fn), encoding="utf-8") as f:
            txt = f.read()
        txt = re.sub(r"/\*.*?\*/", " ", txt, flags=re.S)
        txt = re.sub(r"//[^\n]*", " ", txt)
        txt = " ".join(txt.split())
        h.update(fn.encode() + b"\0" + txt.encode() + b"\0")
    return h.hexdigest()


def run_gpu(args):
    import torch
    import exact_io_aware_43_b200 as fa

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rank, world = dist_init("nccl")
    W = WORKLOAD
    B, H, N, d, causal = W["B"], W["H"], W["N"], W["d"], W["causal"]
    s = ai.default_scale(d)
    x = ai.make_inputs(B, H, N, d, seed=rank_seed(rank), kv_heads=W.get("H_kv"))
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) for k, v in x.items()}
    q, k, v, do = (host[t].to(dev) for t in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_gqa_workspace_size(B, H, W.get("H_kv", H), N, d), dtype=torch.uint8,
                     device=dev)
    flush = L2Flush(dev)

    def step():
        fa.forward(q, k, v, causal, s, out=o, lse=lse)
        fa.backward(q, k, v, o, lse, do, causal, s, workspace=ws, grads=(dq, dk, dv))

    for _ in range(max(3, args.warmup)):
        flush()
        step()
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0, "a kernel reported a timeout during warm-up"
    for kk in range(4):
        fa.fa_timer_read(kk)  # discard anything recorded before the timed region

    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize()
    sampler.begin()
    fa.fa_timer_enable(True)
    for i in range(args.steps):
        flush()  # L2 flushed before every step, outside the timed events
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    sampler.end()
    fa.fa_timer_enable(False)
    barrier(dev)
    clocks = sampler.stop()
    status = fa.fa_device_status()
    ms_local = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    ktimes = {kk: fa.fa_timer_read(kk) for kk in range(4)}
    ms = reduce_max(ms_local, dev)

    ff, fb = flops(B, H, N, d, causal)
    value = world * (ff + fb) / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    fwd_ms = ktimes[fa.FA_KERNEL_FWD][1] / max(1, ktimes[fa.FA_KERNEL_FWD][0])
    bwd_ms = sum(ktimes[kk][1] for kk in (1, 2, 3)) / max(1, ktimes[fa.FA_KERNEL_BWD_MAIN][0])

    # roofline of the dominant kernel (largest share of device time)
    dom = max(range(4), key=lambda kk: ktimes[kk][1])
    n_l, tot = ktimes[dom]
    avg_ms = tot / max(1, n_l)
    if dom in (fa.FA_KERNEL_FWD, fa.FA_KERNEL_BWD_MAIN):
        # the binding roof is the one with the longer ideal time: FLOPs at the tensor peak, or
        # the pass's compulsory HBM bytes (every input read once, every output written once) at
        # the copy bandwidth; short sequences are HBM bound, long ones tensor bound
        work = ff if dom == fa.FA_KERNEL_FWD else fb
        nbytes = pass_bytes(B, H, W.get("H_kv", H), N, d, dom == fa.FA_KERNEL_FWD)
        roof = binding_roofline(work, nbytes, avg_ms, peaks, peak_src)
    else:
        nbytes = (B * H * N * d * 2 * 2 + B * H * N * 4 + B * H * N * d * 4 + 2 * B * H * N * 4
                  if dom == fa.FA_KERNEL_BWD_PRE else B * H * N * d * (4 + 2))
        achieved = nbytes / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{peak_src} hbm_gbs"}
    roof["kernel"] = fa.KERNEL_NAMES[dom]
    roof["launches"] = n_l
    roof["avg_ms"] = avg_ms
    roof["traffic"] = kernel_traffic(fa.KERNEL_NAMES[dom],
                                     {"pass": "bf16 fwd+bwd", "B": B, "H": H,
                                      "H_kv": W.get("H_kv", H), "N": N, "d": d,
                                      "causal": bool(causal)})
    shares = {fa.KERNEL_NAMES[kk]: ktimes[kk][1] / max(1e-9, sum(t for _, t in ktimes.values()))
              for kk in range(4)}

    # end to end through the public API: pinned host inputs -> device -> fwd+bwd -> host
    # gradients, by fa_fwd_bwd_host (copies of one head chunk overlap the kernels of another);
    # grouped heads have no host entry point and keep the serial copy -> step -> copy path
    e2e = None
    if args.e2e_steps > 0:
        hin = {t: host[t].pin_memory() for t in ("q", "k", "v", "do")}
        hout = [torch.empty(t.shape, dtype=torch.bfloat16).pin_memory() for t in (dq, dk, dv)]
        grouped = W.get("H_kv", H) != H
        chunks = max(1, min(args.e2e_chunks, B * H))
        if not grouped:
            hbuf = torch.empty(fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, chunks),
                               dtype=torch.uint8, device=dev)
        st = torch.cuda.current_stream()
        e_ev = []
        torch.cuda.synchronize()
        barrier(dev)
        for i in range(args.e2e_steps + 2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            if grouped:
                for t, dst in (("q", q), ("k", k), ("v", v), ("do", do)):
                    dst.copy_(hin[t], non_blocking=True)
                step()
                for hsrc, dsrc in zip(hout, (dq, dk, dv)):
                    hsrc.copy_(dsrc, non_blocking=True)
            else:
                rc = fa.fa_fwd_bwd_host(hin["q"].data_ptr(), hin["k"].data_ptr(),
                                        hin["v"].data_ptr(), hin["do"].data_ptr(), None, None,
                                        hout[0].data_ptr(), hout[1].data_ptr(),
                                        hout[2].data_ptr(), B, H, N, d, causal, s, chunks,
                                        hbuf.data_ptr(), hbuf.numel(), st.cuda_stream)
                assert rc == 0, fa.fa_last_error()
            b.record()
            if i >= 2:
                e_ev.append((a, b))
        torch.cuda.synchronize()
        e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in e_ev) / len(e_ev), dev)
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in hout)
        e2e = {"value": world * (ff + fb) / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "api": "serial copies around fa_fwd_gqa / fa_bwd_gqa" if grouped else
                      f"fa_fwd_bwd_host, {chunks} head chunks"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME, **WORKLOAD, "scale": s,
                       "flops_per_step_per_gpu": ff + fb,
                       "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so no dirty line is left; outside the events)",
                       "parallelism": f"heads: {world} independent replicas, no collective"},
            "pct_of_peak": value / world / peaks["bf16_tflops"] * 100.0,
            "fwd_tflops": ff / (fwd_ms * 1e-3) / 1e12, "bwd_tflops": fb / (bwd_ms * 1e-3) / 1e12,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "kernel_time_share": shares,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": sum(ktimes[kk][0] for kk in range(4)),
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


DECODE_DEFAULT = "16,32,8,1,8192,128"


def run_decode(args):
    """Split-key forward on a decoding shape: Nq queries at the end of an Nk-key cache (causal),
    K/V shared by groups of query heads.  HBM bound: the algorithmic bytes are the K/V cache
    plus Q, O and L; the roofline peak is the measured copy bandwidth."""
    import torch
    import exact_io_aware_43_b200 as fa

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rank, world = dist_init("nccl")
    parts = [int(x) for x in args.decode.split(",")]
    B, H, Hkv, Nq, Nk, d = parts[:6]
    s = ai.default_scale(d)
    xq = ai.make_inputs(B, H, Nq, d, seed=rank_seed(rank), with_do=False)["q"]
    xkv = ai.make_inputs(B, Hkv, Nk, d, seed=rank_seed(rank) + 1, with_do=False)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(xq), to_dev(xkv["k"]), to_dev(xkv["v"])
    splits = parts[6] if len(parts) > 6 else fa.default_splits(B, H, Nq, Nk, dev, Hkv)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, fa.fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits)),
                     dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)

    def step():
        fa.forward_splitkv(q, k, v, True, s, splits=splits, out=o, lse=lse, workspace=ws)

    for _ in range(max(3, args.warmup)):
        flush()
        step()
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0, "a kernel reported a timeout during warm-up"
    for kk in range(5):
        fa.fa_timer_read(kk)
    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize()
    sampler.begin()
    fa.fa_timer_enable(True)
    for i in range(args.steps):
        flush()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    sampler.end()
    fa.fa_timer_enable(False)
    barrier(dev)
    clocks = sampler.stop()
    status = fa.fa_device_status()
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev) / args.steps, dev)
    kt = {kk: fa.fa_timer_read(kk) for kk in (fa.FA_KERNEL_FWD, fa.FA_KERNEL_FWD_MERGE)}
    algo_bytes = (2 * B * Hkv * Nk * d * 2) + (2 * B * H * Nq * d * 2) + 4 * B * H * Nq
    peaks, peak_src = load_peaks()
    value = world * algo_bytes / (ms * 1e-3) / 1e9
    n_f, t_f = kt[fa.FA_KERNEL_FWD]
    fwd_ms = t_f / max(1, n_f)
    roof = {"bound": "hbm", "achieved": algo_bytes / (fwd_ms * 1e-3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": algo_bytes / (fwd_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "peak_source": f"{peak_src} hbm_gbs", "kernel": "fa_fwd_kernel", "launches": n_f,
            "avg_ms": fwd_ms,
            "traffic": kernel_traffic("fa_fwd_kernel", {"pass": "decode", "B": B, "H": H,
                                                        "H_kv": Hkv, "Nq": Nq, "Nk": Nk, "d": d,
                                                        "splits": splits}),
            "algorithmic_bytes": algo_bytes}
    if rank == 0:
        line = {
            "metric": "split-key decode attention, HBM GB/s (K/V cache + Q, O, L bytes per step)",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"decode: B={B} H={H} H_kv={Hkv} Nq={Nq} Nk={Nk} d={d} causal, "
                                   f"{splits} key ranges", "B": B, "H": H, "H_kv": Hkv,
                       "Nq": Nq, "Nk": Nk, "d": d, "splits": splits,
                       "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so no dirty line is left; outside the events)"},
            "kernel_ms": {"fa_fwd_kernel": fwd_ms,
                          "fa_fwd_merge_kernel": kt[fa.FA_KERNEL_FWD_MERGE][1] /
                          max(1, kt[fa.FA_KERNEL_FWD_MERGE][0])},
            "roofline": roof, "clocks": clocks,
            "gpu_launches": n_f + kt[fa.FA_KERNEL_FWD_MERGE][0], "device_status": status,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_fp8(args):
    """FP8 (e4m3) forward on the workload's shape: per-tensor scaled e4m3 Q, K, V resident on the
    device, bf16 O and fp32 L out.  Tensor-bound like the bf16 forward; the roofline peak is the
    measured dense bf16 rate times the nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s = 2)."""
    import torch
    import exact_io_aware_43_b200 as fa

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rank, world = dist_init("nccl")
    W = WORKLOAD
    B, H, N, d, causal = W["B"], W["H"], W["N"], W["d"], W["causal"]
    s = ai.default_scale(d)
    x = ai.make_inputs_fp8(B, H, N, d, seed=rank_seed(rank))
    host = {t: torch.from_numpy(c) for t, (c, _) in x.items()}
    sc = {t: sc_ for t, (_, sc_) in x.items()}
    q, k, v = (host[t].to(dev) for t in ("q", "k", "v"))
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)

    def step():
        fa.forward_fp8(q, k, v, sc["q"], sc["k"], sc["v"], causal, s, out=o, lse=lse)

    for _ in range(max(3, args.warmup)):
        flush()
        step()
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0, "a kernel reported a timeout during warm-up"
    fa.fa_timer_read(fa.FA_KERNEL_FWD)
    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize()
    sampler.begin()
    fa.fa_timer_enable(True)
    for i in range(args.steps):
        flush()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    sampler.end()
    fa.fa_timer_enable(False)
    barrier(dev)
    clocks = sampler.stop()
    status = fa.fa_device_status()
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev) / args.steps, dev)
    n_f, t_f = fa.fa_timer_read(fa.FA_KERNEL_FWD)
    ff, _ = flops(B, H, N, d, causal)
    peaks, peak_src = load_peaks()
    peak = 2.0 * peaks["bf16_tflops"]
    kern_ms = t_f / max(1, n_f)
    achieved = ff / (kern_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "peak_source": f"{peak_src} bf16_tflops (burst) x 2, the nominal fp8/bf16 ratio",
            "frac_of_bf16_peak": achieved / peaks["bf16_tflops"], "kernel": "fa_fwd_fp8_kernel",
            "launches": n_f, "avg_ms": kern_ms,
            "traffic": kernel_traffic("fa_fwd_fp8_kernel", {"pass": "fp8 fwd", "B": B, "H": H,
                                                            "N": N, "d": d,
                                                            "causal": bool(causal)})}
    # end to end through the public API: e4m3 codes from pinned host memory, O and L back
    e2e = None
    if args.e2e_steps > 0:
        hin = {t: host[t].pin_memory() for t in ("q", "k", "v")}
        ho = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
        hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        e_ev = []
        torch.cuda.synchronize()
        for i in range(args.e2e_steps + 2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for t, dst in (("q", q), ("k", k), ("v", v)):
                dst.copy_(hin[t], non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            b.record()
            if i >= 2:
                e_ev.append((a, b))
        torch.cuda.synchronize()
        e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in e_ev) / len(e_ev), dev)
        e2e = {"value": world * ff / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(t.numel() for t in hin.values()),
               "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4, "ms_per_step": e_ms,
               "api": "serial copies around fa_fwd_fp8"}
    if rank == 0:
        line = {
            "metric": "attention fwd TFLOP/s fp8 (e4m3 Q, K, V, per-tensor scales) at N=8K d=128 "
                      "causal; % of B200 FP8 peak",
            "value": world * ff / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic",
            "config": {"workload": f"FP8 forward, B={B} H={H} N={N} d={d} causal={causal}",
                       **WORKLOAD, "scale": s, "flops_per_step_per_gpu": ff,
                       "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so no dirty line is left; outside the events)"},
            "roofline": roof, "e2e": e2e, "clocks": clocks, "gpu_launches": n_f,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def sweep_workloads():
    """(name, B, H, N, d, causal) of every parity workload that has a fwd+bwd step, besides the
    headline one: GPT-2-small shape, BERT-large shape, and the B*H*N = 131072 sweep."""
    out = [("GPT-2-small-shaped causal fwd+bwd, B=8 H=12 N=1024 d=64 bf16", 8, 12, 1024, 64, True),
           ("BERT-large-shaped non-causal fwd+bwd, B=16 H=16 N=512 d=64 bf16", 16, 16, 512, 64,
            False)]
    for pt in ai.sweep_points():
        out.append((f"sweep point B*H*N=131072: B={pt['B']} H={pt['H']} N={pt['N']} d={pt['d']} "
                    f"{'causal' if pt['causal'] else 'non-causal'} fwd+bwd bf16",
                    pt["B"], pt["H"], pt["N"], pt["d"], pt["causal"]))
    return out


def run_sweep(args):
    global WORKLOAD_NAME
    args.no_cpu_baseline = True
    args.e2e_steps = 0
    for (name, B, H, N, d, causal) in sweep_workloads():
        WORKLOAD.clear()
        WORKLOAD.update(B=B, H=H, N=N, d=d, causal=causal)
        WORKLOAD_NAME = name
        run_gpu(args)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.decode is not None:
        return run_decode(args)
    if args.fp8:
        return run_fp8(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
