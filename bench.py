#!/usr/bin/env python
"""FAVOR forward benchmark: tokens/s (B*H*L per second) at B=4, H=8, L=4096, d=64, M=256.

One step is one pass of the hot path over one batch: the trig and the ReLU feature maps, each
bidirectional and causal, on the same bf16 inputs. value = head-tokens processed per second
over all ranks (4 variants x B*H*L per step per rank). Inputs are resident in HBM. Four
rotating input sets (268 MB in total, more than 2x the 126 MB L2) keep every step reading HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched by torch.distributed.run. Each rank runs its own batch on its own GPU (the
heads are independent), so per-GPU work is fixed ("weak" scaling) and there is no data-path
collective. Timing: one CUDA graph per input set holds a step (the four variants back to back);
the timed region replays K of them between CUDA events on the launching stream, barrier +
synchronize on both sides, max over ranks. Per-kernel launch durations (for the roofline) come
from each variant's own graph, replayed between CUDA events in the same run.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(B=4, H=8, L=4096, d=64, M=256)
VARIANTS = [("trig_bidir", 0, False), ("relu_bidir", 1, False), ("trig_causal", 0, True), ("relu_causal", 1, True)]
# kernel launches per call of each variant: bidirectional = key states, merge, queries
LAUNCHES = {"trig_bidir": 3, "relu_bidir": 3, "trig_causal": 1, "relu_causal": 1}
N_SETS = 4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "FAVOR fwd tokens/s (B·H·L/s) at L=4096,d=64,M=256; % of tensor/HBM roofline"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of each variant's kernel
# at this workload, from one ncu capture (profiles/), with the SHA-1 of the kernel sources the
# capture was taken with. A value whose sources have changed since is reported as null.
TRAFFIC = {"trig_causal": (51402752, "ff014ab33611f8622d9d069095ec8d10a98cec92")}
_CSRC = "linear_kernelized_attention_b200/csrc/"
_CAUSAL_SOURCES = [_CSRC + "ptx.cuh", _CSRC + "sincos_poly.cuh", _CSRC + "kernel_causal_fs.cuh"]
_BIDIR_SOURCES = [_CSRC + "ptx.cuh", _CSRC + "sincos_poly.cuh", _CSRC + "kernel_bidir_split.cuh"]
KERNEL_SOURCES = {"trig_causal": _CAUSAL_SOURCES, "relu_causal": _CAUSAL_SOURCES,
                  "trig_bidir": _BIDIR_SOURCES, "relu_bidir": _BIDIR_SOURCES}


def kernel_sources_sha(variant):
    """sha1 of the sources a variant's kernels are built from: a stored DRAM traffic figure holds
    only while they are unchanged."""
    import hashlib
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[variant]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def max_over_ranks(x, device=None):
    """Max of a per-rank number over all ranks of the default process group (the number itself
    when torch.distributed is not initialised). Every rank must call it."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def flops_per_token(d, M, kind):
    F = 2 * M if kind == 0 else M
    return 4 * d * M + 4 * F * (d + 1)


def bytes_per_token(d):
    return 4 * d * 2  # read q, k, v and write out, bf16


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f), "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi samples (SM clock, max clock, throttle reasons) while the timed region runs."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.rows, self.proc, self.t = index, [], None, None
        self.active = threading.Event()

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        time.sleep(0.5)

    def _read(self):
        for line in self.proc.stdout:
            if self.active.is_set():
                self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm = []
        mx = None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                for n, val in zip(names, r[3:7]):
                    if val.lower() == "active":
                        reasons.add(n)
            except Exception:
                continue
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(seconds, per_step=False):
    """Time the fp64 oracle (as it stands) on whole heads of the bench workload."""
    import numpy as np

    import favor_inputs as fi
    from oracle import favor_oracle as O
    W = WORKLOAD
    q, k, v = fi.qkv(1, 1, W["L"], W["d"], seed=123)
    G, R = fi.orf_gaussians(1, W["M"], W["d"], seed=123)
    om = O.orf_matrices(G, R, W["M"])[0]
    q, k, v = (x[0, 0].astype(np.float64) for x in (q, k, v))
    tokens, t0, heads = 0, time.perf_counter(), 0
    while True:
        for _, kind, causal in VARIANTS:
            (O.favor_causal_head if causal else O.favor_bidirectional_head)(q, k, v, om, kind)
            tokens += W["L"]
        heads += 1
        if per_step or time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return tokens / dt, dt, heads


def oracle_timed(fn, seconds):
    """Call fn() (one unit of oracle work, returning the units it did) until `seconds` have
    passed; returns (units per second, seconds, calls)."""
    units, calls, t0 = 0, 0, time.perf_counter()
    while True:
        units += fn()
        calls += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return units / dt, dt, calls


def fp32_alu_peak_tflops(sm_mhz=1965.0, sms=148):
    """fp32 CUDA-core peak: 128 FMA lanes per SM, 2 FLOP each, at the given clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def run_reference(args, rank):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(0, per_step=True)
    tok, dt = 0.0, 0.0
    for _ in range(args.steps):
        r, t, _ = oracle_sample(0, per_step=True)
        tok += r * t
        dt += t
    value = tok / dt
    W = WORKLOAD
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "favor_fwd_B4_H8_L4096_d64_M256", **W,
                   "variants": [n for n, _, _ in VARIANTS]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": "one head (L=4096 tokens) per variant per step, fp64 numpy oracle"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def lsweep_points(Ls, dev, stream, reps_budget=64):
    """Throughput against sequence length at B=1, H=16, d=64, M=256 (trig, bidirectional and
    causal): one dict per (L, variant). Constant tokens/s across L is linear scaling. Rotating
    input sets keep every point's reads above twice the L2 size; each point replays a CUDA graph
    of one call per input set between CUDA events."""
    import numpy as np
    import torch

    import favor_inputs as fi
    import linear_kernelized_attention_b200 as F
    B, H, d, M = 1, 16, 64, 256
    G, R = fi.orf_gaussians(H, M, d, seed=0)
    omega = F.favor_orf_omega(torch.from_numpy(G).to(dev), torch.from_numpy(R).to(dev), M, dtype=torch.bfloat16)
    points = []
    for L in Ls:
        nbytes = 3 * B * H * L * d * 2
        nsets = max(1, int(np.ceil(2 * 126e6 / nbytes)))
        sets = []
        for si in range(nsets):
            q, k, v = fi.qkv(B, H, L, d, seed=si)
            sets.append([fi.round_to(x, "bf16").to(dev) for x in (q, k, v)])
        out = torch.empty_like(sets[0][0])
        for causal in (False, True):
            for si in range(nsets):
                F.favor_attention(*sets[si], omega, out=out, feature_kind=0, causal=causal, stream=stream)
            torch.cuda.synchronize()
            if F.favor_sync_status(stream) != 0:
                raise RuntimeError("device status not OK")
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for si in range(nsets):
                    F.favor_attention(*sets[si], omega, out=out, feature_kind=0, causal=causal, stream=stream)
            g.replay()
            torch.cuda.synchronize()
            reps = max(3, int(reps_budget / nsets))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            us = 1e3 * a.elapsed_time(b) / (reps * nsets)
            points.append({"L": L, "B": B, "H": H, "d": d, "M": M,
                           "variant": "trig_causal" if causal else "trig_bidir", "us_per_call": us,
                           "tokens_per_s": B * H * L / (us * 1e-6), "input_sets": nsets})
            del g
        del sets
    return points


def run_lsweep(args):
    """bench.py --lsweep: the L sweep 4096 .. 65536, one JSON line per (L, variant)."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    for pt in lsweep_points((4096, 8192, 16384, 32768, 65536), dev, stream):
        print(json.dumps({"lsweep": True, **pt}), flush=True)


def decode_bytes_per_call(B, H, d, M, kind):
    """Algorithmic HBM bytes of one decode call: the fp32 state read and written once, q, k, v
    read and out written (bf16), the reference read and written, Omega read once per head."""
    F = 2 * M if kind == 0 else M
    BH = B * H
    return BH * (2 * F * (d + 1) * 4 + 4 * d * 2 + 8) + H * M * d * 2


def run_decode(args):
    """Causal decode: one token per head per call against the carried fp32 state. Two batch
    sizes per feature map: B=512, H=8 (4096 heads; the state, 272-545 MB, is larger than twice
    the L2, so each call streams it from HBM) and B=4, H=8 (32 heads; the 4.3 MB state stays in
    L2: a latency point). T=64 distinct tokens are captured in one CUDA graph and replayed."""
    import torch

    import favor_inputs as fi
    import linear_kernelized_attention_b200 as F
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    H, d, M, T = 8, 64, 256, 64
    G, R = fi.orf_gaussians(H, M, d, seed=0)
    omega = F.favor_orf_omega(torch.from_numpy(G).to(dev), torch.from_numpy(R).to(dev), M, dtype=torch.bfloat16)
    batches = [int(x) for x in args.decode_batches.split(",")]
    kinds = [{"trig": 0, "relu": 1}[x] for x in args.decode_kinds.split(",")]
    for B in batches:
        q, k, v = fi.qkv(B, H, T, d, seed=7)
        q, k, v = (fi.round_to(x, "bf16").permute(2, 0, 1, 3).contiguous().to(dev) for x in (q, k, v))
        out = torch.empty_like(q)
        for kind in kinds:
            st = F.favor_decode_new_state(B, H, d, M, kind, device=dev, stream=stream)
            for t in range(max(args.warmup, 3)):
                F.favor_decode_step(q[t % T], k[t % T], v[t % T], omega, st, out=out[t % T], feature_kind=kind,
                                    stream=stream)
            torch.cuda.synchronize()
            if F.favor_sync_status(stream) != 0:
                raise RuntimeError("device status not OK")
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for t in range(T):
                    F.favor_decode_step(q[t], k[t], v[t], omega, st, out=out[t], feature_kind=kind, stream=stream)
            g.replay()
            torch.cuda.synchronize()
            reps = 10
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            if F.favor_sync_status(stream) != 0:
                raise RuntimeError("device status not OK")
            us = 1e3 * a.elapsed_time(b) / (reps * T)
            nb = decode_bytes_per_call(B, H, d, M, kind)
            gbs = nb / (us * 1e-6) / 1e9
            cpu = None
            if not args.no_cpu_baseline and B == batches[0]:
                import numpy as np

                from oracle import favor_oracle as O
                qh, kh, vh = (fi.as_f64(x[:, 0, 0].cpu()) for x in (q, k, v))
                omh = fi.as_f64(omega[0].cpu())
                S0, z0 = O.favor_decode_state(M, d, kind)

                def one_head():
                    for t in range(T):
                        O.favor_decode_step_head(S0, z0, qh[t], kh[t], vh[t], omh, kind)
                    return T
                r, dt, calls = oracle_timed(one_head, 5.0)
                cpu = {"value": r, "unit": "head-tokens/s", "cores": blas_threads(), "kind": "oracle",
                       "sample": f"{calls} x {T} decode steps of one head (favor_decode_step_head), {dt:.1f} s"}
            print(json.dumps({
                "decode": True, "variant": "trig" if kind == 0 else "relu", "B": B, "H": H, "d": d, "M": M,
                "cpu_baseline": cpu,
                "us_per_call": us, "tokens_per_s": B * H / (us * 1e-6),
                "state_mb": F.favor_decode_state_bytes(B, H, d, M, kind) / 1e6,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "bytes_per_call": nb, "peak_source": f"{peak_src} copy"}}), flush=True)
            del g, st


def run_orf(args):
    """Omega redrawn on the device from a seed (favor_orf_omega_seeded), bf16 output: microseconds
    per call at H = 8 and H = 64 heads, M = 256, d = 64, each call a new seed."""
    import torch

    import linear_kernelized_attention_b200 as F
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    for H in (8, 64):
        M, d = 256, 64
        om = torch.empty((H, M, d), dtype=torch.bfloat16, device=dev)
        for s in range(max(args.warmup, 3)):
            F.favor_orf_omega_seeded(s, H, M, d, out=om, stream=stream)
        torch.cuda.synchronize()
        n = 50
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for s in range(n):
            F.favor_orf_omega_seeded(1000 + s, H, M, d, out=om, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if F.favor_sync_status(stream) != 0:
            raise RuntimeError("device status not OK")
        us = 1e3 * a.elapsed_time(b) / n
        cpu = None
        if not args.no_cpu_baseline and H == 8:
            from oracle import favor_oracle as O

            def one_head():
                G, R = O.seeded_orf_gaussians(7, 1, M, d)
                O.orf_matrices(G, R, M)
                return 1
            r, dt, calls = oracle_timed(one_head, 5.0)
            cpu = {"value": 1e6 / r * H, "unit": "us per call (H heads)", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{calls} head(s) of seeded_orf_gaussians + orf_matrices, {dt:.1f} s"}
        print(json.dumps({"orf": True, "H": H, "M": M, "d": d, "us_per_call": us,
                          "blocks": H * (-(-M // d)), "dtype": "bf16 out, fp64 Gram-Schmidt",
                          "cpu_baseline": cpu}), flush=True)


def run_backward(args):
    """fp32 backward (dq, dk, dv) at B=4, H=8, L=4096, d=64, M=256, each variant: microseconds
    per call and FLOP/s of the algorithmic work, against the fp32 CUDA-core peak."""
    import torch

    import favor_inputs as fi
    import linear_kernelized_attention_b200 as F
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    W = WORKLOAD
    B, H, L, d, M = W["B"], W["H"], W["L"], W["d"], W["M"]
    q, k, v = (fi.round_to(x, "f32").to(dev) for x in fi.qkv(B, H, L, d, seed=2))
    dO = torch.randn(B, H, L, d, device=dev, generator=torch.Generator(device=dev).manual_seed(3))
    G, R = fi.orf_gaussians(H, M, d, seed=2)
    om = F.favor_orf_omega(torch.from_numpy(G).to(dev), torch.from_numpy(R).to(dev), M, dtype=torch.float32)
    for name, kind, causal in VARIANTS:
        for _ in range(max(args.warmup, 3)):
            F.favor_attention_backward_f32(q, k, v, om, dO, feature_kind=kind, causal=causal, stream=stream)
        torch.cuda.synchronize()
        n = 5
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            F.favor_attention_backward_f32(q, k, v, om, dO, feature_kind=kind, causal=causal, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if F.favor_sync_status(stream) != 0:
            raise RuntimeError("device status not OK")
        us = 1e3 * a.elapsed_time(b) / n
        Fe = 2 * M if kind == 0 else M
        # algorithmic FLOP per head-token: forward projections and state (recomputed) + the
        # backward's: q and k projections and their transposes, g, h, dv, R and S (2 F (d+1) each)
        flops = (4 * d * M + 4 * Fe * (d + 1)) + (4 * d * M + 4 * d * M + 10 * Fe * (d + 1))
        tf = flops * B * H * L / (us * 1e-6) / 1e12
        cpu = None
        if not args.no_cpu_baseline:
            import numpy as np

            from oracle import favor_oracle as O
            Lh = 1024
            qh, kh, vh, dh = (fi.as_f64(x[0, 0, :Lh].cpu()) for x in (q, k, v, dO))
            omh = fi.as_f64(om[0].cpu())
            r, dt, calls = oracle_timed(lambda: (O.favor_backward_head(qh, kh, vh, omh, kind, causal, dh), Lh)[1], 4.0)
            cpu = {"value": r, "unit": "head-tokens/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{calls} call(s) of favor_backward_head on one head, L={Lh} (quadratic form), {dt:.1f} s"}
        peak = fp32_alu_peak_tflops()
        print(json.dumps({"backward": True, "variant": name, "B": B, "H": H, "L": L, "d": d, "M": M,
                          "dtype": "f32", "us_per_call": us, "tokens_per_s": B * H * L / (us * 1e-6),
                          "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                       "frac": tf / peak,
                                       "peak_source": "fp32 FMA lanes: 148 SMs x 128 x 2 FLOP x 1965 MHz"},
                          "cpu_baseline": cpu}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lsweep", action="store_true", help="leave the L = 4096 / 65536 points out of the bench line")
    ap.add_argument("--lsweep", action="store_true",
                    help="throughput against L (B=1, H=16, trig) instead of the bench line")
    ap.add_argument("--decode", action="store_true",
                    help="causal decode calls (carried state) instead of the bench line")
    ap.add_argument("--decode-batches", default="512,4", help="batch sizes B for --decode (H=8)")
    ap.add_argument("--decode-kinds", default="trig,relu", help="feature maps for --decode")
    ap.add_argument("--orf", action="store_true", help="time Omega redrawn on the device from a seed")
    ap.add_argument("--backward", action="store_true", help="time the fp32 backward pass")
    args = ap.parse_args()
    if args.backward:
        return run_backward(args)
    if args.orf:
        return run_orf(args)
    if args.lsweep:
        return run_lsweep(args)
    if args.decode:
        return run_decode(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    args.warmup = max(args.warmup, 3)

    import numpy as np
    import torch

    import favor_inputs as fi
    import linear_kernelized_attention_b200 as F

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    W = WORKLOAD
    B, H, L, d, M = W["B"], W["H"], W["L"], W["d"], W["M"]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    variants = VARIANTS

    # inputs: N_SETS rotating sets, Omega built on the device from seeded Gaussian draws
    sets = []
    for s in range(N_SETS):
        q, k, v = fi.qkv(B, H, L, d, seed=1000 * rank + s)
        sets.append([fi.round_to(x, "bf16").to(dev) for x in (q, k, v)])
    G, R = fi.orf_gaussians(H, M, d, seed=rank)
    omega = F.favor_orf_omega(torch.from_numpy(G).to(dev), torch.from_numpy(R).to(dev), M,
                              dtype=torch.bfloat16)
    outs = [[torch.empty_like(sets[0][0]) for _ in variants] for _ in range(N_SETS)]

    def launch(s, j, st):
        q, k, v = sets[s]
        _, kind, causal = variants[j]
        F.favor_attention(q, k, v, omega, out=outs[s][j], feature_kind=kind, causal=causal, stream=st)

    # eager warm-up (first-call set-up happens here); the graphs below then launch the kernels
    # without the per-call host work
    for i in range(args.warmup):
        for j in range(len(variants)):
            launch(i % N_SETS, j, stream)
    torch.cuda.synchronize()
    if F.favor_sync_status(stream) != 0:
        raise RuntimeError("device status not OK after warm-up")
    # one CUDA graph per input set holding the four variants back to back (a step), and one per
    # variant holding its launch on each input set (for the per-kernel durations)
    step_graphs = [torch.cuda.CUDAGraph() for _ in range(N_SETS)]
    for s in range(N_SETS):
        with torch.cuda.graph(step_graphs[s], stream=stream):
            for j in range(len(variants)):
                launch(s, j, stream)
    var_graphs = [torch.cuda.CUDAGraph() for _ in variants]
    for j in range(len(variants)):
        with torch.cuda.graph(var_graphs[j], stream=stream):
            for s in range(N_SETS):
                launch(s, j, stream)
    torch.cuda.synchronize()
    for i in range(args.warmup):
        step_graphs[i % N_SETS].replay()
    for g in var_graphs:          # a graph's first replay uploads it: keep that out of the timing
        g.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    # clock window: about a second of the same step replays, untimed, right before the timed
    # region, so the clock record has samples under this load even when the timed region is
    # shorter than the sampling interval; the timed region itself is sampled too
    clocks.active.set()
    t_win = time.perf_counter()
    i = 0
    while time.perf_counter() - t_win < 1.0:
        for _ in range(50):
            step_graphs[i % N_SETS].replay()
            i += 1
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step_graphs[i % N_SETS].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.active.clear()
    if dist:
        dist.barrier()
    clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    if F.favor_sync_status(stream) != 0:
        raise RuntimeError("device status not OK after the timed region")
    # per-kernel average launch duration: each variant's graph (one launch per input set, back to
    # back) replayed between CUDA events on the launching stream
    reps = max(10, min(args.steps, 200) // N_SETS)
    per_variant = {}
    for j, (name, _, _) in enumerate(variants):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            var_graphs[j].replay()
        b.record(stream)
        torch.cuda.synchronize()
        per_variant[name] = a.elapsed_time(b) / (reps * N_SETS)
    tokens_step = len(variants) * B * H * L
    value = world * tokens_step / (ms * 1e-3)

    # linear scaling in L: B=1, H=16 trig at L = 4096 and 65536 (rank 0 only)
    lsw = None
    if rank == 0 and not args.no_lsweep:
        lsw = lsweep_points((4096, 65536), dev, stream, reps_budget=16)
        torch.cuda.set_stream(stream)

    # roofline of the dominant variant (a causal call is one kernel launch; a bidirectional call
    # is three: key states, merge, queries)
    peaks, peak_src = load_peaks()
    dom = max(per_variant, key=per_variant.get)
    kind = [vv[1] for vv in variants if vv[0] == dom][0]
    flops = flops_per_token(d, M, kind) * B * H * L
    achieved = flops / (per_variant[dom] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tr = TRAFFIC.get(dom)
    traffic = tr[0] if tr and tr[1] == kernel_sources_sha(dom) else None
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "kernel": dom,
            "peak_source": f"{peak_src} bf16 burst", "ms_per_launch": per_variant[dom]}

    # end to end through the host-buffer C ABI entry (pinned host memory, copies timed)
    e2e = None
    hq, hk, hv = (x.cpu().pin_memory() for x in sets[0])
    hom = omega.cpu().pin_memory()
    hout = torch.empty_like(hq).pin_memory()
    n_e2e = min(args.steps, 10)
    for _, kind, causal in variants:
        F.favor_attention_host(hq, hk, hv, hom, hout, feature_kind=kind, causal=causal)
    if dist:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        for _, kind, causal in variants:
            F.favor_attention_host(hq, hk, hv, hom, hout, feature_kind=kind, causal=causal)
    e2e_s = max_over_ranks((time.perf_counter() - t0) / n_e2e, dev)
    nx = B * H * L * d * 2
    e2e = {"value": world * tokens_step / e2e_s, "unit": "tokens/s",
           "h2d_bytes_per_step": len(variants) * (3 * nx + H * M * d * 2),
           "d2h_bytes_per_step": len(variants) * nx}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, dt, heads = oracle_sample(10.0)
        cpu = {"value": r, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{heads} head(s) x L=4096 tokens x {len(VARIANTS)} variants, fp64 numpy, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "favor_fwd_B4_H8_L4096_d64_M256", **W,
                       "variants": [vv[0] for vv in variants], "ms_per_launch": per_variant,
                       "l2": f"{N_SETS} rotating input sets ({N_SETS * 4 * B * H * L * d * 2 / 1e6:.0f} MB) > 2x L2",
                       "parallelism": f"replica x{world} (independent heads per rank)",
                       "launches_per_call": LAUNCHES, "lsweep": lsw},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * sum(LAUNCHES[vv[0]] for vv in variants),
            "clocks": {**clocks.summary(), "window": "1 s of the same step replays right before the timed region, and the timed region"},
        }
        print(json.dumps(line), flush=True)
    del step_graphs, var_graphs
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
