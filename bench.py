#!/usr/bin/env python
"""Benchmark of the KDA operator on B200: prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: chunked prefill, B=1, H=32, T=32768, dk=dv=128, bf16 q/k/v, fp32 gates and
state, S0 ~ N(0, 0.02^2).  A "step" is one kda_chunk_fwd call over that batch (all phases of the
chunked prefill).  `value` is tokens/s over all ranks, device-timed with CUDA events on the
launching stream with inputs resident in HBM; `e2e` is the same metric through the public API
with the inputs copied from pinned host memory and out/S_final copied back inside the timed
region.  A decode measurement (256 sequences x 32 heads, 512 successive single-token steps) is
reported under "decode".  With N > 1 (torchrun) every rank runs an independent replica of the
workload on its own GPU (no collective on the data path): weak scaling.

--impl reference times the fp64 CPU oracle (the test oracle, as it stands) on a bounded sample of
the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
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

L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_32k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target duration of the oracle sample")
    ap.add_argument("--only", choices=["prefill", "decode", "backward", "gated_norm"], default=None,
                    help="run one part only (for profiling): no JSON contract line, prints that part's numbers")
    ap.add_argument("--decode-steps", type=int, default=None, help="decode steps to time (default 512)")
    ap.add_argument("--no-extra", action="store_true", help="skip the varlen and 1M-token workloads")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the prefill sequence length (profiling of a smaller case only)")
    ap.add_argument("--output-gate", action="store_true",
                    help="with --only prefill: apply the output gate in the prefill (profiling of that variant)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_traffic(name, units):
    """DRAM bytes per launch of one of our kernels, from the committed ncu summary under profiles/
    (dram__bytes_read.sum + dram__bytes_write.sum per unit, scaled by the units one launch processes).
    Returns (bytes or None, source note); None once the kernel's sources changed since the capture."""
    import glob
    import hashlib
    import re
    pat = re.compile(r"<!-- bench-traffic kernel=(\S+) per_unit_bytes=(\d+) unit=(\S+) sha1=(\w+) sources=(\S+) -->")
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for m in pat.finditer(open(f).read()):
            if m.group(1) != name:
                continue
            h = hashlib.sha1()
            for src in m.group(5).split(","):
                h.update(open(os.path.join(ROOT, src), "rb").read())
            if h.hexdigest()[:16] != m.group(4):
                return None, f"{os.path.basename(f)}: stale, the kernel changed since the capture"
            return int(m.group(2)) * units, f"{os.path.basename(f)} ({m.group(2)} B per {m.group(3)} x {units})"
    return None, "no capture"


# ------------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ------------------------------------------------------------------------------------------------
def init_dist(torch):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(torch, world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(torch, world, x, device="cuda"):
    """Max of a per-rank scalar over all ranks (the slowest rank's time defines the job's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, steps, max_ms):
    """Whole-job throughput: every rank processes its own replica of the workload (weak scaling)."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def replica_seed(seed, rank):
    """Each rank draws an independent problem of the same shape."""
    return seed + 1000 * rank


# ------------------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload
# ------------------------------------------------------------------------------------------------
def cpu_oracle_prefill(w, target_s, seed_offset=0):
    """Time oracle.seq on all H heads of a prefix of the workload, sized to ~target_s seconds."""
    import torch
    import oracle
    from gated_delta_rule_83_b200 import synth
    threads = oracle.default_threads()

    def run(T):
        inp = synth.prefill_inputs(w, device="cpu", T=T, lengths=[T] if w.varlen else None,
                                   seed=w.seed + seed_offset)
        args = [synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta")]
        S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
        t0 = time.perf_counter()
        oracle.seq(*args, S0=S0, threads=threads)
        return time.perf_counter() - t0

    probe_T = 128
    dt = run(probe_T)
    T = int(max(probe_T, min(w.T if not w.varlen else w.varlen[1], probe_T * target_s / max(dt, 1e-6))))
    T = max(64, (T // 64) * 64)
    dt = run(T)
    return {"value": T / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{T} tokens x {w.H} heads (prefix of one sequence of the workload), fp64 sequential "
                      f"recurrence, {threads} threads over heads, {dt:.1f} s"}


def cpu_oracle_decode(w, target_s):
    import oracle
    from gated_delta_rule_83_b200 import synth
    threads = 1
    N = 8
    S = np.asarray(synth.decode_state(w, N=N).double().numpy())
    t0 = time.perf_counter()
    steps = 0
    while time.perf_counter() - t0 < target_s / 2 and steps < w.T:
        inp = synth.decode_inputs(w, steps, N=N)
        _, S = oracle.decode_step(*(synth.to_oracle(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta")), S)
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": N * steps / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{N} sequences x {w.H} heads x {steps} decode steps, fp64, single thread, {dt:.1f} s"}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def run_ours(args):
    import torch
    import gated_delta_rule_83_b200 as kda
    from gated_delta_rule_83_b200 import synth

    world, rank, local = init_dist(torch)
    dev = torch.device("cuda", local)
    hbm, tf, tf_sus, peak_kind = peaks()
    w = synth.WORKLOADS[args.workload]
    if w.kind != "prefill":
        raise SystemExit("the headline workload is a prefill workload; decode is reported under 'decode'")
    if args.only in ("decode", "backward", "gated_norm"):
        stream = torch.cuda.current_stream(dev)
        if args.only == "decode":
            d = bench_decode(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind, steps=args.decode_steps)
        elif args.only == "backward":
            d = bench_backward(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind, steps=args.steps,
                               warmup=args.warmup, tokens=args.tokens)
        else:
            rows = (args.tokens or w.T) * w.B * w.H
            d = bench_gated_norm(torch, kda, dev, stream, world, hbm, peak_kind, rows=rows, d=w.dv, iters=args.steps)
        if rank == 0:
            print(json.dumps(d), flush=True)
        return

    inp = synth.prefill_inputs(w, device=dev, seed=replica_seed(w.seed, rank), T=args.tokens)
    q, k, v, la, beta, S0, cu = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens"))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    tokens = B * T
    out = torch.empty_like(v)
    N = B if cu is None else cu.numel() - 1
    S_fin = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(x.numel() * x.element_size() for x in (q, k, v, la, beta) if x is not None)

    gate = {}
    if args.output_gate:
        if args.only != "prefill":
            raise SystemExit("--output-gate profiles the gated prefill: use it with --only prefill")
        gg = torch.Generator(device=dev).manual_seed(replica_seed(w.seed + 1000, rank))
        gate = dict(z=torch.randn(v.shape, generator=gg, device=dev).to(v.dtype),
                    gate_weight=torch.rand(dv, generator=gg, device=dev) + 0.5, gate_act="sigmoid")

    def step():
        kda.chunk_fwd(q, k, v, la, beta, S0=S0, cu_seqlens=cu, out=out, S_final=S_fin, **gate)

    for _ in range(args.warmup):
        step()
    kda.check()
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    kda.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    prof = kda.profile_end()
    barrier(torch, world)
    clk = clocks.stop()
    kda.check()
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(torch, world, ms_local)
    ms_per_step = ms / args.steps
    value = job_throughput(world, tokens, args.steps, ms)

    # dominant kernel and roofline.  Algorithmic bytes of the prefill per token x head: q, k (bf16),
    # log_alpha (fp32), v (bf16), beta (fp32) read and out (bf16) written -- 1540 B at dk = dv = 128 --
    # plus the state S0 (if given) and S_final, 64 KiB each per (sequence, head).
    launches = sum(n for n, _ in prof.values())
    dom_name, (dom_n, dom_ms) = max(prof.items(), key=lambda kv: kv[1][1])
    tok_heads = tokens * H
    esz = q.element_size()
    alg_bytes = tok_heads * (2 * dk * esz + dv * esz + 4 * dk + 4 + dv * esz) + \
        (2 if S0 is not None else 1) * N * H * dk * dv * 4
    dom_launch_ms = dom_ms / dom_n
    achieved = alg_bytes / (dom_launch_ms / 1e3) / 1e9
    step_dev_ms = sum(t for _, t in prof.values()) / args.steps
    lens = inp["lengths"] if inp["lengths"] is not None else [T] * B
    units = sum((x + 63) // 64 for x in lens) * H  # chunk x head pairs per launch
    traffic, traffic_src = kernel_traffic(dom_name, units)
    roofline = {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic, "traffic_source": traffic_src,
                "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})",
                "alg_bytes_per_launch": alg_bytes, "alg_bytes_per_token_head": alg_bytes / tok_heads,
                "launch_ms": dom_launch_ms, "share_of_step": dom_ms / max(sum(t for _, t in prof.values()), 1e-12),
                "path": {"kernels": sorted(prof), "device_ms_per_step": step_dev_ms,
                         "achieved": alg_bytes / (step_dev_ms / 1e3) / 1e9,
                         "frac": alg_bytes / (step_dev_ms / 1e3) / 1e9 / hbm}}

    # e2e: host buffers through the public API
    e2e = None
    try:
        if args.only is not None:
            raise RuntimeError("skipped (--only)")
        hq, hk, hv, hla, hb = (x.cpu().pin_memory() for x in (q, k, v, la, beta))
        hS0 = S0.cpu().pin_memory() if S0 is not None else None
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hS = torch.empty(S_fin.shape, dtype=torch.float32).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hla, hb)) + \
            (hS0.numel() * 4 if hS0 is not None else 0)
        d2h = hout.numel() * hout.element_size() + hS.numel() * 4
        if cu is not None:
            raise RuntimeError("the host-pipelined entry point takes regular batches")

        def e2e_step():
            # the public host entry point: segments copied in, computed and copied out on
            # overlapping streams (kda_chunk_fwd_host), joined into `stream`
            kda.chunk_fwd_host(hq, hk, hv, hla, hb, S0=hS0, out=hout, S_final=hS, segment_tokens=E2E_SEGMENT,
                               stream=stream, synchronize=False)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        barrier(torch, world)
        n_e2e = max(2, min(args.steps, 5))
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(torch, world, e0.elapsed_time(e1))
        e2e = {"value": world * tokens * n_e2e / (ms_e2e / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e / n_e2e,
               "steps": n_e2e, "api": f"kda_chunk_fwd_host, {E2E_SEGMENT}-token segments, pinned host buffers"}
        del hq, hk, hv, hla, hb
    except Exception as ex:  # pragma: no cover
        e2e = {"value": None, "unit": "tokens/s", "error": str(ex)[:200]}

    del q, k, v, la, beta, out, inp
    torch.cuda.empty_cache()

    extra = None
    if not args.no_extra and args.only is None:
        extra = {}
        for name in ("varlen_64k", "long_1m"):
            torch.cuda.empty_cache()
            extra[name] = bench_prefill_workload(torch, kda, synth, dev, stream, world, rank, name, steps=3, warmup=2)
        torch.cuda.empty_cache()
        # grouped q/k heads (kda_chunk_fwd_ex): the 32K workload with 16 q/k heads shared by 32 value heads
        extra["prefill_32k_qk16"] = bench_prefill_workload(torch, kda, synth, dev, stream, world, rank,
                                                           "prefill_32k", steps=5, warmup=2, qk_heads=16)
        torch.cuda.empty_cache()
        # input prologue (kda_options.prologue = all bits): raw q/k and gate/beta logits, transformed in-kernel
        extra["prefill_32k_prologue"] = bench_prefill_workload(torch, kda, synth, dev, stream, world, rank,
                                                               "prefill_32k", steps=5, warmup=2, prologue=7)
        torch.cuda.empty_cache()
        # bf16 gates (KDA_PROLOGUE_GATE_BF16): the largest input halved, 1284 instead of 1540 B per token-head
        extra["prefill_32k_gate_bf16"] = bench_prefill_workload(torch, kda, synth, dev, stream, world, rank,
                                                                "prefill_32k", steps=5, warmup=2, gate_bf16=True)
        torch.cuda.empty_cache()
        # the output gate in the prefill's epilogue (kda_chunk_fwd_gated): 128-channel group, sigmoid(z)
        extra["prefill_32k_output_gate"] = bench_prefill_workload(torch, kda, synth, dev, stream, world, rank,
                                                                  "prefill_32k", steps=5, warmup=2, output_gate=True)

    gnorm = None
    if not args.no_extra and args.only is None:
        torch.cuda.empty_cache()
        gnorm = bench_gated_norm(torch, kda, dev, stream, world, hbm, peak_kind, rows=B * T * H, d=dv)

    backward = None
    if not args.no_extra and args.only is None:
        torch.cuda.empty_cache()
        backward = bench_backward(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind)
        torch.cuda.empty_cache()

    decode = None
    if not args.no_decode and args.only is None:
        decode = bench_decode(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind, steps=args.decode_steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only is None:
        cpu = cpu_oracle_prefill(w, args.cpu_seconds)

    line = {"metric": "KDA prefill tokens/s (decode tokens/s under 'decode')", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if esz == 2 else "f32",
            "data": "synthetic (seeded; q,k ~N(0,1) L2-normalised, v ~N(0,1), log_alpha = log sigmoid(N(3,1)), "
                    "beta = sigmoid(N(0,1)))",
            "config": {"workload": w.name, "desc": w.desc, "B": B, "T": T, "H": H, "dk": dk, "dv": dv,
                       "chunk": 64, "parallelism": f"replicas x{world} (independent problems, no collective)",
                       "l2": f"inputs {in_bytes / 1e9:.2f} GB per step > L2 {L2_BYTES / 1e6:.0f} MB (no flush)"},
            "roofline": roofline, "kernels": {k_: {"launches": n, "ms": t} for k_, (n, t) in prof.items()},
            "other_workloads": extra, "gated_rmsnorm": gnorm, "backward": backward,
            "gpu_launches": launches, "clocks": clk, "e2e": e2e, "decode": decode, "cpu_baseline": cpu}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_prefill_workload(torch, kda, synth, dev, stream, world, rank, name, steps, warmup, qk_heads=None,
                           prologue=0, gate_bf16=False, output_gate=False):
    """Device-timed throughput of another prefill workload (same method as the headline).  With
    ``qk_heads``, q and k keep only that many heads, shared by groups of value heads.  With
    ``prologue`` the call passes that kda_options.prologue value (the workload's inputs stand in
    for raw projections: the in-kernel transforms cost the same whatever the values).  With
    ``gate_bf16`` log_alpha is passed as bf16 (half its bytes).  With ``output_gate`` the call applies
    the output gate (seeded bf16 z of out's shape, fp32 weight, one 128-channel group, sigmoid) and
    writes the gated output instead of o."""
    w = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(w, device=dev, seed=replica_seed(w.seed, rank))
    q, k, v, la, beta, S0, cu = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens"))
    if qk_heads is not None:
        q, k = q[:, :, :qk_heads].contiguous(), k[:, :, :qk_heads].contiguous()
        inp["q"], inp["k"] = q, k
    if gate_bf16:
        la = la.to(torch.bfloat16)
        inp["log_alpha"] = la
    out = torch.empty_like(v)
    gate = {}
    if output_gate:
        g = torch.Generator(device=dev).manual_seed(replica_seed(w.seed + 1000, rank))
        gate = dict(z=torch.randn(v.shape, generator=g, device=dev).to(torch.bfloat16),
                    gate_weight=torch.rand(w.dv, generator=g, device=dev) + 0.5, gate_act="sigmoid")
    N = q.shape[0] if cu is None else cu.numel() - 1
    S_fin = torch.empty((N, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    tokens = q.shape[0] * q.shape[1]

    def step():
        kda.chunk_fwd(q, k, v, la, beta, S0=S0, cu_seqlens=cu, out=out, S_final=S_fin, prologue=prologue, **gate)

    for _ in range(warmup):
        step()
    kda.check()
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    kda.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    prof = kda.profile_end()
    kda.check()
    ms = max_over_ranks(torch, world, e0.elapsed_time(e1))
    desc = w.desc if qk_heads is None else f"{w.desc}; q/k with {qk_heads} heads shared by groups of value heads"
    if prologue:
        desc += f"; input prologue {prologue} (q/k L2 norm, log-sigmoid gate logits, sigmoid beta logits in-kernel)"
    if gate_bf16:
        desc += "; log_alpha in bf16"
    if output_gate:
        desc += "; output gate in the epilogue (bf16 z read, gated output written instead of o; group 128, sigmoid)"
    res = {"desc": desc, "tokens": tokens, "steps": steps, "ms_per_step": ms / steps,
           "value": job_throughput(world, tokens, steps, ms), "unit": "tokens/s",
           "kernels": {k_: {"launches": n, "ms": t} for k_, (n, t) in prof.items()}}
    del inp, q, k, v, la, beta, S0, out, S_fin, gate
    return res


def bench_gated_norm(torch, kda, dev, stream, world, hbm, peak_kind, rows, d, iters=20):
    """kda_gated_rmsnorm on the prefill output's shape: bf16 o and z, fp32 weight, sigmoid gate,
    full-width groups.  HBM-bound: o and z read once, y written once."""
    g = torch.Generator(device=dev).manual_seed(123)
    o = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
    z = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
    w = torch.rand(d, device=dev, generator=g) + 0.5
    y = torch.empty_like(o)
    for _ in range(3):
        kda.gated_rmsnorm(o, z, weight=w, gate="sigmoid", out=y)
    kda.check()
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        kda.gated_rmsnorm(o, z, weight=w, gate="sigmoid", out=y)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    kda.check()
    us = max_over_ranks(torch, world, e0.elapsed_time(e1)) * 1e3 / iters
    nbytes = 3 * rows * d * 2 + d * 4
    ach = nbytes / (us * 1e-6) / 1e9
    res = {"desc": f"{rows} rows x {d} bf16, sigmoid gate, weight, group = {d}", "us_per_launch": us,
           "rows_per_s": world * rows / (us * 1e-6),
           "roofline": {"bound": "hbm", "kernel": "gated_rmsnorm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                        "frac": ach / hbm, "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})",
                        "alg_bytes_per_launch": nbytes}}
    del o, z, y
    return res


E2E_SEGMENT = 4096  # tokens per pipelined segment of the host entry point
BWD_BYTES_PER_TOKEN_HEAD = 2824  # read q, k, v, dO (bf16), log_alpha, beta; write dq, dk, dv, dlog_alpha, dbeta


def bench_backward(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind, steps=3, warmup=2, tokens=None):
    """kda_chunk_bwd on the 32K-token prefill workload (the training backward of the same call):
    random bf16 cotangent of the output, none on the final state.  Device-timed like the headline;
    the roofline is against the algorithmic bytes of the inputs, cotangent and gradients."""
    w = synth.WORKLOADS["prefill_32k"]
    inp = synth.prefill_inputs(w, device=dev, seed=replica_seed(w.seed, rank), T=tokens)
    g = torch.Generator(device=dev).manual_seed(replica_seed(77, rank))
    do = torch.randn(inp["v"].shape, generator=g, device=dev).to(inp["v"].dtype)
    q, k, v, la, beta, S0 = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "S0"))
    grads = None

    def step():
        nonlocal grads
        grads = kda.chunk_bwd(q, k, v, la, beta, do, S0=S0, grads=grads)

    for _ in range(warmup):
        step()
    kda.check()
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    kda.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    prof = kda.profile_end()
    kda.check()
    ms = max_over_ranks(torch, world, e0.elapsed_time(e1))
    tokens = q.shape[0] * q.shape[1]
    nbytes = BWD_BYTES_PER_TOKEN_HEAD * tokens * w.H
    ach = nbytes / (ms / steps * 1e-3) / 1e9
    res = {"desc": f"{w.desc}; backward (kda_chunk_bwd), bf16 dO; every chunk product and both chains on "
                   "tcgen05 with split-bf16 operands (fp32 accuracy); inverses, scans and element-wise work on CUDA cores",
           "tokens": tokens, "steps": steps, "ms_per_step": ms / steps,
           "value": job_throughput(world, tokens, steps, ms), "unit": "tokens/s",
           "kernels": {k_: {"launches": n, "ms": t} for k_, (n, t) in prof.items()},
           "roofline": {"bound": "hbm", "kernel": "whole backward", "achieved": ach, "peak": hbm, "unit": "GB/s",
                        "frac": ach / hbm, "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})",
                        "alg_bytes_per_token_head": BWD_BYTES_PER_TOKEN_HEAD, "alg_bytes_per_step": nbytes}}
    del inp, q, k, v, la, beta, S0, do, grads
    return res


def bench_decode(torch, kda, synth, dev, stream, world, rank, hbm, peak_kind, steps=None):
    w = synth.WORKLOADS["decode_256x512"]
    steps = steps or w.T
    S = synth.decode_state(w, device=dev, seed=replica_seed(w.seed, rank))
    # per-step inputs, drawn fresh per step, pre-generated in HBM (one tensor per field with a step axis)
    inp = synth.decode_inputs(w, 0, device=dev, steps=steps, seed=replica_seed(w.seed, rank))
    out = torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    fields = [inp[x] for x in ("q", "k", "v", "log_alpha", "beta")]

    def run(n):
        for t in range(n):
            kda.decode_step(fields[0][t], fields[1][t], fields[2][t], fields[3][t], fields[4][t], S, out=out)

    run(8)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    kda.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    prof = kda.profile_end()
    kda.check()
    ms = max_over_ranks(torch, world, e0.elapsed_time(e1))
    n, kms = prof["decode_step"]
    pairs = w.B * w.H
    alg = pairs * (2 * w.dk * w.dv * 4 + 2 * w.dk * 2 + w.dv * 2 + 4 * w.dk + 4 + w.dv * 2)
    ach = alg / (kms / n / 1e3) / 1e9
    traffic, traffic_src = kernel_traffic("decode_step", pairs)
    # the same loop of calls captured once in a CUDA graph and replayed (no host launch cost)
    graph_us = None
    try:
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            run(steps)
        graph.replay()
        torch.cuda.synchronize(dev)
        barrier(torch, world)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        kda.check()
        graph_us = max_over_ranks(torch, world, e0.elapsed_time(e1)) * 1e3 / steps
        del graph
    except Exception as ex:  # pragma: no cover
        graph_us = f"unavailable: {str(ex)[:120]}"
    return {"metric": "KDA decode tokens/s", "workload": w.name, "desc": w.desc,
            "value": job_throughput(world, w.B, steps, ms), "unit": "tokens/s", "steps": steps,
            "us_per_step": ms * 1e3 / steps, "graph_us_per_step": graph_us,
            "roofline": {"bound": "hbm", "kernel": "decode_step", "achieved": ach, "peak": hbm, "unit": "GB/s",
                         "frac": ach / hbm, "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})", "traffic": traffic,
                         "traffic_source": traffic_src,
                         "alg_bytes_per_launch": alg, "device_us_per_launch": kms / n * 1e3},
            "gpu_launches": n}


# ------------------------------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ------------------------------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from gated_delta_rule_83_b200 import synth
    w = synth.WORKLOADS[args.workload]
    per_step = max(1.0, 60.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        cpu_oracle_prefill(w, min(per_step, 2.0))
    vals, samples = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_oracle_prefill(w, per_step)
        vals.append(r["value"])
        samples.append(r)
    wall = time.perf_counter() - t0
    v = statistics.median(vals)
    cb = dict(samples[0])
    cb["value"] = v
    line = {"impl": "reference", "metric": "KDA prefill tokens/s (decode tokens/s under 'decode')", "value": v,
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * wall / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, same generator as our arm)",
            "config": {"workload": w.name, "desc": w.desc, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "chunk": 64, "parallelism": "host cores (oracle)"},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
