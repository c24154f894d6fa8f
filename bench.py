"""Benchmark of the deterministic attention backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload INDEX] [--schedule NAME] [--all-workloads]

One step = one backward pass (Delta preprocess + persistent kernel) of the
workload through the C ABI, inputs resident in HBM.  L2 is flushed (a 512 MiB
write) before every timed step; each step is timed with CUDA events on the
launching stream and the steps are bracketed by a barrier and synchronisation.
Rank 0 prints one JSON line.  With torchrun (N > 1) every rank runs the same
workload on its own GPU (weak scaling: the B*H heads of one workload per GPU;
heads are independent, so no data-path collective exists) and the time is the
maximum over ranks.

--impl reference times the fp64 CPU oracle (the only other implementation of
the same computation) on a bounded sample of heads of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from persistent_sm_attn_b200.inputs import WORKLOADS, seed_of  # noqa: E402

METRIC = "deterministic attn-bwd TFLOPS (% of B200 bf16 peak); det/nondet throughput ratio"
DEFAULT_WORKLOAD = 3  # causal_b4_h32_s16384_d64, the workload with the most FLOPs


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


def _recorded_traffic(workload: str, schedule: str):
    """DRAM bytes per launch recorded from an ncu capture, or None when no
    capture exists for this workload/schedule or the kernel sources changed
    since it was taken."""
    import hashlib

    h = hashlib.sha256()
    for f in ("bwd_kernel.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "persistent_sm_attn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.txt")) as fh:
            for line in fh:
                parts = line.split()
                if len(parts) == 4 and not line.startswith("#"):
                    if parts[0] == workload and parts[1] == schedule and parts[3] == digest:
                        return int(parts[2])
    except OSError:
        pass
    return None


def _workload(args):
    """The workload of this run: one of the configurations, or --shape B,H,S,D,mask (a
    shape of the caller's, same input recipe and seed as the --workload configuration)."""
    from persistent_sm_attn_b200.inputs import WORKLOADS, Workload
    if not args.shape:
        return WORKLOADS[args.workload]
    b, h, s, d, mask = args.shape.split(",")
    B, H, S, D, causal = int(b), int(h), int(s), int(d), mask.strip() == "causal"
    N = S // 128
    if causal and N % 4 == 0:
        scheds = ("sym_shift", "sym_shift_pairs", "descending")
    elif causal:
        scheds = ("sym_shift", "descending") if N % 2 == 0 else ("descending",)
    elif N % 2 == 0:
        scheds = ("shift", "shift_pairs", "descending")
    else:
        scheds = ("shift", "descending")
    scheds = scheds + ("atomic",)
    return Workload(f"{'causal' if causal else 'full'}_b{B}_h{H}_s{S}_d{D}", B, H, S, D, causal,
                    1.0, scheds)


def _config(w, sched, world, h_kv):
    """The config object of a JSON line; both arms print the same one, so the
    reference arm's line names exactly the workload this arm times."""
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": h_kv, "S": w.S, "D": w.D,
            "mask": "causal" if w.causal else "full", "sigma": w.sigma, "schedule": sched,
            "parallelism": f"dp{world} (independent heads)",
            "l2": "flushed before every timed step (512 MiB write)"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, maxmhz, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                maxmhz.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxmhz),
                "reasons": sorted(reasons), "samples": len(mhz)}


def _dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_ours(args):
    import datetime

    import torch

    from persistent_sm_attn_b200 import binding
    from persistent_sm_attn_b200.inputs import draw
    from persistent_sm_attn_b200.parallel import max_over_ranks

    world, rank, local = _dist_init(args)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = _workload(args)
    if args.heads:
        # a smaller case of the same kernel (profiling): B=1 and the given head count
        w = dataclasses.replace(w, B=1, H=args.heads, name=f"{w.name}_as_b1_h{args.heads}")
    gqa = bool(args.kv_heads) and args.kv_heads != w.H
    if gqa:
        # grouped-query attention: the same query heads over fewer K/V heads
        w = dataclasses.replace(w, name=f"{w.name}_kv{args.kv_heads}")
    sched = args.schedule or w.schedules[0]
    q, k, v, do = draw(w.B, w.H, w.S, w.D, w.sigma, seed_of(args.workload) + 1000 * rank,
                       device="cuda")
    if gqa:
        _, k, v, _ = draw(w.B, args.kv_heads, w.S, w.D, w.sigma,
                          seed_of(args.workload) + 1000 * rank + 1, device="cuda")
        fwd_call = binding.dash_attn_fwd_gqa
        split = args.gqa_split or binding.dash_bwd_gqa_split_for(
            binding.dash_bwd_num_ctas(local, w.D), w.B, args.kv_heads, w.H // args.kv_heads,
            w.S, w.causal, sched)

        def bwd_call(*a):
            return binding.dash_attn_bwd_gqa(*a, split=split)
    else:
        fwd_call, bwd_call = binding.dash_attn_fwd, binding.dash_attn_bwd
    o, lse = fwd_call(q, k, v, w.causal)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    binding.dash_set_dq_chain_mode(args.dq_chain_mode)
    binding.dash_set_head_interleave(args.head_interleave)
    binding.dash_set_slot_placement(args.slot_placement)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def time_schedule(name, steps, warmup, clocks=None):
        dq = torch.empty_like(q)
        dk = torch.empty_like(k)
        dv = torch.empty_like(v)
        for _ in range(warmup):
            bwd_call(q, k, v, o, do, lse, w.causal, name, dq, dk, dv)
        st = binding.dash_attn_sync_status()
        if st != 0:
            raise RuntimeError(f"warm-up status {binding.dash_status_string(st)}")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        barrier()
        binding.dash_profile_begin()
        ctx = clocks if clocks is not None else _Null()
        with ctx:
            for i in range(steps):
                flush.fill_(float(i))
                evs[i][0].record(stream)
                bwd_call(q, k, v, o, do, lse, w.causal, name, dq, dk, dv)
                evs[i][1].record(stream)
            barrier()
        main_ms, aux_ms, n_calls = binding.dash_profile_end()
        st = binding.dash_attn_sync_status()
        if st != 0:
            raise RuntimeError(f"timed status {binding.dash_status_string(st)}")
        step_ms = sum(a.elapsed_time(b) for a, b in evs)
        step_ms = max_over_ranks(step_ms, "cuda")
        main_ms = max_over_ranks(main_ms, "cuda")
        return step_ms / steps, main_ms / steps, aux_ms / steps, n_calls

    clocks = ClockSampler(local)
    ms, main_ms, aux_ms, n_calls = time_schedule(sched, args.steps, args.warmup, clocks)
    results = {sched: ms}
    compare = [s for s in w.schedules if s != sched] if not args.no_compare else []
    for other in compare:
        results[other] = time_schedule(other, max(5, args.steps // 2), 3)[0]

    # the attention block around it: the library forward (O, LSE) timed the same way,
    # outside the backward's timed region
    fo, fl = torch.empty_like(q), torch.empty_like(lse)
    for _ in range(2):
        fwd_call(q, k, v, w.causal, fo, fl)
    fwd_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(max(3, args.steps // 2))]
    barrier()
    for i, (a, b) in enumerate(fwd_ev):
        flush.fill_(float(i))
        a.record(stream)
        fwd_call(q, k, v, w.causal, fo, fl)
        b.record(stream)
    barrier()
    if binding.dash_attn_sync_status() != 0:
        raise RuntimeError("forward status")
    fwd_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in fwd_ev) / len(fwd_ev), "cuda")
    # the attention block: forward then backward back to back on one stream, in one
    # event pair per step (the backward reads the O and LSE this forward wrote)
    bq, bk, bv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for _ in range(2):
        fwd_call(q, k, v, w.causal, fo, fl)
        bwd_call(q, k, v, fo, do, fl, w.causal, sched, bq, bk, bv)
    blk_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(max(3, args.steps // 2))]
    barrier()
    for i, (a, b) in enumerate(blk_ev):
        flush.fill_(float(i))
        a.record(stream)
        fwd_call(q, k, v, w.causal, fo, fl)
        bwd_call(q, k, v, fo, do, fl, w.causal, sched, bq, bk, bv)
        b.record(stream)
    barrier()
    if binding.dash_attn_sync_status() != 0:
        raise RuntimeError("block status")
    block_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in blk_ev) / len(blk_ev), "cuda")
    del fo, fl, bq, bk, bv

    sim = None
    if rank == 0 and not args.no_compare and not gqa:
        sim = simulator_vs_measured(w, q, k, v, o, do, lse, sched, results)

    # end to end through the public API's host-buffer entry point: every step copies
    # the pinned host inputs in and the results out, overlapped with the compute
    # (multi-head only: there is no grouped-query host-buffer entry)
    e2e = None
    if not gqa:
        host_in = [t.cpu().pin_memory() for t in (q, k, v, o, do, lse)]
        host_out = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(3)]
        e2e_steps = max(3, args.steps // 2)
        for it in range(e2e_steps + 2):
            if it == 2:
                barrier()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            binding.dash_attn_bwd_host(*host_in, w.causal, sched, *host_out)
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, "cuda")
        e2e = {"value": round(w.flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host_in),
               "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in host_out)}

    if rank == 0:
        peak, _, peak_kind = _peaks()
        tflops = lambda msec: w.flops * world / (msec * 1e-3) / 1e12
        value = tflops(ms)
        kern = w.flops / (main_ms * 1e-3) / 1e12
        atomic_ms = results.get("atomic")
        det = {s: round(tflops(m), 2) for s, m in results.items()}
        best_det = max((v_ for s, v_ in det.items() if s != "atomic"), default=None)
        il = (binding.dash_bwd_head_interleave(binding.dash_bwd_num_ctas(local, w.D), w.D,
                                               sched, w.B * w.H, w.S, w.causal)
              if not gqa else (w.H // args.kv_heads) // split)
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 Q, K, V, dO; O and LSE from the library forward)",
            "config": dict(_config(w, sched, world, args.kv_heads if gqa else w.H),
                           **({"gqa_split": split} if gqa else {})),
            "pct_of_peak": round(100 * value / (peak * world), 2),
            "schedules_tflops": det,
            "det_nondet_ratio": (round(best_det / det["atomic"], 4)
                                 if atomic_ms and best_det else None),
            "dq_chain": ("red" if binding.dash_dq_chain_uses_red(sched, w.S, w.D, il)
                         else "load-add-store") if sched != "atomic" else None,
            "heads_per_unit": il if not gqa else None,
            "slot_placement": ("cta_pairs" if sched in ("shift_pairs", "sym_shift_pairs") else
                               "sm_id" if binding.dash_slot_placement_by_smid(w.S)
                               else "launch_order"),
            "roofline": {"bound": "tensor", "achieved": round(kern, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(kern / peak, 4),
                         "traffic": _recorded_traffic(w.name, sched),
                         "kernel": "dash_bwd_kernel", "peak_kind": f"{peak_kind} bf16 burst",
                         "kernel_ms": round(main_ms, 4), "aux_ms": round(aux_ms, 4)},
            "e2e": e2e,
            "gpu_launches": int(n_calls) * (3 if sched == "atomic" else 2),
            "fwd_bwd": {"fwd_ms": round(fwd_ms, 4),
                        "fwd_tflops": round(0.4 * w.flops * world / (fwd_ms * 1e-3) / 1e12, 2),
                        "block_ms": round(block_ms, 4),
                        "block_tflops": round(1.4 * w.flops * world /
                                              (block_ms * 1e-3) / 1e12, 2),
                        "note": "fwd_ms: the library forward alone (4 B H S^2 D FLOPs, half "
                                "causal); block_ms: forward then this line's backward, back to "
                                "back, in one event pair per step, L2 flushed before each"},
            "clocks": clocks.summary(),
        }
        if sim is not None:
            line["simulator"] = sim
        if not args.no_cpu_baseline and world == 1 and not gqa:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def simulator_vs_measured(w, q, k, v, o, do, lse, main_sched, measured_ms):
    """DAG-simulator prediction of the deterministic schedules' order, with
    weights taken from two traced launches (outside the timed region): c = the
    atomic kernel's median pair period on a CTA, r = the deterministic
    kernel's median time from ticket grant to published reduction."""
    import numpy as np

    from persistent_sm_attn_b200 import binding

    *_, tr_a = binding.dash_trace_bwd(q, k, v, o, do, lse, w.causal, "atomic")
    *_, tr_d = binding.dash_trace_bwd(q, k, v, o, do, lse, w.causal, main_sched)
    periods = []
    for c in range(tr_a.shape[0]):
        e0 = tr_a[c, :, 0].astype(np.int64)
        e0 = e0[e0 > 0]
        periods += list(np.diff(e0))
    e6, e7 = tr_d[:, :, 6].astype(np.int64), tr_d[:, :, 7].astype(np.int64)
    m = (e6 > 0) & (e7 > 0)
    c_us = float(np.median(periods)) / 1000.0 if periods else 1.0
    r_us = float(np.median(e7[m] - e6[m])) / 1000.0 if m.any() else 0.0
    ctas = binding.dash_bwd_num_ctas(0, w.D)
    pred = {}
    for s_ in measured_ms:
        if s_ == "atomic":
            continue
        cp, *_ = binding.dash_sched_simulate(w.B * w.H, w.n_tiles, w.causal, s_, ctas, c_us,
                                             r_us, 2, 2)
        pred[s_] = round(cp / 1000.0, 4)
    det = {s_: m_ for s_, m_ in measured_ms.items() if s_ != "atomic"}
    return {"c_us": round(c_us, 3), "r_us": round(r_us, 3), "dq_buffers": 2, "dq_chains": 2,
            "ctas": ctas,
            "predicted_ms": pred, "predicted_order": sorted(pred, key=pred.get),
            "measured_ms": {s_: round(m_, 4) for s_, m_ in det.items()},
            "measured_order": sorted(det, key=det.get)}


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def _oracle_heads_tflops(w, seconds: float, index: int):
    """Time the fp64 oracle's per-head backward on seeded heads of workload w
    until ``seconds`` of CPU work have been spent (at least one head)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import attention as A
    from persistent_sm_attn_b200.inputs import draw

    flops_per_head = w.flops / (w.B * w.H)
    heads = 0
    t_total = 0.0
    scale = 1.0 / np.sqrt(w.D)
    while heads == 0 or t_total < seconds:
        q, k, v, do = (t[0, 0].float().numpy()
                       for t in draw(1, 1, w.S, w.D, w.sigma, seed_of(index) + heads))
        t0 = time.perf_counter()
        A.head_backward(q, k, v, do, w.causal, scale)
        t_total += time.perf_counter() - t0
        heads += 1
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    return flops_per_head * heads / t_total / 1e12, heads, t_total, threads


def cpu_baseline(w, seconds):
    index = WORKLOADS.index(w)
    tf, heads, t, cores = _oracle_heads_tflops(w, seconds, index)
    return {"value": round(tf, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} head(s) of {w.name} (S={w.S}, D={w.D}), fp64 numpy oracle, "
                      f"{t:.1f} s; backward FLOPs counted as in the metric"}


def run_reference(args):
    world, rank, _ = _dist_init(args)
    if rank != 0:
        return
    w = _workload(args)
    gqa = bool(args.kv_heads) and args.kv_heads != w.H
    if gqa:
        # the oracle's grouped-query backward is the per-head backward of every query
        # head plus the sums of dK, dV over each group, so its cost per query head is
        # the per-head backward timed here
        w = dataclasses.replace(w, name=f"{w.name}_kv{args.kv_heads}")
    per_step = []
    last = None
    for _ in range(args.warmup):
        _oracle_heads_tflops(w, 0.0, args.workload)
    for _ in range(args.steps):
        last = _oracle_heads_tflops(w, args.cpu_seconds / max(1, args.steps), args.workload)
        per_step.append(last[0])
    value = statistics.mean(per_step)
    tf, heads, t, cores = last
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded normal bf16 Q, K, V, dO widened to fp64)",
        "config": _config(w, args.schedule or w.schedules[0], world,
                          args.kv_heads if gqa else w.H),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: >= {args.cpu_seconds / max(1, args.steps):.1f} s "
                                   f"of per-head fp64 backward of {w.name}"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    # the default is the largest workload: B=4 H=32 S=16384 D=64, causal
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--schedule", default=None)
    ap.add_argument("--no-compare", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--all-workloads", action="store_true",
                    help="one JSON line per workload (1-4), rank 0 only")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="time grouped-query attention with this many K/V heads (a side "
                         "measurement: no host-buffer e2e, simulator or CPU baseline)")
    ap.add_argument("--shape", default="",
                    help="B,H,S,D,mask (mask full or causal): time this shape instead of a "
                         "configuration, with the same input recipe")
    ap.add_argument("--dq-chain-mode", type=int, default=0, choices=(0, 1, 2),
                    help="how the ordered dQ chains add a middle position: 0 the library's "
                         "choice, 1 red in L2, 2 load-add-store (bitwise the same results)")
    ap.add_argument("--slot-placement", type=int, default=0, choices=(0, 1, 2),
                    help="table slots on the SMs: 0 the library's choice, 1 by SM id, "
                         "2 launch order (bitwise the same results)")
    ap.add_argument("--head-interleave", type=int, default=0, choices=(0, 1, 2, 4),
                    help="heads per unit of the multi-head table: 0 the library's choice, "
                         "1 none, 2 or 4 forced")
    ap.add_argument("--gqa-split", type=int, default=0,
                    help="with --kv-heads: sub-groups per K/V head (0 = the library's choice)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload's shape with B=1 and this many heads (a smaller "
                         "case of the same kernel, for profiling); 0 = the workload as named")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
        return
    if args.all_workloads:
        for i in range(1, len(WORKLOADS)):
            args.workload = i
            run_ours(args)
        return
    run_ours(args)


if __name__ == "__main__":
    main()
