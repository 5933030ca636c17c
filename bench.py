"""Benchmark of the FlashBlock attention step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload dllm_8k] [--no-e2e]

A timed "step" is one pass of the whole hot path over one workload: the
diffusion-LM schedule of one attention layer (dllm_8k: B 1, 32 query / 8 KV
heads, head dim 128, prefix 8192 tokens growing by 32 per block, blocks of 32
tokens, 8 diffusion steps per block, 4 blocks, tau = 8).  Every diffusion step
runs fb_step under the reuse policy, and every block ends with fb_kv_append.
The metric is query tokens per second (B * Nb per diffusion step) with reuse
on; the same schedule with tau = 0 (every step recomputes over the whole KV
cache) is reported beside it.  L2 is flushed (a 1 GiB write) before every
diffusion step, outside the event-timed interval, so each step reads the KV
cache from HBM as it would between the layers of a model; the flush also keeps
the GPU busy long enough for the host to enqueue the next step, so the timed
interval holds no host launch gaps.

Each diffusion step is captured once as a CUDA graph (fb_step plus, at a
block's end, fb_kv_append; the reuse decisions are taken on the host while
capturing, in schedule order) and the timed region replays them; the same
steps as eager library calls are reported under "eager", and the per-kernel
breakdown behind "roofline" comes from a separate eager pass with CUDA events
around every launch.

`--impl reference` times the fp64 CPU oracle on this host's cores on a
bounded sample of the same schedule (the reference arm; there is no other
implementation to run).  Under torchrun, each rank runs an independent replica
(weak scaling, no collective on the data path); rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_diffusion_attention_flashblock_b200 import workloads as wl  # noqa: E402

METRIC = "block-diffusion attention step latency & query tok/s vs full-KV recompute"
UNIT = "query tok/s"
L2_FLUSH_BYTES = 1 << 30


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _describe(spec) -> str:
    return (f"{spec.name}: B{spec.B} Hq{spec.Hq} Hkv{spec.Hkv} D{spec.D} prefix {spec.prefix0}"
            f" (+{spec.Nb}/block) Nb {spec.Nb}, {spec.steps} steps x {spec.blocks} blocks"
            + (f", tau {spec.tau}" if spec.tau is not None else "")
            + (f", gamma {spec.gamma}" if spec.gamma is not None else "")
            + (f", sparse k {spec.sel_k}" if spec.sel_k else ""))


# ------------------------------------------------------------------ clocks ---
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------- ours ---
class Schedule:
    """All inputs of one workload pass, resident on the device, plus host copies for e2e."""

    def __init__(self, spec, device):
        self.spec = spec
        w = wl.Workload(spec)
        kp, vp = w.prefix_kv()
        self.kp, self.vp = kp.to(device), vp.to(device)
        self.steps = []
        for st in w.schedule():
            self.steps.append(dict(st=st, q=st.q.to(device), kin=st.kin.to(device), vin=st.vin.to(device),
                                   sel=None if st.sel is None else st.sel.to(device),
                                   hq=st.q.pin_memory(), hk=st.kin.pin_memory(), hv=st.vin.pin_memory()))
        self.query_tokens = spec.B * spec.Nb * len(self.steps)


def run_ours(args, spec, rank, world, device):
    from block_diffusion_attention_flashblock_b200 import fb
    torch.cuda.set_device(device)
    fb.fb_debug_set_prefix_kernel({"auto": 0, "generic": 1, "tcgen05": 2}[args.prefix_kernel])
    sched = Schedule(spec, device)
    s = spec
    dt = s.torch_dtype
    o = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=dt, device=device)
    lse = torch.empty(s.B, s.Hq, s.Nb, dtype=torch.float32, device=device)
    q_like = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=dt, device=device)
    k_like = torch.empty(s.B, s.Hkv, s.Nb, s.D, dtype=dt, device=device)
    layer = fb.FlashBlockLayer(q_like, k_like, sched.kp, o, max_prefix=s.lcap, gamma=s.gamma is not None,
                               sparse=s.sel_k is not None, max_sel_k=s.sel_k or 0)
    gamma = torch.full((s.Hq,), s.gamma, device=device) if s.gamma is not None else None
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    ho = torch.empty(o.shape, dtype=dt, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)

    def one_pass(tau, events, e2e=False, kinds=None):
        for item in sched.steps:
            st = item["st"]
            if st.step == 0:
                layer.begin_block()
            flush.zero_()                                   # evict the KV cache from L2
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if e2e:
                item["q"].copy_(item["hq"], non_blocking=True)
                item["kin"].copy_(item["hk"], non_blocking=True)
                item["vin"].copy_(item["hv"], non_blocking=True)
            layer.step(item["q"], item["kin"], item["vin"], sched.kp, sched.vp, st.prefix_len, st.M, tau, o,
                       lse, gamma, item["sel"])
            if st.last_in_block:
                fb.fb_kv_append(layer.desc, sched.kp, sched.vp, st.prefix_len, item["kin"], item["vin"])
            if e2e:
                ho.copy_(o, non_blocking=True)
                hl.copy_(lse, non_blocking=True)
            e1.record(stream)
            events.append((e0, e1, layer.last_recomputed()))

    def timed(tau, steps, warmup, e2e=False, profile=False):
        for _ in range(warmup):
            one_pass(tau, [], e2e)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        if profile:
            fb.fb_profile_read(reset=True)
            fb.fb_profile_enable(True)
        events = []
        for _ in range(steps):
            one_pass(tau, events, e2e)
        torch.cuda.synchronize()
        if profile:
            fb.fb_profile_enable(False)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b, _ in events]
        kinds = [k for _, _, k in events]
        total = torch.tensor([sum(ms)], dtype=torch.float64, device=device)
        if world > 1:
            torch.distributed.all_reduce(total, op=torch.distributed.ReduceOp.MAX)
        prof = fb.fb_profile_read(reset=True) if profile else None
        return total.item() / steps, ms, kinds, prof

    def capture(tau):
        """One CUDA graph per diffusion step: its fb_step and, at a block's end,
        the append.  The reuse decisions are taken on the host while capturing,
        in schedule order, exactly as an eager pass takes them."""
        graphs = []
        for item in sched.steps:
            st = item["st"]
            if st.step == 0:
                layer.begin_block()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                layer.step(item["q"], item["kin"], item["vin"], sched.kp, sched.vp, st.prefix_len, st.M, tau, o,
                           lse, gamma, item["sel"])
                if st.last_in_block:
                    fb.fb_kv_append(layer.desc, sched.kp, sched.vp, st.prefix_len, item["kin"], item["vin"])
            graphs.append((g, layer.last_recomputed()))
        torch.cuda.synchronize()
        return graphs

    def timed_graphs(graphs, steps, warmup):
        def run(events):
            for g, rec in graphs:
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                events.append((e0, e1, rec))
        for _ in range(warmup):
            run([])
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        events = []
        for _ in range(steps):
            run(events)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b, _ in events]
        total = torch.tensor([sum(ms)], dtype=torch.float64, device=device)
        if world > 1:
            torch.distributed.all_reduce(total, op=torch.distributed.ReduceOp.MAX)
        return total.item() / steps, ms, [k for _, _, k in events]

    tau_on = s.tau if s.tau is not None else fb.FB_TAU_OFF
    props = torch.cuda.get_device_properties(device)
    try:
        smi_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except AttributeError:
        smi_id = str(device.index)
    clocks = ClockSampler(smi_id)
    # eager library calls (no per-kernel events inside the timed steps)
    ms_eager, _, _, _ = timed(tau_on, args.steps, args.warmup)
    # the same steps replayed from CUDA graphs (the headline number)
    clocks.start()
    if args.eager:
        ms_on, per_on, kinds_on = ms_eager, *timed(tau_on, args.steps, 0)[1:3]
    else:
        graphs_on = capture(tau_on)
        ms_on, per_on, kinds_on = timed_graphs(graphs_on, args.steps, args.warmup)
    clk = clocks.stop()
    # per-kernel CUDA events around every launch, in a separate eager pass
    _, _, _, prof = timed(tau_on, args.steps, 1, profile=True)
    if args.profile_run:
        ms_full, per_full = float("nan"), []
    elif args.eager:
        ms_full, per_full, _, _ = timed(0, args.steps, args.warmup)
    else:
        graphs_full = capture(0)
        ms_full, per_full, _ = timed_graphs(graphs_full, args.steps, args.warmup)
    e2e = None
    if not args.no_e2e and not args.profile_run:
        ms_e2e, _, _, _ = timed(tau_on, args.steps, args.warmup, e2e=True)
        item = sched.steps[0]
        h2d = sum(it["hq"].numel() * it["hq"].element_size() + 2 * it["hk"].numel() * it["hk"].element_size()
                  for it in sched.steps)
        d2h = len(sched.steps) * (ho.numel() * ho.element_size() + hl.numel() * hl.element_size())
        e2e = {"value": world * sched.query_tokens / (ms_e2e * 1e-3), "unit": UNIT,
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    layer.close()
    assert fb.fb_get_device_status() == fb.FB_OK

    # roofline of the dominant kernel kind (largest event-timed share)
    hbm, tf, tf_sus, peak_src = _peaks()
    dom = max(prof, key=lambda k: prof[k][1])
    n, tot_ms, byts = prof[dom]
    achieved = (byts / n) / ((tot_ms / n) * 1e-3) / 1e9
    traffic = _ncu_traffic(dom, spec.name)
    roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": f"{peak_src} hbm_gbs",
            "traffic": traffic, "alg_bytes_per_launch": byts / n, "avg_launch_us": 1e3 * tot_ms / n,
            "launches": n}
    kernels = {k: {"launches": v[0], "total_ms_per_step": v[1] / args.steps,
                   "avg_us": (1e3 * v[1] / v[0]) if v[0] else None,
                   "achieved_GBps": (v[2] / (v[1] * 1e-3) / 1e9) if v[1] else None} for k, v in prof.items()}
    n_full = sum(kinds_on) // args.steps
    per_kind = {}
    for kind in (True, False):
        xs = [m for m, k in zip(per_on, kinds_on) if k == kind]
        if xs:
            per_kind["full_step_us" if kind else "reuse_step_us"] = 1e3 * statistics.mean(xs)
    gpu_launches = sum(v[0] for v in prof.values())
    return {
        "metric": METRIC, "value": world * sched.query_tokens / (ms_on * 1e-3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_on,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": spec.dtype,
        "data": "synthetic (seeded; shapes of the pages' diffusion-LM workload)",
        "config": {"workload": _describe(spec), "query_tokens_per_step": sched.query_tokens,
                   "prefix_kernel": args.prefix_kernel,
                   "diffusion_steps_per_step": len(sched.steps), "l2": "flushed (1 GiB write) before every "
                   "diffusion step, outside the timed interval", "parallelism": f"replicas x{world}",
                   "full_steps_per_step": n_full},
        "step_latency": {"mean_us": 1e3 * ms_on / len(sched.steps), **per_kind},
        "timing": "CUDA graph per diffusion step, replayed" if not args.eager else "eager library calls",
        "eager": {"value": world * sched.query_tokens / (ms_eager * 1e-3), "ms_per_step": ms_eager},
        "full_recompute": None if args.profile_run else {"value": world * sched.query_tokens / (ms_full * 1e-3), "ms_per_step": ms_full,
                           "mean_step_us": 1e3 * ms_full / len(sched.steps)},
        "speedup_vs_full_recompute": None if args.profile_run else ms_full / ms_on,
        "e2e": e2e, "roofline": roof, "kernels": kernels, "gpu_launches": gpu_launches // 1,
        "gpu_launches_per_step": gpu_launches / args.steps, "clocks": clk,
    }


def _ncu_traffic(kind, workload):
    """Per-launch DRAM bytes of this kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(f"{kind}:{workload}")
        if not d:
            return None
        src = os.path.join(ROOT, d["source"])
        import hashlib
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return d["dram_bytes_per_launch"] if h == d["source_sha"] else None
    except Exception:
        return None


# ----------------------------------------------------------- CPU baseline ---
def cpu_baseline(spec, budget_s: float):
    """The fp64 oracle on this host's cores over a bounded prefix of the schedule."""
    from oracle import flashblock_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count()
    w = wl.Workload(spec)
    kp, vp = w.prefix_kv()
    kp64, vp64 = orc.to64(kp), orc.to64(vp)
    o = orc.FlashBlockOracle(spec.B, spec.Hq, spec.Hkv, spec.D, spec.Nb,
                             gamma=None if spec.gamma is None else [spec.gamma] * spec.Hq)
    t0 = time.perf_counter()
    n = 0
    for st in w.schedule():
        if st.step == 0:
            o.begin_block()
        o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, st.M, spec.tau,
               None if st.sel is None else st.sel.numpy())
        n += 1
        if st.last_in_block:
            kp64, vp64, _ = orc.kv_append(kp64, vp64, st.prefix_len, orc.to64(st.kin), orc.to64(st.vin))
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": spec.B * spec.Nb * n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {n} diffusion steps of the schedule (all heads), fp64 numpy", "seconds": dt}


def run_reference(args, spec):
    per = []
    last = None
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(spec, budget_s=max(2.0, 20.0 / max(1, args.steps)))
        if i >= args.warmup:
            per.append(r["value"]); last = r
    v = statistics.mean(per)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * spec.B * spec.Nb / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": _describe(spec)},
            "cpu_baseline": {k: last[k] for k in ("kind", "cores", "sample")} | {"value": v, "unit": UNIT},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dllm_8k", choices=list(wl.SPECS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--prefix-kernel", default="auto", choices=["auto", "generic", "tcgen05"])
    ap.add_argument("--eager", action="store_true", help="time eager library calls instead of graph replays")
    ap.add_argument("--profile-run", action="store_true",
                    help="only the reuse-on schedule (no full-recompute, e2e or CPU legs): for ncu captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    spec = wl.get_spec(args.workload)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, spec)))
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    out = run_ours(args, spec, rank, world, device)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.profile_run:
            out["cpu_baseline"] = cpu_baseline(spec, args.cpu_budget)
        print(json.dumps(out))


if __name__ == "__main__":
    main()
