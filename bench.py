"""Benchmark of the FlashBlock attention step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload dllm_64k_b4] [--extra video_1560,dllm_8k] [--no-e2e]

A timed "step" is one pass of the whole hot path over one workload, by default
the long-context diffusion-LM layer (dllm_64k_b4: B 4, 32 query / 8 KV heads,
head dim 128, prefix 65,536 tokens, blocks of 64 tokens, 16 diffusion steps,
tau = 16), the largest workload that fits one GPU, for each of NL attention
layers, every layer with its own KV cache, cache state and inputs.  Every
diffusion step runs fb_step for each layer in turn under the reuse policy, and
every block ends with fb_kv_append.  NL is chosen so that the layers' KV caches
together exceed twice the L2: as between the layers of a model, each layer's
data has left L2 by the time its next step runs.  L2 is also flushed (a 1 GiB
write) before every timed step, outside the timed interval.

The metric is query tokens per second: B * Nb per layer-step (one fb_step of
one layer, all heads), over all layer-steps of the timed step.  The same
schedule with tau = 0 (every step recomputes over the whole KV cache) is
reported beside it, and the per-step latencies follow from the two.

The whole step is captured once as a CUDA graph (the reuse decisions are taken
on the host while capturing, in schedule order) and replayed between two CUDA
events; the same calls made eagerly are reported under "eager", and "e2e"
repeats the eager pass with every layer-step's inputs copied from pinned host
memory and its outputs read back.

The roofline is that of the dominant kernel, timed L2-cold: the prefix
kernel's launches bracketed by CUDA events on their stream, with L2 flushed
before each round of calls; the in-block call (one kernel) as a graph over
enough distinct input sets that each call's data has left L2.  Its bytes are
the method's (K/V and Q read once, one (A, L) written; split partials and their
merge do not count).  The warm figure (the same call repeated) is reported
beside it.  The other workloads named by --extra are measured the same way
and reported under "workloads".

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
L2_BYTES = 126 << 20


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time: every rank takes part, every rank gets the max."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def n_layers(spec) -> int:
    """Independent layer states stepped in turn: enough that the layers' KV
    caches together exceed twice the L2 (so each layer's data has left L2 by
    the time its next step runs), at least 2, at most 8."""
    kv = 2 * spec.B * spec.Hkv * spec.lcap * spec.D * (4 if spec.dtype == "f32" else 2)
    return int(min(8, max(2, -(-2 * L2_BYTES // kv))))


class Layers:
    """NL attention layers of one workload, each with its own KV cache, cache
    state, per-step inputs and outputs, all resident on the device (plus
    pinned host copies of layer 0's inputs for the end-to-end leg)."""

    def __init__(self, spec, device, nl):
        from block_diffusion_attention_flashblock_b200 import fb
        self.spec, self.nl = spec, nl
        w = wl.Workload(spec)
        kp, vp = w.prefix_kv()
        self.steps = list(w.schedule())
        dt = spec.torch_dtype
        self.L = []
        for _ in range(nl):
            d = dict(kp=kp.to(device), vp=vp.to(device),
                     o=torch.empty(spec.B, spec.Hq, spec.Nb, spec.D, dtype=dt, device=device),
                     lse=torch.empty(spec.B, spec.Hq, spec.Nb, dtype=torch.float32, device=device),
                     x=[dict(q=st.q.to(device), kin=st.kin.to(device), vin=st.vin.to(device),
                             sel=None if st.sel is None else st.sel.to(device),
                             active=None if st.active is None else st.active.to(device)) for st in self.steps])
            d["layer"] = fb.FlashBlockLayer(d["x"][0]["q"], d["x"][0]["kin"], d["kp"], d["o"],
                                            max_prefix=spec.lcap, gamma=spec.gamma is not None,
                                            sparse=spec.sel_k is not None, max_sel_k=spec.sel_k or 0,
                                            active=spec.lock_rate is not None)
            if spec.sel_k and spec.select == "mass":
                # the block's selection by attention mass, made at its step 0
                d["mass_sel"] = torch.empty(spec.B, spec.Hq, spec.sel_k, dtype=torch.int32, device=device)
                d["mass_ws"] = torch.empty(fb.fb_select_workspace_bytes(d["layer"].desc, spec.lcap),
                                           dtype=torch.uint8, device=device)
                for x in d["x"]:
                    x["sel"] = d["mass_sel"]
            self.L.append(d)
        self.host = [dict(q=st.q.pin_memory(), kin=st.kin.pin_memory(), vin=st.vin.pin_memory()) for st in self.steps]
        self.query_tokens = spec.B * spec.Nb * len(self.steps) * nl   # layer-steps x B x Nb

    def close(self):
        for d in self.L:
            d["layer"].close()


def _call_cost(spec):
    """Algorithmic bytes and FLOPs of one library call of each kind, by the
    method's definition: every input read once, every output written once;
    split-KV partials, their merge and re-reads do not count."""
    s = spec
    e = 4 if s.dtype == "f32" else 2
    rows = s.B * s.Hq * s.Nb
    P = s.prefix0
    q = rows * s.D * e
    part = rows * (s.D + 1) * 4                       # one fp32 (A, L)
    kv_prefix = 2 * s.B * s.Hkv * P * s.D * e
    kv_block = 2 * s.B * s.Hkv * s.Nb * s.D * e
    out = rows * (s.D * e + 4)                        # O in the input dtype, LSE fp32
    return {
        "prefix_attention": {"bytes": kv_prefix + q + part, "flops": 4.0 * rows * P * s.D},
        "inblock_merge": {"bytes": q + kv_block + part + out, "flops": 4.0 * rows * s.Nb * s.D},
    }


def measure_workload(args, spec, rank, world, device, headline):
    """Run and time one workload; returns the fields of its JSON record."""
    from block_diffusion_attention_flashblock_b200 import fb
    torch.cuda.set_device(device)
    nl = n_layers(spec)
    S = Layers(spec, device, nl)
    s = spec
    gamma = torch.full((s.Hq,), s.gamma, device=device) if s.gamma is not None else None
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    nsteps = len(S.steps)

    def schedule(tau):
        """The whole schedule: per diffusion step, every layer's fb_step (and at
        a block's end its fb_kv_append).  Returns the recompute decisions."""
        rec = []
        for t, st in enumerate(S.steps):
            for li, d in enumerate(S.L):
                x = d["x"][t]
                if st.step == 0:
                    d["layer"].begin_block()
                if st.step == 0 and "mass_sel" in d:
                    fb.fb_select_mass(d["layer"].desc, x["q"], d["kp"], d["vp"], st.prefix_len, s.sel_k,
                                      d["mass_sel"], d["mass_ws"])
                d["layer"].step(x["q"], x["kin"], x["vin"], d["kp"], d["vp"], st.prefix_len, st.M, tau, d["o"],
                                d["lse"], gamma, x["sel"], active=x["active"])
                if st.last_in_block:
                    fb.fb_kv_append(d["layer"].desc, d["kp"], d["vp"], st.prefix_len, x["kin"], x["vin"])
            rec.append(S.L[0]["layer"].last_recomputed())
        return rec

    # End to end: every layer-step's Q, K_in and V_in cross from pinned host
    # memory and its O and LSE go back, pipelined: the host-to-device copies
    # run ahead on their own stream (each step has its own device inputs), the
    # device-to-host copies on another, and the library calls on the timed
    # stream wait only for their own inputs and for the read-back of the
    # output buffer they reuse (two per layer, one with active-query subsets,
    # whose locked rows keep the previous step's output).
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    nbuf = 1 if s.lock_rate is not None else 2
    for d in S.L:
        d["ob"] = [d["o"]] + [torch.empty_like(d["o"]) for _ in range(nbuf - 1)]
        d["lb"] = [d["lse"]] + [torch.empty_like(d["lse"]) for _ in range(nbuf - 1)]

    def schedule_e2e(tau):
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        ev_in = {}
        with torch.cuda.stream(s_in):
            for t, st in enumerate(S.steps):
                h = S.host[t]
                for li, d in enumerate(S.L):
                    x = d["x"][t]
                    x["q"].copy_(h["q"], non_blocking=True)
                    x["kin"].copy_(h["kin"], non_blocking=True)
                    x["vin"].copy_(h["vin"], non_blocking=True)
                    ev_in[t, li] = torch.cuda.Event()
                    ev_in[t, li].record(s_in)
        ev_read = {}
        for t, st in enumerate(S.steps):
            for li, d in enumerate(S.L):
                x = d["x"][t]
                b = t % nbuf
                if st.step == 0:
                    d["layer"].begin_block()
                stream.wait_event(ev_in[t, li])
                if (li, b) in ev_read:
                    stream.wait_event(ev_read[li, b])
                if st.step == 0 and "mass_sel" in d:
                    fb.fb_select_mass(d["layer"].desc, x["q"], d["kp"], d["vp"], st.prefix_len, s.sel_k,
                                      d["mass_sel"], d["mass_ws"])
                d["layer"].step(x["q"], x["kin"], x["vin"], d["kp"], d["vp"], st.prefix_len, st.M, tau,
                                d["ob"][b], d["lb"][b], gamma, x["sel"], active=x["active"])
                if st.last_in_block:
                    fb.fb_kv_append(d["layer"].desc, d["kp"], d["vp"], st.prefix_len, x["kin"], x["vin"])
                done = torch.cuda.Event()
                done.record(stream)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    ho[t].copy_(d["ob"][b], non_blocking=True)
                    hl[t].copy_(d["lb"][b], non_blocking=True)
                ev_read[li, b] = torch.cuda.Event()
                ev_read[li, b].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    def timed_region(fn, steps, warmup, do_flush=True):
        """Flush L2, then time fn() between two CUDA events; max over ranks."""
        for _ in range(warmup):
            if do_flush:
                flush.zero_()
            fn()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ev = []
        for _ in range(steps):
            if do_flush:
                flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / steps, world, device)

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            out = fn()
        torch.cuda.synchronize()
        return g, out

    tau_on = s.tau if s.tau is not None else fb.FB_TAU_OFF
    ho = [torch.empty(S.L[0]["o"].shape, dtype=S.L[0]["o"].dtype, pin_memory=True) for _ in S.steps]
    hl = [torch.empty(S.L[0]["lse"].shape, dtype=torch.float32, pin_memory=True) for _ in S.steps]
    clk = None
    steps = args.steps if headline else max(3, args.steps // 2)

    # eager library calls
    ms_eager = timed_region(lambda: schedule(tau_on), steps, args.warmup)
    # the whole schedule as one CUDA graph (the headline number)
    g_on, rec_on = graph_of(lambda: schedule(tau_on))
    if headline:
        props = torch.cuda.get_device_properties(device)
        try:
            smi_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        except AttributeError:
            smi_id = str(device.index)
        clocks = ClockSampler(smi_id)
        clocks.start()
    ms_on = timed_region(g_on.replay, steps, args.warmup)
    if headline:
        clk = clocks.stop()
    del g_on
    # per-kernel launch counts and algorithmic bytes (one eager pass, events per launch)
    fb.fb_profile_read(reset=True)
    fb.fb_profile_enable(True)
    schedule(tau_on)
    torch.cuda.synchronize()
    fb.fb_profile_enable(False)
    prof = fb.fb_profile_read(reset=True)
    ms_full = None
    if not args.profile_run:
        g_full, _ = graph_of(lambda: schedule(0))
        ms_full = timed_region(g_full.replay, steps, args.warmup)
        del g_full
    e2e = None
    if headline and not args.no_e2e and not args.profile_run:
        ms_e2e = timed_region(lambda: schedule_e2e(tau_on), steps, args.warmup)
        h2d = nl * sum(h["q"].numel() * h["q"].element_size() + 2 * h["kin"].numel() * h["kin"].element_size()
                       for h in S.host)
        d2h = nl * (sum(x.numel() * x.element_size() for x in ho) + sum(x.numel() * x.element_size() for x in hl))
        e2e = {"value": world * S.query_tokens / (ms_e2e * 1e-3), "unit": UNIT, "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "eager calls; every layer-step copies its Q, K_in, V_in from pinned host memory and reads "
                       "its O and LSE back, inside the timed region; the copies run on two copy streams, "
                       "overlapped with the calls"}

    # Reuse-step latency, measured directly: after one full step per layer, a
    # graph of R rounds over the layers of a step that reuses the cache (the
    # block's step 1 inputs, M = 0 with tau on; the gamma gate, where on,
    # still decides per head), L2 flushed before it.
    R = 4
    st1 = S.steps[1] if len(S.steps) > 1 else S.steps[0]
    for d in S.L:
        x = d["x"][0]
        d["layer"].begin_block()
        if "mass_sel" in d:
            fb.fb_select_mass(d["layer"].desc, x["q"], d["kp"], d["vp"], S.steps[0].prefix_len, s.sel_k,
                              d["mass_sel"], d["mass_ws"])
        d["layer"].step(x["q"], x["kin"], x["vin"], d["kp"], d["vp"], S.steps[0].prefix_len, 0, 0, d["o"], d["lse"],
                        gamma, x["sel"], active=x["active"])

    def reuse_round():
        for d in S.L:
            x = d["x"][1 if len(S.steps) > 1 else 0]
            d["layer"].step(x["q"], x["kin"], x["vin"], d["kp"], d["vp"], st1.prefix_len, 0, tau_on, d["o"],
                            d["lse"], gamma, x["sel"], active=x["active"])

    g_reuse, _ = graph_of(lambda: [reuse_round() for _ in range(R)])
    reuse_recomputed = S.L[0]["layer"].last_recomputed()
    ms_reuse = timed_region(g_reuse.replay, steps, args.warmup)
    del g_reuse

    # ---- per-kind call and kernel durations --------------------------------
    P = S.steps[0].prefix_len
    cost = _call_cost(s)
    parts = []
    for d in S.L:
        a = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=torch.float32, device=device)
        l = torch.empty(s.B, s.Hq, s.Nb, dtype=torch.float32, device=device)
        ws = torch.empty(max(16, fb.fb_outblock_workspace_bytes(d["layer"].desc, P)), dtype=torch.uint8,
                         device=device)
        parts.append((a, l, ws))

    def call_prefix():
        for d, (a, l, ws) in zip(S.L, parts):
            x = d["x"][0]
            fb.fb_attn_outblock(d["layer"].desc, x["q"], d["kp"], d["vp"], P, a, l, ws)

    call_prefix()
    torch.cuda.synchronize()
    # distinct in-block input sets, enough that together they exceed twice the
    # L2, so a pass over them finds each call's data cold
    ib_bytes = cost["inblock_merge"]["bytes"]
    n_sets = int(min(512, max(nl, -(-2 * L2_BYTES // ib_bytes))))
    x0 = S.L[0]["x"][0]
    a0, l0, _ = parts[0]
    sets = []
    for i in range(n_sets):
        sets.append(dict(q=x0["q"].clone(), kin=x0["kin"].clone(), vin=x0["vin"].clone(), a=a0.clone(),
                         l=l0.clone(), o=torch.empty_like(S.L[0]["o"]), lse=torch.empty_like(S.L[0]["lse"])))
    desc0 = S.L[0]["layer"].desc

    def call_inblock_set(z):
        fb.fb_attn_inblock(desc0, z["q"], z["kin"], z["vin"], z["o"], z["lse"], [z["a"]], [z["l"]])

    per_kind = {}
    # prefix: the kernel alone, cold (events per launch from the profiling
    # hook, L2 flushed before each round over the layers), and the whole call
    # (kernel + merge of its split parts) warm, as a graph of repeated calls
    fb.fb_profile_read(reset=True)
    for r in range(R + 1):
        flush.zero_()
        torch.cuda.synchronize()
        fb.fb_profile_enable(r > 0)
        call_prefix()
        torch.cuda.synchronize()
    fb.fb_profile_enable(False)
    pk = fb.fb_profile_read(reset=True)
    n_prefix_launch = pk["prefix_attention"][0]
    us_prefix_cold = 1e3 * pk["prefix_attention"][1] / max(1, n_prefix_launch)
    g, _ = graph_of(lambda: [call_prefix() for _ in range(R)])
    ms = timed_region(g.replay, steps, args.warmup)
    del g
    us_prefix_call_warm = 1e3 * ms / (R * nl)
    G = s.Hq // s.Hkv
    tiles_per_kv = -(-G // (128 // s.Nb)) if s.Nb <= 128 else G * -(-s.Nb // 128)
    kname = ("attn generic" if not (s.dtype == "bf16" and s.D == 128) else
             "attn_pair_kernel (tcgen05, two query tiles per CTA) + pair_merge_kernel" if tiles_per_kv >= 2 else
             "attn_tc_kernel (tcgen05) + merge of its key splits")
    per_kind["prefix_attention"] = {
        "call": "fb_attn_outblock", "kernel": kname,
        "kernels_per_call": (pk["prefix_attention"][0] + pk["aux"][0]) / (R * nl),
        "avg_launch_us_cold": us_prefix_cold, "avg_call_us_warm": us_prefix_call_warm,
        "alg_bytes_per_launch": cost["prefix_attention"]["bytes"],
        "alg_flops_per_launch": cost["prefix_attention"]["flops"],
        "timing": f"cold: CUDA events around each of {R * nl} kernel launches, L2 flushed before each round of "
                  f"{nl}; warm: one graph of {R * nl} calls (kernel + merge of its parts)"}
    # in-block: a graph over n_sets distinct input sets (cold), and a graph of
    # the same set repeated (warm)
    g, _ = graph_of(lambda: [call_inblock_set(z) for z in sets])
    ms_cold = timed_region(g.replay, steps, args.warmup)
    del g
    g, _ = graph_of(lambda: [call_inblock_set(sets[0]) for _ in range(n_sets)])
    ms_warm = timed_region(g.replay, steps, args.warmup)
    del g
    fb.fb_profile_read(reset=True)
    fb.fb_profile_enable(True)
    call_inblock_set(sets[0])
    torch.cuda.synchronize()
    fb.fb_profile_enable(False)
    pk_ib = fb.fb_profile_read(reset=True)
    per_kind["inblock_merge"] = {
        "call": "fb_attn_inblock with one cached external part" + (
            "" if s.Nb <= 64 else " (above 64-token blocks this public call runs the generic kernel; fb_step "
                                  "runs the tcgen05 pass)"),
        "kernels_per_call": sum(v[0] for v in pk_ib.values()),
        "avg_launch_us_cold": 1e3 * ms_cold / n_sets, "avg_call_us_warm": 1e3 * ms_warm / n_sets,
        "alg_bytes_per_launch": cost["inblock_merge"]["bytes"],
        "alg_flops_per_launch": cost["inblock_merge"]["flops"],
        "timing": f"cold: one graph over {n_sets} distinct input sets (together > 2x L2), L2 flushed before; "
                  f"warm: one graph of {n_sets} calls on one set"}
    del sets
    assert fb.fb_get_device_status() == fb.FB_OK
    S.close()

    hbm, tf, tf_sus, peak_src = _peaks()
    ridge = tf * 1e12 / (hbm * 1e9)
    for k, v in per_kind.items():
        for tag in ("cold", "warm"):
            t = v["avg_launch_us_cold"] if tag == "cold" else v["avg_call_us_warm"]
            v[f"achieved_GBps_{tag}"] = v["alg_bytes_per_launch"] / (t * 1e-6) / 1e9
            v[f"achieved_TFLOPs_{tag}"] = v["alg_flops_per_launch"] / (t * 1e-6) / 1e12
    # the dominant kernel: its launches in the schedule x its cold launch duration
    share = {k: prof[k][0] * per_kind[k]["avg_launch_us_cold"] for k in per_kind}
    total = sum(share.values()) or 1.0
    dom = max(share, key=share.get)
    pkd = per_kind[dom]
    traffic = _ncu_traffic(dom, spec.name)
    tensor = pkd["alg_flops_per_launch"] / pkd["alg_bytes_per_launch"] > ridge
    roof = {"kernel": dom, "call": pkd["call"], "bound": "tensor" if tensor else "hbm",
            "achieved": pkd["achieved_TFLOPs_cold"] if tensor else pkd["achieved_GBps_cold"],
            "peak": tf if tensor else hbm, "unit": "TFLOP/s" if tensor else "GB/s",
            "frac": pkd["achieved_TFLOPs_cold"] / tf if tensor else pkd["achieved_GBps_cold"] / hbm,
            "peak_source": f"{peak_src} " + ("bf16_tflops (burst)" if tensor else "hbm_gbs (burst)"),
            "frac_hbm": pkd["achieved_GBps_cold"] / hbm, "frac_tensor": pkd["achieved_TFLOPs_cold"] / tf,
            "frac_warm": (pkd["achieved_TFLOPs_warm"] / tf if tensor else pkd["achieved_GBps_warm"] / hbm),
            "traffic": traffic, "alg_bytes_per_launch": pkd["alg_bytes_per_launch"],
            "alg_flops_per_launch": pkd["alg_flops_per_launch"], "avg_launch_us": pkd["avg_launch_us_cold"],
            "share_of_kernel_time": share[dom] / total, "timing": pkd["timing"]}
    kernels = {k: {"launches_per_step": v[0], "alg_bytes_per_step": v[2]} for k, v in prof.items()}
    n_full = sum(rec_on)
    layer_steps = nsteps * nl
    step_lat = {"mean_us": 1e3 * ms_on / layer_steps}
    if ms_full is not None:
        step_lat["full_step_us"] = 1e3 * ms_full / layer_steps
    step_lat["reuse_step_us"] = 1e3 * ms_reuse / (R * nl)
    if reuse_recomputed:
        step_lat["reuse_step_note"] = "the gate recomputed at least one head in the measured reuse step"
    gpu_launches = sum(v[0] for v in prof.values())
    return {
        "value": world * S.query_tokens / (ms_on * 1e-3), "ms_per_step": ms_on, "steps": steps,
        "dtype": spec.dtype,
        "config": {"workload": _describe(spec), "layers": nl,
                   "query_tokens_per_step": S.query_tokens,
                   "prefix_kernel": args.prefix_kernel, "diffusion_steps_per_layer": nsteps,
                   "programmatic_dependent_launch": not args.no_pdl, "inblock_loads": args.inblock_loads,
                   "inblock_kernel": args.inblock_kernel,
                   "l2": f"flushed (1 GiB write) before every timed step; inside it {nl} layers with their own "
                         f"KV caches are stepped in turn, so each layer's data has left L2 when it runs",
                   "parallelism": f"replicas x{world}", "full_steps_per_layer": n_full},
        "step_latency": step_lat,
        "eager": {"value": world * S.query_tokens / (ms_eager * 1e-3), "ms_per_step": ms_eager},
        "full_recompute": None if ms_full is None else {
            "value": world * S.query_tokens / (ms_full * 1e-3), "ms_per_step": ms_full,
            "mean_step_us": 1e3 * ms_full / layer_steps},
        "speedup_vs_full_recompute": None if ms_full is None else ms_full / ms_on,
        "e2e": e2e, "roofline": roof, "per_call": per_kind, "kernels": kernels,
        "gpu_launches_per_step": gpu_launches, "clocks": clk,
    }


def run_ours(args, spec, rank, world, device):
    from block_diffusion_attention_flashblock_b200 import fb
    torch.cuda.set_device(device)
    fb.fb_debug_set_prefix_kernel({"auto": 0, "generic": 1, "tcgen05": 2, "tcgen05-nocluster": 3,
                                   "tcgen05-cluster": 4}[args.prefix_kernel])
    fb.fb_debug_set_pdl(not args.no_pdl)
    fb.fb_debug_set_inblock_loads(args.inblock_loads == "bulk")
    fb.fb_debug_set_inblock_kernel(1 if args.inblock_kernel == "paired" else 0)
    r = measure_workload(args, spec, rank, world, device, headline=True)
    out = {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": r["dtype"],
        "data": "synthetic (seeded; shapes of the pages' diffusion-LM and video workloads)",
        "config": r["config"], "step_latency": r["step_latency"],
        "timing": "one CUDA graph of the whole schedule (all layers), replayed; CUDA events around each replay",
    }
    for k in ("eager", "full_recompute", "speedup_vs_full_recompute", "e2e", "roofline", "per_call", "kernels",
              "clocks"):
        out[k] = r[k]
    out["gpu_launches"] = r["gpu_launches_per_step"] * args.steps
    out["gpu_launches_per_step"] = r["gpu_launches_per_step"]
    extras = {}
    for name in [n for n in (args.extra or "").split(",") if n and n != spec.name]:
        e = measure_workload(args, wl.get_spec(name), rank, world, device, headline=False)
        extras[name] = {k: e[k] for k in ("value", "ms_per_step", "steps", "dtype", "step_latency",
                                          "speedup_vs_full_recompute", "roofline", "per_call")}
        extras[name]["workload"] = e["config"]["workload"]
        extras[name]["layers"] = e["config"]["layers"]
    if extras:
        out["workloads"] = extras
    return out


def kernels_only(spec, device, n):
    """N full steps then N reuse steps of one layer (the first block's steps
    0 and 1 at its size), with an L2 flush before each: the launches an ncu
    capture of the hot kernels needs, in the configuration bench.py times."""
    from block_diffusion_attention_flashblock_b200 import fb
    torch.cuda.set_device(device)
    S = Layers(spec, device, 1)
    d = S.L[0]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    gamma = torch.full((spec.Hq,), spec.gamma, device=device) if spec.gamma is not None else None
    st0 = S.steps[0]
    x = d["x"][0]
    if "mass_sel" in d:
        fb.fb_select_mass(d["layer"].desc, x["q"], d["kp"], d["vp"], st0.prefix_len, spec.sel_k, d["mass_sel"],
                          d["mass_ws"])
    for tau in (0, fb.FB_TAU_OFF):   # every step recomputes; then every step reuses the cache
        for _ in range(n):
            flush.zero_()
            d["layer"].step(x["q"], x["kin"], x["vin"], d["kp"], d["vp"], st0.prefix_len, 0, tau, d["o"], d["lse"],
                            gamma, x["sel"], active=x["active"])
    torch.cuda.synchronize()
    assert fb.fb_get_device_status() == fb.FB_OK
    S.close()
    print(json.dumps({"kernels_only": spec.name, "full_steps": n, "reuse_steps": n}))


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
    sel = None
    for st in w.schedule():
        if st.step == 0:
            o.begin_block()
            if spec.sel_k and spec.select == "mass":
                mass = orc.attention_mass(orc.to64(st.q), kp64, st.prefix_len, 1.0 / np.sqrt(spec.D))
                sel = orc.select_top_k(mass, spec.sel_k)
        if st.sel is not None:
            sel = st.sel.numpy()
        o.step(orc.to64(st.q), orc.to64(st.kin), orc.to64(st.vin), kp64, vp64, st.prefix_len, st.M, spec.tau,
               sel, None if st.active is None else st.active.numpy())
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
    ap.add_argument("--workload", default="dllm_64k_b4", choices=list(wl.SPECS))
    ap.add_argument("--extra", default="video_1560,dllm_8k",
                    help="comma-separated workloads also measured and reported under 'workloads' ('' for none)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-pdl", action="store_true", help="launch kernels in plain stream order")
    ap.add_argument("--inblock-loads", default="cpasync", choices=["cpasync", "bulk"],
                    help="how the small in-block kernel loads its rows")
    ap.add_argument("--inblock-kernel", default="auto", choices=["auto", "paired"],
                    help="the kernel of block-internal passes")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--prefix-kernel", default="auto", choices=["auto", "generic", "tcgen05", "tcgen05-nocluster", "tcgen05-cluster"])
    ap.add_argument("--kernels-only", type=int, default=0, metavar="N",
                    help="run N full and N reuse steps of one layer of the workload, untimed, and exit "
                         "(a small case for ncu captures)")
    ap.add_argument("--profile-run", action="store_true",
                    help="only the reuse-on schedule (no full-recompute, e2e or CPU legs): for ncu captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    if args.profile_run or args.kernels_only:
        args.extra = ""
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
    if args.kernels_only:
        kernels_only(spec, device, args.kernels_only)
        return
    out = run_ours(args, spec, rank, world, device)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.profile_run:
            out["cpu_baseline"] = cpu_baseline(spec, args.cpu_budget)
        print(json.dumps(out))


if __name__ == "__main__":
    main()
