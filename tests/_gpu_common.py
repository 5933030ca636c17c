"""Shared helpers of the GPU parity tests: run a workload schedule through the
C-ABI (libfb via its ctypes binding) and through the fp64 oracle, and compare
them under the stated tolerances.

Tolerances (FlashBlock step, stated for the build): relative to output scale,
err_O = max|O_gpu - O_oracle| / max|O_oracle| and
err_L = max|L_gpu - L_oracle| / max(1, max|L_oracle|), at most 1e-5 for fp32
inputs and 2e-3 for bf16 inputs.  A bf16-stored O may differ by a further half
unit in the last place of the oracle value (its own rounding).
"""
import math

import numpy as np
import torch

from block_diffusion_attention_flashblock_b200 import fb
from block_diffusion_attention_flashblock_b200 import workloads as wl
from oracle import flashblock_oracle as orc

TOL = {"f32": 1e-5, "bf16": 2e-3}
GAMMA_BAND = 2e-3   # decisions are compared only where |sim - gamma| exceeds this


def rel_err(gpu, ref) -> float:
    g = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    scale = np.max(np.abs(r)) if r.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - r)) / scale)


def lse_err(gpu, ref) -> float:
    g = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    both_inf = np.isneginf(g) & np.isneginf(r)
    assert np.array_equal(np.isneginf(g), np.isneginf(r)), "empty rows differ"
    if both_inf.all():
        return 0.0
    d = np.abs(np.where(both_inf, 0.0, g - r))
    return float(np.max(d) / max(1.0, np.max(np.abs(r[~both_inf]))))


def assert_o_close(gpu, ref, tol, what=""):
    e = rel_err(gpu, ref)
    if gpu.dtype == torch.bfloat16:
        g = gpu.double().cpu().numpy(); r = np.asarray(ref, np.float64)
        scale = np.max(np.abs(r))
        half_ulp = np.where(r == 0, 0.0, np.exp2(np.floor(np.log2(np.abs(r) + 1e-300)) - 8))
        ok = np.abs(g - r) <= tol * scale + half_ulp
        assert ok.all(), f"{what}: bf16 O outside tol+half-ulp (rel err {e:.3g})"
        return e
    assert e <= tol, f"{what}: O rel err {e:.3g} > {tol}"
    return e


def assert_lse_close(gpu, ref, tol, what=""):
    e = lse_err(gpu, ref)
    assert e <= tol, f"{what}: LSE err {e:.3g} > {tol}"
    return e


def cuda(t):
    return None if t is None else t.cuda()


class GpuSchedule:
    """Run a WorkloadSpec's block schedule through fb_step on cuda:0."""

    def __init__(self, spec, out_dtype=torch.float32):
        self.spec = spec
        self.w = wl.Workload(spec)
        kp, vp = self.w.prefix_kv()
        self.kp, self.vp = kp.cuda(), vp.cuda()
        s = spec
        dt = s.torch_dtype
        self.q_like = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=dt, device="cuda")
        self.kin_like = torch.empty(s.B, s.Hkv, s.Nb, s.D, dtype=dt, device="cuda")
        self.o_like = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=out_dtype, device="cuda")
        self.out_dtype = out_dtype
        self.layer = fb.FlashBlockLayer(self.q_like, self.kin_like, self.kp, self.o_like, max_prefix=s.lcap,
                                        gamma=s.gamma is not None, sparse=s.sel_k is not None,
                                        max_sel_k=s.sel_k or 0, active=s.lock_rate is not None)
        self.gamma = (torch.full((s.Hq,), s.gamma, dtype=torch.float32, device="cuda")
                      if s.gamma is not None else None)
        self.tau = s.tau if s.tau is not None else fb.FB_TAU_OFF

    def select_mass(self, q, prefix_len):
        """The block's selection by attention mass (fb_select_mass) and the masses."""
        s = self.spec
        k = min(s.sel_k, prefix_len)
        sel = torch.empty(s.B, s.Hq, k, dtype=torch.int32, device="cuda")
        mass = torch.empty(s.B, s.Hq, prefix_len, dtype=torch.float32, device="cuda")
        ws = torch.empty(fb.fb_select_workspace_bytes(self.layer.desc, prefix_len), dtype=torch.uint8, device="cuda")
        fb.fb_select_mass(self.layer.desc, q, self.kp, self.vp, prefix_len, k, sel, ws, mass_out=mass)
        return sel, mass

    def run(self):
        s = self.spec
        o = lse = None
        block_sel = None
        for st in self.w.schedule():
            if st.step == 0:
                self.layer.begin_block()
            q, kin, vin = st.q.cuda(), st.kin.cuda(), st.vin.cuda()
            sel = cuda(st.sel)
            if s.sel_k and s.select == "mass":
                if st.step == 0:
                    block_sel, self.last_mass = self.select_mass(q, st.prefix_len)
                sel = block_sel
                st.sel = block_sel.cpu()   # the oracle steps over the same selection
            if st.active is None or st.step == 0:
                o = torch.empty(s.B, s.Hq, s.Nb, s.D, dtype=self.out_dtype, device="cuda")
                lse = torch.empty(s.B, s.Hq, s.Nb, dtype=torch.float32, device="cuda")
            else:   # locked positions keep the previous step's rows: the same buffers, unwritten
                o, lse = o.clone(), lse.clone()
            reuse = torch.full((s.B, s.Hq), -1, dtype=torch.int8, device="cuda")
            sim = torch.empty(s.B, s.Hq, dtype=torch.float32, device="cuda")
            self.layer.step(q, kin, vin, self.kp, self.vp, st.prefix_len, st.M, self.tau, o, lse,
                            self.gamma, sel, reuse, sim, active=cuda(st.active))
            recomputed = self.layer.last_recomputed()
            torch.cuda.synchronize()
            yield st, o, lse, reuse.cpu(), sim.cpu(), recomputed
            if st.last_in_block:
                fb.fb_kv_append(self.layer.desc, self.kp, self.vp, st.prefix_len, kin, vin)

    def close(self):
        self.layer.close()


class OracleSchedule:
    """The oracle's policy over the same schedule, for all heads or for one
    (b, kv-head) group slice at a time (heads are independent under the policy)."""

    def __init__(self, spec, groups=None):
        self.spec = spec
        s = spec
        self.groups = groups  # None: all heads; else list of (b, kv head)
        self.oracles = {}
        keys = [None] if groups is None else groups
        for key in keys:
            B, Hq, Hkv = (s.B, s.Hq, s.Hkv) if key is None else (1, s.G, 1)
            gam = None if s.gamma is None else [s.gamma] * Hq
            self.oracles[key] = orc.FlashBlockOracle(B, Hq, Hkv, s.D, s.Nb, gamma=gam)
        self.kp = {}
        self.vp = {}

    def _slice(self, key, t, heads_q):
        if key is None:
            return t
        b, g = key
        G = self.spec.G
        return t[b:b + 1, g * G:(g + 1) * G] if heads_q else t[b:b + 1, g:g + 1]

    def init_prefix(self, kp, vp):
        for key in self.oracles:
            self.kp[key] = orc.to64(self._slice(key, kp, False))
            self.vp[key] = orc.to64(self._slice(key, vp, False))

    def step(self, st):
        s = self.spec
        out = {}
        for key, o in self.oracles.items():
            if st.step == 0:
                o.begin_block()
            sel = None if st.sel is None else self._slice(key, st.sel, True).numpy()
            act = None
            if st.active is not None:
                act = st.active.numpy() if key is None else st.active.numpy()[key[0]:key[0] + 1]
            r = o.step(orc.to64(self._slice(key, st.q, True)), orc.to64(self._slice(key, st.kin, False)),
                       orc.to64(self._slice(key, st.vin, False)), self.kp[key], self.vp[key],
                       st.prefix_len, st.M, s.tau, sel, act)
            out[key] = r
            if st.last_in_block:
                self.kp[key], self.vp[key], _ = orc.kv_append(
                    self.kp[key], self.vp[key], st.prefix_len, orc.to64(self._slice(key, st.kin, False)),
                    orc.to64(self._slice(key, st.vin, False)))
        return out

    def gpu_slice(self, key, t):
        """The part of a GPU [B, Hq, ...] tensor that corresponds to an oracle slice."""
        return self._slice(key, t, True)


MASS_TOL = 2e-5   # fp32 mass vs fp64, relative to the head's largest mass


def check_mass_selection(spec, st, gpu_mass, os_):
    """fb_select_mass against the oracle on the sampled groups: the masses
    within MASS_TOL; the selection equal to the oracle's top-k on every key
    whose oracle mass lies outside MASS_TOL of the k-th largest (near-ties at
    the boundary may rank either way in fp32), and a valid top-k on the rest."""
    sel = st.sel.numpy()
    for key in os_.oracles:
        b0, b1, h0, h1 = (0, spec.B, 0, spec.Hq) if key is None else (
            key[0], key[0] + 1, key[1] * spec.G, (key[1] + 1) * spec.G)
        kp = os_.kp[key]
        q64 = orc.to64(st.q[b0:b1, h0:h1])
        M = orc.attention_mass(q64, kp, st.prefix_len, 1 / math.sqrt(spec.D))
        gm = gpu_mass[b0:b1, h0:h1].double().cpu().numpy()
        scale = M.max(axis=2, keepdims=True)
        err = float(np.max(np.abs(gm - M) / scale))
        assert err <= MASS_TOL, f"mass rel err {err:.3g}"
        k = sel.shape[-1]
        ref = orc.select_top_k(M, k)
        for b in range(b1 - b0):
            for h in range(h1 - h0):
                g_sel = sel[b0 + b, h0 + h]
                assert len(g_sel) == k and np.all(np.diff(g_sel) > 0), "selection not ascending and distinct"
                if k == 0:
                    continue
                m = M[b, h]
                kth = np.sort(m)[::-1][k - 1]
                band = MASS_TOL * m.max()
                sure_in = np.flatnonzero(m > kth + band)
                sure_out = np.flatnonzero(m < kth - band)
                assert np.isin(sure_in, g_sel).all(), "a key well above the k-th mass is not selected"
                assert not np.isin(sure_out, g_sel).any(), "a key well below the k-th mass is selected"
                assert np.isin(sure_in, ref[b, h]).all() and not np.isin(sure_out, ref[b, h]).any()


def compare_schedule(spec, groups=None, out_dtype=torch.float32, check_every=1, report=None):
    """Run GPU and oracle side by side; assert parity on every step; return stats."""
    tol = TOL[spec.dtype]
    gs = GpuSchedule(spec, out_dtype)
    os_ = OracleSchedule(spec, groups)
    w = gs.w
    kp, vp = w.prefix_kv()
    os_.init_prefix(kp, vp)
    stats = {"err_o": 0.0, "err_l": 0.0, "steps": 0, "recomputed": [], "sim_err": 0.0, "reuse": []}
    prev_sim = {}
    prev_o = prev_l = None
    for st, o, lse, reuse, sim, recomputed in gs.run():
        if spec.sel_k and spec.select == "mass" and st.step == 0:
            check_mass_selection(spec, st, gs.last_mass, os_)
        ref = os_.step(st)
        if st.active is not None and st.step > 0:
            # locked positions: their rows of O and LSE were not written at all
            for b in range(spec.B):
                locked = np.setdiff1d(np.arange(spec.Nb), st.active[b].numpy())
                assert torch.equal(o[b][:, locked], prev_o[b][:, locked]), f"step {st.step}: a locked row of O changed"
                assert torch.equal(lse[b][:, locked], prev_l[b][:, locked]), f"step {st.step}: a locked LSE changed"
        prev_o, prev_l = o, lse
        for key, r in ref.items():
            stats["recomputed"].append(recomputed)
            assert recomputed == r.recompute, f"step {st.block}.{st.step}: tau decision differs"
            go = os_.gpu_slice(key, o)
            gl = os_.gpu_slice(key, lse)
            greuse = os_.gpu_slice(key, reuse).numpy().astype(bool)
            what = f"{spec.name} block {st.block} step {st.step} group {key}"
            if spec.gamma is not None:
                # decisions at this step come from the previous step's similarity
                if key in prev_sim:
                    live = ~np.isnan(prev_sim[key])
                    assert np.all(np.abs(prev_sim[key][live] - spec.gamma) > GAMMA_BAND), \
                        f"{what}: a similarity lies within {GAMMA_BAND} of gamma; pick another seed"
                gsim = os_.gpu_slice(key, sim).numpy()
                defined = ~np.isnan(r.sim)
                assert np.array_equal(defined, ~np.isnan(gsim)), f"{what}: sim definedness differs"
                if defined.any():
                    stats["sim_err"] = max(stats["sim_err"], float(np.max(np.abs(gsim[defined] - r.sim[defined]))))
                prev_sim[key] = r.sim.copy()
            assert np.array_equal(greuse, r.head_reuse), f"{what}: reuse mask differs"
            stats["reuse"].append(r.head_reuse.mean())
            if st.active is not None:   # compare the active rows (locked rows: checked above)
                b0 = 0 if key is None else key[0]
                rows = st.active.numpy()[b0]
                go, gl = go[:, :, rows], gl[:, :, rows]
                ro, rl = r.o[:, :, rows], r.lse[:, :, rows]
                if key is None and spec.B > 1:   # every batch element has its own positions
                    go = torch.stack([o[b][:, st.active[b].numpy()] for b in range(spec.B)])
                    gl = torch.stack([lse[b][:, st.active[b].numpy()] for b in range(spec.B)])
                    ro = np.stack([r.o[b][:, st.active[b].numpy()] for b in range(spec.B)])
                    rl = np.stack([r.lse[b][:, st.active[b].numpy()] for b in range(spec.B)])
            else:
                ro, rl = r.o, r.lse
            if st.step % check_every == 0 or st.step == spec.steps - 1:
                stats["err_o"] = max(stats["err_o"], assert_o_close(go, ro, tol, what))
                stats["err_l"] = max(stats["err_l"], assert_lse_close(gl, rl, tol, what))
        stats["steps"] += 1
    gs.close()
    if report is not None:
        report(stats)
    return stats
