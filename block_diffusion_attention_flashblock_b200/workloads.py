"""Seeded synthetic inputs for the FlashBlock attention step.

This module draws the tensors a block-diffusion attention layer sees: the
prefix KV cache, the current block's Q/K/V at each diffusion step, the count M
of tokens updated between steps, per-head perturbation scales for the video
workload, and the sparse-attention key selection.  It holds none of the
method's arithmetic (no attention, merge, gate or cache logic): the CPU oracle
and the CUDA library are both fed from here, and neither one is imported.

The workloads restate the five shapes of the FlashBlock pages' experiments
("FlashBlock: Attention Caching for Efficient Long-Context Block Diffusion",
section "Résultats Expérimentaux": diffusion LMs with small blocks, long
context, video frames, sparse attention at low density).  No dataset item is
reproduced; every value is a seeded pseudo-random draw.

Conventions
-----------
* Tensors are torch CPU tensors, row-major [B, H, T, D] with D contiguous.
* bf16 workloads draw fp32 normals and round them to bf16 (round to nearest
  even, torch cast).  An updated token is ``bf16(float(old) + noise)``.
* Sub-streams: ``numpy.random.Generator(PCG64(SeedSequence(seed, spawn_key=
  (block, step, tensor))))`` so any single tensor can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Iterator, Optional, Tuple

import numpy as np
import torch

# tensor codes of the sub-streams
_T_PREFIX_K, _T_PREFIX_V, _T_Q, _T_K, _T_V = 0, 1, 2, 3, 4
_T_M, _T_POS, _T_NQ, _T_NK, _T_NV, _T_SIGMA, _T_SCORE, _T_LOCK = 5, 6, 7, 8, 9, 10, 11, 12

INT32_MAX = 2**31 - 1


@dataclass(frozen=True)
class WorkloadSpec:
    """One attention layer's block-diffusion schedule."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    prefix0: int          # prefix (KV cache) length when block 0 starts
    Nb: int               # block length (query tokens per step)
    steps: int            # diffusion steps per block
    blocks: int           # consecutive blocks; the cache grows by Nb each
    dtype: str            # "f32" or "bf16"
    std: float            # std of the Q/K/V draws
    m_model: Tuple        # ("uniform", lo, hi) | ("binomial", n, p) | ("all",)
    pert_std: Optional[float] = None          # noise std of an updated token
    sigma_range: Optional[Tuple[float, float]] = None  # per-head noise std range
    tau: Optional[int] = None                 # None: tau gate off
    gamma: Optional[float] = None             # None: gamma gate off
    sel_k: Optional[int] = None               # sparse: keys kept per query head
    lock_rate: Optional[float] = None         # active-query subsets: share of the still-active
                                              # positions that lock at each step (None: all active)
    select: str = "score"                     # sparse: "score" (seeded scores, drawn here) or "mass"
                                              # (top-k attention mass of the block's first queries,
                                              # computed by the caller at each block's step 0)
    seed: int = 2026_0000
    sigma_redraws: Tuple[Tuple[int, int], ...] = field(default=())
    """(block, head) pairs whose sigma is redrawn from the next sub-seed, to keep
    the gamma decision away from its threshold.  Empty for every workload here:
    the parity tests assert that each similarity they compare decisions on lies
    outside a band around gamma, and none has needed a redraw."""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def lcap(self) -> int:
        return self.prefix0 + self.blocks * self.Nb

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


# The five workloads.  Names say what they are.
SPECS = {
    "tiny_f32": WorkloadSpec(
        name="tiny_f32", B=1, Hq=4, Hkv=4, D=64, prefix0=256, Nb=32, steps=4,
        blocks=1, dtype="f32", std=1.0, m_model=("uniform", 0, 8),
        pert_std=0.05, tau=4, seed=2026_0000),
    "dllm_8k": WorkloadSpec(
        name="dllm_8k", B=1, Hq=32, Hkv=8, D=128, prefix0=8192, Nb=32, steps=8,
        blocks=4, dtype="bf16", std=0.5, m_model=("binomial", 32, 0.15),
        pert_std=0.05, tau=8, seed=2026_0001),
    "dllm_64k_b4": WorkloadSpec(
        name="dllm_64k_b4", B=4, Hq=32, Hkv=8, D=128, prefix0=65536, Nb=64,
        steps=16, blocks=1, dtype="bf16", std=0.5,
        m_model=("binomial", 64, 0.1), pert_std=0.05, tau=16, seed=2026_0002),
    # the sparse layer with its keys chosen by attention mass (NEXT-3): the
    # top 2048 prefix keys per head by the mass the block's first queries put
    # on them, computed at each block's start
    "sparse_32k_mass": WorkloadSpec(
        name="sparse_32k_mass", B=1, Hq=32, Hkv=8, D=128, prefix0=32768,
        Nb=32, steps=8, blocks=1, dtype="bf16", std=0.5,
        m_model=("binomial", 32, 0.15), pert_std=0.05, tau=8, sel_k=2048, select="mass",
        seed=2026_0080),
    # context-length sweep of the long-context shape at B = 1 (the pages'
    # latency-growth claim, 100k to 800k tokens of context)
    **{f"dllm_ctx_{n // 1000}k": WorkloadSpec(
        name=f"dllm_ctx_{n // 1000}k", B=1, Hq=32, Hkv=8, D=128, prefix0=n, Nb=64,
        steps=16, blocks=1, dtype="bf16", std=0.5,
        m_model=("binomial", 64, 0.1), pert_std=0.05, tau=16, seed=2026_0010 + i)
       for i, n in enumerate((100_000, 200_000, 400_000, 800_000))},
    # small blocks (NEXT-2): the dllm_8k layer with blocks of 4 tokens; tau 2
    # reuses while at most one token changed, about as often as dllm_8k's tau 8
    "dllm_8k_nb4": WorkloadSpec(
        name="dllm_8k_nb4", B=1, Hq=32, Hkv=8, D=128, prefix0=8192, Nb=4, steps=8,
        blocks=4, dtype="bf16", std=0.5, m_model=("binomial", 4, 0.15),
        pert_std=0.05, tau=2, seed=2026_0020),
    # active-query subsets (NEXT-4): the dllm_8k layer where a quarter of the
    # still-active block positions lock at every step (32, 24, 18, 13, 10, 8,
    # 6, 4 active); only active positions change and are recomputed
    "dllm_8k_lock": WorkloadSpec(
        name="dllm_8k_lock", B=1, Hq=32, Hkv=8, D=128, prefix0=8192, Nb=32, steps=8,
        blocks=4, dtype="bf16", std=0.5, m_model=("binomial", 32, 0.15),
        pert_std=0.05, tau=8, lock_rate=0.25, seed=2026_0040),
    "video_1560": WorkloadSpec(
        name="video_1560", B=1, Hq=24, Hkv=24, D=128, prefix0=31200, Nb=1560,
        steps=8, blocks=1, dtype="bf16", std=1.0, m_model=("all",),
        sigma_range=(0.01, 0.3), gamma=0.95, seed=2026_0003),
    "sparse_32k_k2048": WorkloadSpec(
        name="sparse_32k_k2048", B=1, Hq=32, Hkv=8, D=128, prefix0=32768,
        Nb=32, steps=8, blocks=1, dtype="bf16", std=0.5,
        m_model=("binomial", 32, 0.15), pert_std=0.05, tau=8, sel_k=2048,
        seed=2026_0004),
    # sparse density sweep (NEXT-3, top-k by score only): 20, 30 and 40 % of
    # the 32k prefix selected
    **{f"sparse_32k_d{pct}": WorkloadSpec(
        name=f"sparse_32k_d{pct}", B=1, Hq=32, Hkv=8, D=128, prefix0=32768,
        Nb=32, steps=8, blocks=1, dtype="bf16", std=0.5,
        m_model=("binomial", 32, 0.15), pert_std=0.05, tau=8, sel_k=32768 * pct // 100,
        seed=2026_0030 + pct)
       for pct in (20, 30, 40)},
}


def _rng(spec: WorkloadSpec, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(spec.seed, spawn_key=tuple(int(k) for k in key))
    return np.random.Generator(np.random.PCG64(ss))


def _cast(x: np.ndarray, spec: WorkloadSpec) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(spec.torch_dtype)


def _normal(spec, shape, std, *key) -> torch.Tensor:
    g = _rng(spec, *key)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return _cast(x, spec)


@dataclass
class Step:
    block: int
    step: int
    prefix_len: int
    M: int                      # tokens updated since the previous step (0 at step 0)
    q: torch.Tensor             # [B, Hq, Nb, D]
    kin: torch.Tensor           # [B, Hkv, Nb, D]
    vin: torch.Tensor           # [B, Hkv, Nb, D]
    sel: Optional[torch.Tensor]  # int32 [B, Hq, sel_k] ascending, or None
    last_in_block: bool
    active: Optional[torch.Tensor] = None   # int32 [B, n_active] ascending block positions, or None (all)


class Workload:
    """Deterministic generator for one WorkloadSpec."""

    def __init__(self, spec: WorkloadSpec):
        self.spec = spec

    # -- prefix cache -----------------------------------------------------
    def prefix_kv(self) -> Tuple[torch.Tensor, torch.Tensor]:
        """Kp, Vp of shape [B, Hkv, lcap, D]; rows [0, prefix0) drawn, rest 0."""
        s = self.spec
        kp = torch.zeros(s.B, s.Hkv, s.lcap, s.D, dtype=s.torch_dtype)
        vp = torch.zeros_like(kp)
        for b in range(s.B):
            for h in range(s.Hkv):
                # one sub-stream per (b, h) keeps peak host memory small
                kp[b, h, :s.prefix0] = _normal(s, (s.prefix0, s.D), s.std, _T_PREFIX_K, b, h)
                vp[b, h, :s.prefix0] = _normal(s, (s.prefix0, s.D), s.std, _T_PREFIX_V, b, h)
        return kp, vp

    # -- block inputs -------------------------------------------------------
    def block_start(self, blk: int):
        s = self.spec
        q = _normal(s, (s.B, s.Hq, s.Nb, s.D), s.std, _T_Q, blk)
        k = _normal(s, (s.B, s.Hkv, s.Nb, s.D), s.std, _T_K, blk)
        v = _normal(s, (s.B, s.Hkv, s.Nb, s.D), s.std, _T_V, blk)
        return q, k, v

    def head_sigmas(self, blk: int) -> np.ndarray:
        """Per-head noise std for the video workload, shape [Hq] (fp32)."""
        s = self.spec
        lo, hi = s.sigma_range
        sig = _rng(s, _T_SIGMA, blk).uniform(lo, hi, size=s.Hq).astype(np.float32)
        for (b_, h_) in s.sigma_redraws:
            if b_ == blk:
                sig[h_] = _rng(s, _T_SIGMA, blk, 1 + h_).uniform(lo, hi)
        return sig

    def draw_M(self, blk: int, step: int) -> int:
        s = self.spec
        g = _rng(s, _T_M, blk, step)
        kind = s.m_model[0]
        if kind == "uniform":
            return int(g.integers(s.m_model[1], s.m_model[2] + 1))
        if kind == "binomial":
            return int(g.binomial(s.m_model[1], s.m_model[2]))
        if kind == "all":
            return s.Nb
        raise ValueError(kind)

    def step_update(self, blk: int, step: int, q, kin, vin, active=None):
        """Inputs of diffusion step ``step`` (>= 1) from those of step - 1.
        With ``active`` ([B, n] positions), only active positions change and
        M counts updated active positions (at most n)."""
        s = self.spec
        M = self.draw_M(blk, step)
        if active is not None:
            M = min(M, active.shape[1])
        q = q.clone(); kin = kin.clone(); vin = vin.clone()
        if s.m_model[0] == "all":
            sig = self.head_sigmas(blk)
            nq = _rng(s, _T_NQ, blk, step).standard_normal(
                (s.B, s.Hq, s.Nb, s.D), dtype=np.float32) * sig[None, :, None, None]
            nk = _rng(s, _T_NK, blk, step).standard_normal(
                (s.B, s.Hkv, s.Nb, s.D), dtype=np.float32) * sig[None, ::s.G, None, None]
            nv = _rng(s, _T_NV, blk, step).standard_normal(
                (s.B, s.Hkv, s.Nb, s.D), dtype=np.float32) * sig[None, ::s.G, None, None]
            q = _cast(q.float().numpy() + nq, s)
            kin = _cast(kin.float().numpy() + nk, s)
            vin = _cast(vin.float().numpy() + nv, s)
            return M, q, kin, vin
        if M == 0:
            return 0, q, kin, vin
        gp = _rng(s, _T_POS, blk, step)
        for b in range(s.B):
            if active is None:
                pos = np.sort(gp.choice(s.Nb, size=M, replace=False))
            else:
                pos = np.sort(gp.choice(active[b].numpy(), size=M, replace=False))
            idx = torch.from_numpy(pos)
            for t, code, H in ((q, _T_NQ, s.Hq), (kin, _T_NK, s.Hkv), (vin, _T_NV, s.Hkv)):
                noise = _rng(s, code, blk, step, b).standard_normal(
                    (H, M, s.D), dtype=np.float32) * np.float32(s.pert_std)
                cur = t[b][:, idx].float().numpy()
                t[b][:, idx] = _cast(cur + noise, s)
        return M, q, kin, vin

    # -- sparse selection -----------------------------------------------------
    def selection(self, blk: int, prefix_len: int) -> torch.Tensor:
        """Top-``sel_k`` prefix keys per (b, query head) by a seeded fp32 score.

        Score_j ~ Uniform(0, 1) in fp32; ties go to the lower index; the list is
        returned ascending, int32 [B, Hq, k].  This stands in for a sparse
        attention method's key choice, which the FlashBlock step takes as input.
        """
        s = self.spec
        k = min(s.sel_k, prefix_len)
        out = np.empty((s.B, s.Hq, k), dtype=np.int32)
        g = _rng(s, _T_SCORE, blk)
        for b in range(s.B):
            score = g.random((s.Hq, prefix_len), dtype=np.float32)
            for h in range(s.Hq):
                order = np.argsort(-score[h], kind="stable")[:k]
                out[b, h] = np.sort(order)
        return torch.from_numpy(out)

    # -- active-query subsets -----------------------------------------------
    def n_active(self, step: int) -> int:
        """Positions still active at a block's step: all Nb at step 0, then a
        share lock_rate of them locks at every step (at least one stays)."""
        s = self.spec
        return max(1, int(round(s.Nb * (1.0 - s.lock_rate) ** step)))

    def lock_step(self, blk: int, step: int, active: Optional[torch.Tensor]) -> torch.Tensor:
        """Active positions at ``step``: a seeded random subset of the previous
        step's active positions (locking is monotone), int32 [B, n] ascending."""
        s = self.spec
        n = self.n_active(step)
        if active is None:
            return torch.arange(s.Nb, dtype=torch.int32).repeat(s.B, 1)
        g = _rng(s, _T_LOCK, blk, step)
        out = np.stack([np.sort(g.choice(active[b].numpy(), size=n, replace=False)) for b in range(s.B)])
        return torch.from_numpy(out.astype(np.int32))

    # -- the whole schedule -------------------------------------------------
    def schedule(self) -> Iterator[Step]:
        s = self.spec
        for blk in range(s.blocks):
            plen = s.prefix0 + blk * s.Nb
            sel = self.selection(blk, plen) if s.sel_k and s.select == "score" else None
            q, kin, vin = self.block_start(blk)
            active = None
            for st in range(s.steps):
                if s.lock_rate is not None:
                    active = self.lock_step(blk, st, active)
                M = 0
                if st > 0:
                    M, q, kin, vin = self.step_update(blk, st, q, kin, vin, active)
                yield Step(blk, st, plen, M, q, kin, vin, sel, st == s.steps - 1, active)


def get_spec(name: str, **overrides) -> WorkloadSpec:
    spec = SPECS[name]
    return spec.scaled(**overrides) if overrides else spec


def tensor(shape, seed: int, std: float = 1.0, dtype: str = "bf16") -> torch.Tensor:
    """A seeded N(0, std^2) tensor (fp32 draw, bf16 by round-to-nearest-even)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    x = g.standard_normal(size=tuple(shape), dtype=np.float32) * np.float32(std)
    t = torch.from_numpy(x)
    return t if dtype == "f32" else t.to(torch.bfloat16)


def uniform(shape, seed: int, lo: float, hi: float) -> torch.Tensor:
    """A seeded Uniform(lo, hi) fp32 tensor."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    return torch.from_numpy(g.uniform(lo, hi, size=tuple(shape)).astype(np.float32))


def random_selection(B: int, Hq: int, prefix_len: int, k: int, seed: int) -> torch.Tensor:
    """k distinct ascending prefix positions per (b, h), int32 [B, Hq, k]."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    out = np.stack([np.stack([np.sort(g.choice(prefix_len, size=k, replace=False)) for _ in range(Hq)])
                    for _ in range(B)]).astype(np.int32)
    return torch.from_numpy(out.reshape(B, Hq, k))
