"""Plain fp64 CPU oracle of the FlashBlock block-diffusion attention step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product.  It is slow on purpose: every function is the
textbook definition written out in float64 numpy, with matrix products as the
only library primitive, so a reader can check it against the pages by eye.

Source: "FlashBlock: Attention Caching for Efficient Long-Context Block
Diffusion" (gist.science technical summary, section "Mécanisme Central" and
"Stratégies de Réutilisation Adaptatives"; fugumt abstract page, "Abstract").

What the pages define, and how it is written here
-------------------------------------------------
* Attention over a key set J, for one query q (section "Mécanisme Central"):
  s_j = scale * q.k_j, Z = sum_j exp(s_j), A = sum_j exp(s_j) v_j / Z and the
  log-normaliser L = log Z.  ``attention_part``.
* The split into block-internal keys J_in (the current block) and
  block-external keys J_out (everything outside the block: the prefix KV
  cache), giving (A_in, L_in) and (A_out, L_out).  ``inblock``, ``outblock``.
* The log-space merge: m = max(L_out, L_in),
  A = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}).
  The merged normaliser L = m + log(e^{L_out-m} + e^{L_in-m}) follows from
  L = log Z (Z adds over disjoint key sets).  ``merge`` (N-way).
* Reuse of the cached (A_out, L_out) of an earlier diffusion step when the
  updated-token count M < tau (discrete diffusion), and only in heads whose
  similarity exceeds gamma (video) (section "Stratégies de Réutilisation
  Adaptatives").  ``FlashBlockOracle.step``.
* Sparse attention compatibility: the keys a sparse method did not select
  are treated as the block-external set and their residual contribution is
  cached (same section, third bullet).  ``outblock_selected``.
* Selection of the sparse keys by attention mass (same section, sparse bullet,
  and "Résultats Expérimentaux", SparseD bullet; the rule is a reading):
  ``attention_mass``, ``select_top_k``.
* Active-query subsets (SureLock page, "Principes de Fonctionnement", items 2
  and 3): only the M_t still-unlocked positions of the block query, over the
  cached K/V of every token; a locked position keeps its output.  Combined
  here with the FlashBlock cache of A_out.  ``FlashBlockOracle.step(active=)``.

Readings where the pages are silent (each one is listed in the design notes):
scale = 1/sqrt(D); natural log; bidirectional attention inside the block;
query head h uses KV head floor(h / G); M is the per-step count supplied by
the caller, compared strictly (M == tau recomputes); the cached A_out is the
most recently computed one; the similarity is the cosine of the flattened
[Nb, D] block-external output of a head between the fresh and the cached
value, defined from step 1 on, compared strictly, and a head that reuses keeps
its cache and similarity until the block ends; an empty key set gives
(A, L) = (0, -inf).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


def default_scale(D: int) -> float:
    """Softmax scale when the caller gives none: 1/sqrt(D) (pages silent)."""
    return 1.0 / math.sqrt(D)


def attention_part(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Softmax attention of queries q [n, D] over keys k, values v [m, D].

    Returns (A [n, D], L [n]) with L = log sum_j exp(scale q.k_j) (natural log)
    and A = sum_j softmax_j v_j ("Mécanisme Central": A with L = log Z).
    An empty key set (m = 0) gives A = 0 and L = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, D = q.shape
    if k.shape[0] == 0:
        return np.zeros((n, v.shape[1])), np.full(n, NEG_INF)
    s = scale * (q @ k.T)                       # [n, m]
    mx = s.max(axis=1, keepdims=True)           # shift for exp range only
    e = np.exp(s - mx)
    z = e.sum(axis=1, keepdims=True)
    A = (e @ v) / z
    L = (mx + np.log(z))[:, 0]
    return A, L


def merge(parts: Sequence[Tuple[np.ndarray, np.ndarray]]):
    """N-way log-space merge of attention parts over disjoint key sets.

    With m = max_p L_p and w_p = exp(L_p - m):
        A = sum_p w_p A_p / sum_p w_p,   L = m + log sum_p w_p
    which for two parts is the merge formula of "Mécanisme Central".  Rows
    whose parts all have L = -inf give (0, -inf) (no key at all); a part with
    L = -inf has weight exactly 0, so merging with it is the identity.
    """
    As = [np.asarray(a, dtype=np.float64) for a, _ in parts]
    Ls = [np.asarray(l, dtype=np.float64) for _, l in parts]
    Lstack = np.stack(Ls)                                   # [P, ...]
    m = Lstack.max(axis=0)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w = [np.where(np.isneginf(l), 0.0, np.exp(l - m_safe)) for l in Ls]
    wsum = np.sum(w, axis=0)
    num = np.zeros_like(As[0])
    for wp, ap in zip(w, As):
        num = num + wp[..., None] * ap
    den = np.where(empty, 1.0, wsum)
    A = np.where(empty[..., None], 0.0, num / den[..., None])
    L = np.where(empty, NEG_INF, m_safe + np.log(den))
    return A, L


def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """KV head of query head h under grouped-query attention (contiguous groups)."""
    return h // (Hq // Hkv)


def outblock(Q, Kp, Vp, prefix_len: int, scale: float):
    """Block-external attention over the prefix KV cache J_out.

    Q [B, Hq, Nb, D]; Kp, Vp [B, Hkv, >=prefix_len, D].
    Returns A_out [B, Hq, Nb, D], L_out [B, Hq, Nb].
    """
    B, Hq, Nb, D = Q.shape
    Hkv = Kp.shape[1]
    A = np.zeros((B, Hq, Nb, D))
    L = np.zeros((B, Hq, Nb))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            A[b, h], L[b, h] = attention_part(
                Q[b, h], Kp[b, g, :prefix_len], Vp[b, g, :prefix_len], scale)
    return A, L


def inblock(Q, Kin, Vin, scale: float):
    """Block-internal attention over the block's own keys J_in (bidirectional)."""
    B, Hq, Nb, D = Q.shape
    Hkv = Kin.shape[1]
    A = np.zeros((B, Hq, Nb, D))
    L = np.zeros((B, Hq, Nb))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            A[b, h], L[b, h] = attention_part(Q[b, h], Kin[b, g], Vin[b, g], scale)
    return A, L


def outblock_selected(Q, Kp, Vp, prefix_len: int, scale: float, sel, residual: bool):
    """Sparse split of the prefix (section "Stratégies de Réutilisation
    Adaptatives", sparse bullet): each query head h keeps the prefix positions
    sel[b, h] (set S); the rest U = prefix minus S is the block-external set
    whose contribution FlashBlock caches.

    Returns (A_S, L_S) over S, or with ``residual`` (A_U, L_U) over U;
    each [B, Hq, Nb, D] / [B, Hq, Nb].
    """
    B, Hq, Nb, D = Q.shape
    Hkv = Kp.shape[1]
    A = np.zeros((B, Hq, Nb, D)); L = np.zeros((B, Hq, Nb))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            chosen = np.zeros(prefix_len, dtype=bool)
            chosen[np.asarray(sel[b, h], dtype=np.int64)] = True
            keep = ~chosen if residual else chosen
            K = Kp[b, g, :prefix_len]; V = Vp[b, g, :prefix_len]
            A[b, h], L[b, h] = attention_part(Q[b, h], K[keep], V[keep], scale)
    return A, L


def attention_mass(Q, Kp, prefix_len: int, scale: float):
    """Attention mass of each prefix key per (b, query head): the sum over the
    block's queries of the key's softmax probability over the prefix,
        mass[b, h, j] = sum_i exp(s_ij - L_out,i),  s_ij = scale * q_i . k_j,
    with L_out,i = log sum_j exp(s_ij) over the prefix.  Each query's
    probabilities sum to 1, so a head's masses sum to Nb.  This is the score by
    which the sparse selection keeps keys (the pages name a sparse method,
    SparseD, without its rule; the top-k by mass is the reading taken).
    Returns [B, Hq, prefix_len]."""
    B, Hq, Nb, D = Q.shape
    Hkv = Kp.shape[1]
    out = np.zeros((B, Hq, prefix_len))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            s = scale * (np.asarray(Q[b, h], dtype=np.float64) @ np.asarray(Kp[b, g, :prefix_len], dtype=np.float64).T)
            mx = s.max(axis=1, keepdims=True)
            L = mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))
            out[b, h] = np.exp(s - L).sum(axis=0)
    return out


def select_top_k(mass, k: int):
    """Per (b, h): the k keys of largest mass, ties to the lower index, as
    ascending int32 positions [B, Hq, k]."""
    B, Hq, n = mass.shape
    k = min(k, n)
    out = np.empty((B, Hq, k), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            order = sorted(range(n), key=lambda j: (-mass[b, h, j], j))[:k]
            out[b, h] = np.sort(np.asarray(order, dtype=np.int64))
    return out


def full_attention(Q, Kin, Vin, Kp, Vp, prefix_len: int, scale: float):
    """Plain attention of the block's queries over prefix and block keys together."""
    B, Hq, Nb, D = Q.shape
    Hkv = Kp.shape[1]
    A = np.zeros((B, Hq, Nb, D)); L = np.zeros((B, Hq, Nb))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            K = np.concatenate([Kp[b, g, :prefix_len], Kin[b, g]])
            V = np.concatenate([Vp[b, g, :prefix_len], Vin[b, g]])
            A[b, h], L[b, h] = attention_part(Q[b, h], K, V, scale)
    return A, L


def cosine_similarity(a: np.ndarray, c: np.ndarray) -> float:
    """cos(a, c) of two flattened vectors; 0 when either has zero norm."""
    a = np.asarray(a, dtype=np.float64).ravel()
    c = np.asarray(c, dtype=np.float64).ravel()
    na = math.sqrt(float(a @ a)); nc = math.sqrt(float(c @ c))
    if na == 0.0 or nc == 0.0:
        return 0.0
    return float(a @ c) / (na * nc)


def kv_append(Kp, Vp, prefix_len: int, Kin, Vin):
    """Write the finished block's K/V at prefix positions [prefix_len, prefix_len + Nb)."""
    Nb = Kin.shape[2]
    Kp = np.array(Kp, copy=True); Vp = np.array(Vp, copy=True)
    Kp[:, :, prefix_len:prefix_len + Nb] = Kin
    Vp[:, :, prefix_len:prefix_len + Nb] = Vin
    return Kp, Vp, prefix_len + Nb


@dataclass
class StepResult:
    o: np.ndarray             # [B, Hq, Nb, D] merged attention output
    lse: np.ndarray           # [B, Hq, Nb] natural-log normaliser of o
    recompute: bool           # tau decision: False = cached block-external part allowed
    head_reuse: np.ndarray    # bool [B, Hq]: this step used the cached part
    sim: np.ndarray           # [B, Hq] last computed similarity (nan: undefined)


class FlashBlockOracle:
    """The FlashBlock step policy, one attention layer, run step by step.

    State: the cached block-external part (A, L) per (b, h) (the prefix part,
    or for sparse attention the residual over the non-selected keys), its
    validity, and for the gamma gate each head's last similarity.
    """

    def __init__(self, B, Hq, Hkv, D, Nb, scale: Optional[float] = None,
                 gamma: Optional[Sequence[float]] = None):
        self.B, self.Hq, self.Hkv, self.D, self.Nb = B, Hq, Hkv, D, Nb
        self.scale = default_scale(D) if not scale else float(scale)
        self.gamma = None if gamma is None else np.asarray(gamma, dtype=np.float64)
        self.cache_A = np.zeros((B, Hq, Nb, D))
        self.cache_L = np.full((B, Hq, Nb), NEG_INF)
        self.key_set = None
        self.begin_block()

    def begin_block(self):
        """A new block: the cache no longer describes this block's queries."""
        self.valid = False
        self.sim = np.full((self.B, self.Hq), np.nan)
        # outputs of the previous step: the value a locked position keeps
        self.last_o = np.full((self.B, self.Hq, self.Nb, self.D), np.nan)
        self.last_lse = np.full((self.B, self.Hq, self.Nb), np.nan)
        self.last_active = None

    def step(self, q, kin, vin, kp, vp, prefix_len: int, M: int,
             tau: Optional[int], sel=None, active=None) -> StepResult:
        """One diffusion step.  ``active`` ([B, n] block positions, n the
        same for every b), if given, restricts the step to the queries that are
        still unlocked (SureLock page, "Principes de Fonctionnement", items 2
        and 3): only their block-external part is recomputed on a full step,
        only they attend to the block's keys (all Nb of them, locked ones
        included), and a locked position keeps its output of the previous
        step.  Locking is monotone within a block.  Used without sparse
        selection or the gamma gate."""
        if active is not None:
            return self._step_active(q, kin, vin, kp, vp, prefix_len, M, tau, np.asarray(active, dtype=np.int64))
        B, Hq = self.B, self.Hq
        # The cached part is attention over one block-external key set J_out
        # ("Mécanisme Central"): the prefix, or for sparse steps the prefix
        # minus the selection.  A step over another set cannot reuse it and
        # starts over as at a new block.
        key_set = (prefix_len, None if sel is None else np.asarray(sel).tobytes())
        if self.valid and key_set != self.key_set:
            self.begin_block()
        self.key_set = key_set
        tau_reuse = self.valid and (tau is None or M < tau)   # strict "M < tau"
        if self.gamma is None:
            head_reuse = np.full((B, Hq), tau_reuse)
        else:
            sim_ok = ~np.isnan(self.sim) & (self.sim > self.gamma[None, :])
            head_reuse = tau_reuse & sim_ok

        fresh_S = None
        if sel is not None:
            fresh_S = outblock_selected(q, kp, vp, prefix_len, self.scale, sel, residual=False)

        for b in range(B):
            for h in range(Hq):
                if head_reuse[b, h]:
                    continue            # keep the cached part and its similarity
                g = kv_head(h, Hq, self.Hkv)
                K = kp[b, g, :prefix_len]; V = vp[b, g, :prefix_len]
                if sel is not None:     # sparse: block-external set = unselected keys
                    keep = np.ones(prefix_len, dtype=bool)
                    keep[np.asarray(sel[b, h], dtype=np.int64)] = False
                    K, V = K[keep], V[keep]
                a_new, l_new = attention_part(q[b, h], K, V, self.scale)
                if self.gamma is not None and self.valid:
                    self.sim[b, h] = cosine_similarity(a_new, self.cache_A[b, h])
                self.cache_A[b, h] = a_new
                self.cache_L[b, h] = l_new
        self.valid = True

        a_in, l_in = inblock(q, kin, vin, self.scale)
        parts = [(self.cache_A, self.cache_L), (a_in, l_in)]
        if fresh_S is not None:
            parts.insert(0, fresh_S)
        o, lse = merge(parts)
        self.last_o, self.last_lse, self.last_active = o.copy(), lse.copy(), None
        return StepResult(o, lse, not tau_reuse, head_reuse.copy(), self.sim.copy())

    def _step_active(self, q, kin, vin, kp, vp, prefix_len, M, tau, active):
        B, Hq = self.B, self.Hq
        assert self.gamma is None, "active-query subsets are used without the gamma gate"
        assert active.shape[0] == B and 1 <= active.shape[1] <= self.Nb
        if self.last_active is not None:     # monotone locking: no position comes back
            for b in range(B):
                assert set(active[b].tolist()) <= set(self.last_active[b].tolist()), "a locked position came back"
        key_set = (prefix_len, None)
        if self.valid and key_set != self.key_set:
            self.begin_block()
        self.key_set = key_set
        tau_reuse = self.valid and (tau is None or M < tau)
        o = self.last_o.copy()
        lse = self.last_lse.copy()
        for b in range(B):
            rows = active[b]
            for h in range(Hq):
                g = kv_head(h, Hq, self.Hkv)
                qa = q[b, h, rows]
                if not tau_reuse:
                    A, L = attention_part(qa, kp[b, g, :prefix_len], vp[b, g, :prefix_len], self.scale)
                    self.cache_A[b, h, rows] = A
                    self.cache_L[b, h, rows] = L
                a_in, l_in = attention_part(qa, kin[b, g], vin[b, g], self.scale)
                ob, lb = merge([(self.cache_A[b, h, rows], self.cache_L[b, h, rows]), (a_in, l_in)])
                o[b, h, rows] = ob
                lse[b, h, rows] = lb
        self.valid = True
        self.last_o, self.last_lse, self.last_active = o.copy(), lse.copy(), active.copy()
        return StepResult(o, lse, not tau_reuse, np.full((B, Hq), tau_reuse), self.sim.copy())


def to64(t) -> np.ndarray:
    """Exact widening of a torch (bf16/fp32) or numpy tensor to float64."""
    if hasattr(t, "detach"):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)
