"""GPU-vs-oracle parity through the C-ABI (needs a B200).

Each test feeds the same seeded inputs to libfb (through its ctypes binding)
and to the fp64 oracle, then compares element by element under the tolerances
of tests/_gpu_common.py; reuse decisions and masks must agree bit for bit.
"""
import numpy as np
import pytest
import torch

from block_diffusion_attention_flashblock_b200 import fb
from block_diffusion_attention_flashblock_b200 import workloads as wl
from oracle import flashblock_oracle as orc

from _gpu_common import TOL, assert_lse_close, assert_o_close, compare_schedule

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fb.lib()


def _mk(B, Hq, Hkv, D, Nb, Lp, dtype, seed, cap_extra=64, std=1.0):
    q = wl.tensor((B, Hq, Nb, D), seed, std, dtype)
    kin = wl.tensor((B, Hkv, Nb, D), seed + 1, std, dtype)
    vin = wl.tensor((B, Hkv, Nb, D), seed + 2, std, dtype)
    kp = wl.tensor((B, Hkv, Lp + cap_extra, D), seed + 3, std, dtype)
    vp = wl.tensor((B, Hkv, Lp + cap_extra, D), seed + 4, std, dtype)
    return q, kin, vin, kp, vp


SHAPES = [
    # (B, Hq, Hkv, D, Nb, Lp, dtype)
    (1, 4, 4, 64, 32, 256, "f32"),        # the tiny fp32 workload
    (2, 4, 2, 128, 7, 300, "f32"),        # fp32, GQA, ragged
    (1, 32, 8, 128, 32, 1000, "bf16"),    # dLLM shape, ragged prefix tail (1000 = 15*64 + 40)
    (2, 8, 2, 64, 24, 700, "bf16"),       # D=64, G*Nb = 96 rows -> two row tiles
    (1, 2, 2, 128, 200, 333, "bf16"),     # long block: several row tiles per head
    (1, 32, 8, 128, 32, 8192, "bf16"),    # dLLM prefix at full size
    (1, 8, 8, 128, 1, 129, "bf16"),       # one query, one key past a tile
]


@pytest.fixture
def prefix_kernel():
    """Force one block-external kernel for a test, restore automatic choice after."""
    def use(which):
        fb.fb_debug_set_prefix_kernel(which)
    yield use
    fb.fb_debug_set_prefix_kernel(fb.PREFIX_AUTO)


def _outblock_check(shape, seed=11):
    B, Hq, Hkv, D, Nb, Lp, dt = shape
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, Lp, dt, seed=seed)
    qd, kpd, vpd = q.cuda(), kp.cuda(), vp.cuda()
    a = torch.full((B, Hq, Nb, D), float("nan"), device="cuda")
    l = torch.full((B, Hq, Nb), float("nan"), device="cuda")
    desc = fb.make_desc(qd, kin.cuda(), kpd, a)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
    fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, a, l, ws)
    assert fb.fb_get_device_status() == fb.FB_OK
    A, L = orc.outblock(orc.to64(q), orc.to64(kp), orc.to64(vp), Lp, 1 / np.sqrt(D))
    assert_o_close(a, A, TOL[dt], "A_out")
    assert_lse_close(l, L, TOL[dt], "L_out")


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_outblock_dense(shape, prefix_kernel):
    prefix_kernel(fb.PREFIX_GENERIC)
    _outblock_check(shape)


TC_SHAPES = [
    # (B, Hq, Hkv, D, Nb, Lp, dtype): tcgen05 tilings
    (1, 32, 8, 128, 32, 1000, "bf16"),    # 4 heads x 32 queries per tile, ragged last key tile (104 keys)
    (1, 32, 8, 128, 32, 8192, "bf16"),    # dLLM prefix at full size
    (2, 32, 8, 128, 64, 3000, "bf16"),    # 2 heads x 64 queries per tile, two tiles per KV head
    (1, 8, 4, 128, 32, 500, "bf16"),      # G*Nb = 64: half-filled tiles
    (1, 4, 4, 128, 200, 2000, "bf16"),    # one head per tile, 128 queries, ragged query tail
    (1, 8, 2, 128, 1560, 1700, "bf16"),   # video-like block with GQA, 13 query tiles per head
    (1, 2, 2, 128, 64, 129, "bf16"),      # second key tile holds one key
    (1, 2, 1, 128, 64, 1, "bf16"),        # a single prefix key
]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("mode", ["cluster", "merge"])
def test_outblock_dense_tcgen05(shape, mode, prefix_kernel):
    """tcgen05 prefix pass; key splits reduced in-kernel across a cluster, or by the merge pass."""
    prefix_kernel(fb.PREFIX_TC_CLUSTER if mode == "cluster" else fb.PREFIX_TC_NO_CLUSTER)
    _outblock_check(shape, seed=13)


PAIR_SHAPES = [
    # (B, Hq, Hkv, D, Nb, Lp, dtype): two or more 128-row query tiles per KV head
    (2, 32, 8, 128, 64, 3000, "bf16"),     # 2 heads x 64 queries per tile, one pair per KV head
    (4, 32, 8, 128, 64, 4100, "bf16"),     # the long-context shape, small: CTAs span several pairs
    (1, 16, 4, 128, 64, 777, "bf16"),      # ragged last key tile (777 = 6 * 128 + 9)
    (1, 4, 4, 128, 200, 2000, "bf16"),     # one head per tile, ragged query tail (200 = 128 + 72)
    (1, 6, 6, 128, 300, 1000, "bf16"),     # three tiles per head: one pair and one lone tile
    (1, 8, 2, 128, 1560, 1700, "bf16"),    # video-like block with GQA, 52 tiles per KV head
    (1, 2, 2, 128, 1560, 31200, "bf16"),   # a video frame block over the full 20-frame prefix
]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_outblock_dense_paired(shape, prefix_kernel):
    """The paired stream-K tcgen05 prefix pass (two query tiles per CTA, one
    thread per row) and the merge of its slots."""
    prefix_kernel(fb.PREFIX_TC)
    _outblock_check(shape, seed=17)


@pytest.mark.parametrize("v_scale", [2.0 ** 17, 2.0 ** -10, 2.0 ** 12, 2.0 ** -3, "mixed"],
                         ids=["huge", "tiny", "fp16-top", "fp16-bottom", "mixed"])
def test_outblock_paired_v_ranges(v_scale, prefix_kernel):
    """The paired kernel runs P V in fp16 on V tiles whose largest |v| has a
    binary exponent in [-4, 15] and in bf16 hi/lo on any other tile; values
    scaled out of that window (huge, tiny) take the bf16 path, values at its
    edges the fp16 one, and a prefix whose first tiles are huge mixes both
    within one accumulation."""
    prefix_kernel(fb.PREFIX_TC)
    B, Hq, Hkv, D, Nb, Lp = 1, 8, 2, 128, 64, 2000
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, Lp, "bf16", seed=19)
    vf = vp.float()
    if v_scale == "mixed":
        vf[:, :, :512] *= 2.0 ** 17
    else:
        vf *= v_scale
    vp = vf.to(torch.bfloat16)
    qd, kpd, vpd = q.cuda(), kp.cuda(), vp.cuda()
    a = torch.full((B, Hq, Nb, D), float("nan"), device="cuda")
    l = torch.full((B, Hq, Nb), float("nan"), device="cuda")
    desc = fb.make_desc(qd, kin.cuda(), kpd, a)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
    fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, a, l, ws)
    assert fb.fb_get_device_status() == fb.FB_OK
    A, L = orc.outblock(orc.to64(q), orc.to64(kp), orc.to64(vp), Lp, 1 / np.sqrt(D))
    assert_o_close(a, A, TOL["bf16"], "A_out")
    assert_lse_close(l, L, TOL["bf16"], "L_out")


@pytest.mark.parametrize("which", ["generic", "tcgen05", "tcgen05-cluster", "paired"])
def test_outblock_rising_and_falling_scores(which, prefix_kernel):
    """Scores that grow along the prefix (KV head 0) force the running max to
    move on every key tile, so O is rescaled in place many times; scores that
    fall (KV head 1) never move it after the first tile."""
    prefix_kernel({"generic": fb.PREFIX_GENERIC, "tcgen05": fb.PREFIX_TC_NO_CLUSTER,
                   "tcgen05-cluster": fb.PREFIX_TC_CLUSTER, "paired": fb.PREFIX_TC}[which])
    # 8 row tiles x 64 key tiles (ragged last): several key tiles per CTA;
    # blocks of 64 for the paired kernel (two row tiles per KV head)
    B, Hq, Hkv, D, Lp = 1, 32, 8, 128, 8100
    Nb = 64 if which == "paired" else 32
    q = wl.tensor((B, Hq, Nb, D), 61, 0.5, "f32").abs().to(torch.bfloat16)
    ramp = torch.arange(Lp + 64, dtype=torch.float32) * 0.02
    sign = torch.tensor([1.0, -1.0] * (Hkv // 2)).view(1, Hkv, 1, 1)
    kp = (wl.tensor((B, Hkv, Lp + 64, D), 62, 0.5, "f32") + sign * ramp.view(1, 1, -1, 1)).to(torch.bfloat16)
    vp = wl.tensor((B, Hkv, Lp + 64, D), 63, 1.0, "bf16")
    kin = wl.tensor((B, Hkv, Nb, D), 64, 1.0, "bf16")
    qd, kpd, vpd = q.cuda(), kp.cuda(), vp.cuda()
    a = torch.full((B, Hq, Nb, D), float("nan"), device="cuda")
    l = torch.full((B, Hq, Nb), float("nan"), device="cuda")
    desc = fb.make_desc(qd, kin.cuda(), kpd, a)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
    fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, a, l, ws)
    assert fb.fb_get_device_status() == fb.FB_OK
    A, L = orc.outblock(orc.to64(q), orc.to64(kp), orc.to64(vp), Lp, 1 / np.sqrt(D))
    for h0 in range(0, Hq, Hq // Hkv):   # the heads of each KV head separately (their scales differ)
        h1 = h0 + Hq // Hkv
        assert_o_close(a[:, h0:h1], A[:, h0:h1], TOL["bf16"], f"A_out heads {h0}..{h1 - 1}")
        assert_lse_close(l[:, h0:h1], L[:, h0:h1], TOL["bf16"], f"L_out heads {h0}..{h1 - 1}")


@pytest.mark.parametrize("name", ["dllm_8k_small", "dllm_64k_small", "video_small_mixed"])
def test_step_schedule_tcgen05_no_cluster(name, prefix_kernel):
    prefix_kernel(fb.PREFIX_TC_NO_CLUSTER)
    compare_schedule(_spec(name))


@pytest.mark.parametrize("name", ["dllm_8k_small", "dllm_64k_small", "sparse_small"])
def test_step_schedule_tcgen05_cluster(name, prefix_kernel):
    """The split planner takes the in-kernel cluster reduction wherever it saves waves or parts."""
    prefix_kernel(fb.PREFIX_TC_CLUSTER)
    compare_schedule(_spec(name))


def test_outblock_empty_prefix():
    q, kin, vin, kp, vp = _mk(1, 4, 2, 128, 16, 0, "bf16", seed=5)
    qd, kpd = q.cuda(), kp.cuda()
    a = torch.full((1, 4, 16, 128), 7.0, device="cuda")
    l = torch.zeros(1, 4, 16, device="cuda")
    desc = fb.make_desc(qd, kin.cuda(), kpd, a)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, 0), dtype=torch.uint8, device="cuda")
    fb.fb_attn_outblock(desc, qd, kpd, vp.cuda(), 0, a, l, ws)
    assert torch.all(a == 0) and torch.all(torch.isneginf(l))


@pytest.mark.parametrize("shape", [(1, 8, 2, 128, 32, 1500, 100, "bf16"), (1, 4, 4, 64, 32, 256, 40, "f32"),
                                   (1, 32, 8, 128, 32, 32768, 2048, "bf16"), (2, 8, 4, 128, 64, 5000, 300, "bf16"),
                                   (2, 8, 2, 128, 16, 3000, 0, "bf16"), (1, 4, 1, 128, 8, 200, 200, "bf16"),
                                   (1, 8, 2, 128, 32, 300, 300, "bf16"), (1, 4, 4, 128, 200, 2000, 700, "bf16")],
                         ids=lambda s: "x".join(map(str, s)))
def test_outblock_sparse_and_residual(shape):
    B, Hq, Hkv, D, Nb, Lp, k, dt = shape
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, Lp, dt, seed=21)
    sel = wl.random_selection(B, Hq, Lp, k, seed=99)
    qd, kpd, vpd = q.cuda(), kp.cuda(), vp.cuda()
    aS = torch.empty(B, Hq, Nb, D, device="cuda"); lS = torch.empty(B, Hq, Nb, device="cuda")
    aU = torch.empty_like(aS); lU = torch.empty_like(lS)
    desc = fb.make_desc(qd, kin.cuda(), kpd, aS)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp, k), dtype=torch.uint8, device="cuda")
    fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, aS, lS, ws, sel=sel.cuda(), sel_k=k, a_res=aU, l_res=lU)
    sc = 1 / np.sqrt(D)
    AS, LS = orc.outblock_selected(orc.to64(q), orc.to64(kp), orc.to64(vp), Lp, sc, sel.numpy(), residual=False)
    AU, LU = orc.outblock_selected(orc.to64(q), orc.to64(kp), orc.to64(vp), Lp, sc, sel.numpy(), residual=True)
    assert_o_close(aS, AS, TOL[dt], "A_S"); assert_lse_close(lS, LS, TOL[dt], "L_S")
    assert_o_close(aU, AU, TOL[dt], "A_U"); assert_lse_close(lU, LU, TOL[dt], "L_U")


def _random_parts(B, Hq, Nb, D, n, seed, empty_rows=True):
    parts = []
    for p in range(n):
        A = wl.tensor((B, Hq, Nb, D), seed + 10 * p, 1.0, "f32")
        L = wl.tensor((B, Hq, Nb), seed + 10 * p + 1, 3.0, "f32")
        if empty_rows and p == 0:
            L[..., ::5] = -float("inf")
            A[..., ::5, :] = 0.0
        parts.append((A, L))
    return parts


@pytest.mark.parametrize("nparts", [0, 1, 2, 4, 7])
@pytest.mark.parametrize("shape", [(1, 32, 8, 128, 32, "bf16"), (1, 4, 4, 64, 32, "f32"),
                                   (1, 3, 3, 128, 150, "bf16"), (2, 8, 4, 64, 5, "bf16"),
                                   (2, 8, 2, 128, 5, "bf16"), (1, 8, 2, 128, 64, "bf16"),
                                   (3, 4, 4, 128, 16, "bf16"), (1, 2, 1, 128, 1, "bf16"),
                                   (1, 4, 2, 128, 1560, "bf16"), (1, 3, 3, 128, 1000, "bf16")],
                         ids=lambda s: "x".join(map(str, s)))
def test_inblock_merge(shape, nparts):
    B, Hq, Hkv, D, Nb, dt = shape
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, 8, dt, seed=31)
    parts = _random_parts(B, Hq, Nb, D, nparts, seed=300)
    o = torch.empty(B, Hq, Nb, D, device="cuda")
    lse = torch.empty(B, Hq, Nb, device="cuda")
    desc = fb.make_desc(q.cuda(), kin.cuda(), kp.cuda(), o)
    fb.fb_attn_inblock(desc, q.cuda(), kin.cuda(), vin.cuda(), o, lse,
                       [a.cuda() for a, _ in parts], [l.cuda() for _, l in parts])
    Ai, Li = orc.inblock(orc.to64(q), orc.to64(kin), orc.to64(vin), 1 / np.sqrt(D))
    A, L = orc.merge([(orc.to64(a), orc.to64(l)) for a, l in parts] + [(Ai, Li)])
    assert_o_close(o, A, TOL[dt], "O"); assert_lse_close(lse, L, TOL[dt], "LSE")


@pytest.mark.parametrize("rows", [1, 16, 32, 64])
@pytest.mark.parametrize("nparts", [0, 1, 4])
@pytest.mark.parametrize("shape", [(1, 32, 8, 128, 32, "bf16"), (2, 8, 2, 128, 5, "bf16"),
                                   (1, 8, 2, 128, 64, "bf16"), (3, 4, 4, 128, 16, "bf16"),
                                   (1, 2, 1, 128, 1, "bf16"), (2, 12, 4, 128, 50, "bf16")],
                         ids=lambda s: "x".join(map(str, s)))
def test_inblock_small_variants(shape, nparts, rows):
    # both small-block kernels (split-warp CTAs of 16 rows, and one warp per
    # 16 rows with CTAs of 16, 32 or 64 rows), bf16 output
    B, Hq, Hkv, D, Nb, dt = shape
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, 8, dt, seed=37)
    parts = _random_parts(B, Hq, Nb, D, nparts, seed=310)
    o = torch.empty(B, Hq, Nb, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Nb, device="cuda")
    desc = fb.make_desc(q.cuda(), kin.cuda(), kp.cuda(), o)
    try:
        fb.fb_debug_set_inblock_rows(rows)
        fb.fb_attn_inblock(desc, q.cuda(), kin.cuda(), vin.cuda(), o, lse,
                           [a.cuda() for a, _ in parts], [l.cuda() for _, l in parts])
    finally:
        fb.fb_debug_set_inblock_rows(0)
    Ai, Li = orc.inblock(orc.to64(q), orc.to64(kin), orc.to64(vin), 1 / np.sqrt(D))
    A, L = orc.merge([(orc.to64(a), orc.to64(l)) for a, l in parts] + [(Ai, Li)])
    assert_o_close(o, A, TOL[dt], "O"); assert_lse_close(lse, L, TOL[dt], "LSE")


@pytest.mark.parametrize("nparts", [1, 2, 5, 8])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_merge_nway(nparts, out):
    B, Hq, Nb, D = 2, 6, 37, 128
    parts = _random_parts(B, Hq, Nb, D, nparts, seed=500)
    if nparts >= 2:   # rows where every part is empty
        for a, l in parts:
            l[0, 0, 3] = -float("inf"); a[0, 0, 3] = 0.0
    dt = torch.float32 if out == "f32" else torch.bfloat16
    o = torch.empty(B, Hq, Nb, D, dtype=dt, device="cuda")
    lse = torch.empty(B, Hq, Nb, device="cuda")
    q = torch.empty(B, Hq, Nb, D, dtype=torch.bfloat16, device="cuda")
    desc = fb.make_desc(q, q, q, o)
    fb.fb_merge(desc, [a.cuda() for a, _ in parts], [l.cuda() for _, l in parts], o, lse)
    A, L = orc.merge([(orc.to64(a), orc.to64(l)) for a, l in parts])
    assert_o_close(o, A, 1e-6, "merge O")
    assert_lse_close(lse, L, 1e-6, "merge LSE")


def test_kv_append_bit_exact():
    B, Hkv, Nb, D, cap = 2, 3, 40, 128, 300
    kp = wl.tensor((B, Hkv, cap, D), 1); vp = wl.tensor((B, Hkv, cap, D), 2)
    kin = wl.tensor((B, Hkv, Nb, D), 3); vin = wl.tensor((B, Hkv, Nb, D), 4)
    kpd, vpd = kp.cuda(), vp.cuda()
    q = torch.empty(B, Hkv, Nb, D, dtype=torch.bfloat16, device="cuda")
    desc = fb.make_desc(q, kin.cuda(), kpd, q)
    fb.fb_kv_append(desc, kpd, vpd, 100, kin.cuda(), vin.cuda())
    K, V, n = orc.kv_append(kp.float().numpy(), vp.float().numpy(), 100, kin.float().numpy(), vin.float().numpy())
    assert n == 140
    assert np.array_equal(kpd.float().cpu().numpy(), K) and np.array_equal(vpd.float().cpu().numpy(), V)
    with pytest.raises(fb.FbError):
        fb.fb_kv_append(desc, kpd, vpd, 270, kin.cuda(), vin.cuda())


# ------------------------------------------------------------ schedules ---
SCHEDULES = {
    "tiny_f32": dict(),
    # the fp32 path through fb_step with reuse: tau off reuses steps 1..3; tau 8
    # reuses every step (M = 4, 7, 5); tau 6 alternates (reuse, recompute, reuse)
    "tiny_f32_tau_off": dict(base="tiny_f32", tau=None),
    "tiny_f32_tau8": dict(base="tiny_f32", tau=8),
    "tiny_f32_tau6": dict(base="tiny_f32", tau=6),
    "dllm_8k_small": dict(base="dllm_8k", prefix0=1000, blocks=2, steps=8),
    "dllm_64k_small": dict(base="dllm_64k_b4", B=2, prefix0=2000, steps=16),
    "video_small_mixed": dict(base="video_1560", Hq=6, Hkv=6, prefix0=3120, steps=5, sigma_range=(0.01, 1.0)),
    "video_small": dict(base="video_1560", Hq=4, Hkv=4, prefix0=3120, steps=4),
    # more query-tile pairs (76 heads x 2) than SMs with a partial last round:
    # the in-block pass splits the remainder's key tiles and merges their
    # slots with the cached part in the merge kernel
    "video_wide_split": dict(base="video_1560", Hq=76, Hkv=76, Nb=512, prefix0=1024, steps=3),
    "sparse_small": dict(base="sparse_32k_k2048", prefix0=4000, sel_k=256, Hq=8, Hkv=2),
    "tau_zero": dict(base="dllm_8k", prefix0=500, blocks=1, steps=4, tau=0),
    "tau_off": dict(base="dllm_8k", prefix0=500, blocks=1, steps=4, tau=None),
    "nb1_gqa": dict(base="dllm_8k", Nb=1, prefix0=300, steps=3, m_model=("uniform", 0, 1), tau=1),
    "nb4_small": dict(base="dllm_8k_nb4", prefix0=1000, blocks=2),
    "sparse_d40_small": dict(base="sparse_32k_d40", prefix0=3000, sel_k=1200, Hq=8, Hkv=2),
    # gamma gates that always reuse (every similarity exceeds -1) and never
    # reuse: from step 2 on every head is masked, or none is
    "video_gamma_always": dict(base="video_1560", Hq=4, Hkv=4, prefix0=3120, steps=4, gamma=-1.0),
    "video_gamma_never": dict(base="video_1560", Hq=4, Hkv=4, prefix0=3120, steps=4, gamma=1.5),
    # the first block of a sequence: no prefix at all
    "empty_prefix": dict(base="dllm_8k", prefix0=0, blocks=2, steps=3),
    "empty_prefix_nb64": dict(base="dllm_64k_b4", B=1, prefix0=0, blocks=2, steps=3),
    # the sparse keys chosen by attention mass at each block's start
    "mass_small": dict(base="sparse_32k_mass", prefix0=4000, sel_k=256, Hq=8, Hkv=2, blocks=2),
    "mass_nb16_b2": dict(base="sparse_32k_mass", B=2, Nb=16, prefix0=2500, sel_k=700, Hq=16, Hkv=2, steps=5,
                         m_model=("binomial", 16, 0.15), tau=4),
    # active-query subsets: a quarter of the active positions lock per step
    "lock_small": dict(base="dllm_8k_lock", prefix0=1000, blocks=2),
    "lock_b2_nb64": dict(base="dllm_8k_lock", B=2, Nb=64, prefix0=700, blocks=1, steps=6, lock_rate=0.3,
                         m_model=("binomial", 64, 0.1), tau=6),
    "lock_tau_zero": dict(base="dllm_8k_lock", prefix0=1500, blocks=1, steps=6, tau=0),
}


def _spec(name):
    kw = dict(SCHEDULES[name])
    base = kw.pop("base", name)
    return wl.get_spec(base, **kw)


@pytest.mark.parametrize("rows", [1, 16, 64])
@pytest.mark.parametrize("name", ["dllm_64k_small", "lock_b2_nb64", "nb4_small", "sparse_small"])
def test_step_schedule_inblock_variants(name, rows):
    # the full and reuse steps (cache rows written on full steps, active-query
    # subsets) through each small-block in-block kernel
    try:
        fb.fb_debug_set_inblock_rows(rows)
        compare_schedule(_spec(name))
    finally:
        fb.fb_debug_set_inblock_rows(0)


@pytest.mark.parametrize("name", list(SCHEDULES))
def test_step_schedule(name):
    spec = _spec(name)
    st = compare_schedule(spec)
    if name == "tau_zero":
        assert all(st["recomputed"])
    if name in ("tau_off", "tiny_f32_tau_off", "tiny_f32_tau8"):
        assert st["recomputed"] == [True, False, False, False]
    if name == "tiny_f32_tau6":
        assert st["recomputed"] == [True, False, True, False]
    if name == "video_small_mixed":
        r = np.array(st["reuse"])
        assert 0 < r[2:].mean() < 1, "the mixed video case should both reuse and recompute"
    if name == "video_gamma_always":
        assert np.array(st["reuse"])[2:].min() == 1.0
    if name == "video_gamma_never":
        assert np.array(st["reuse"]).max() == 0.0


def test_step_bf16_output():
    spec = wl.get_spec("dllm_8k", prefix0=700, blocks=1, steps=4)
    compare_schedule(spec, out_dtype=torch.bfloat16)


# ------------------------------------------------ full-size workloads ---
def test_full_dllm_8k_all_heads():
    """The benchmarked workload at its full size: 4 blocks x 8 steps, every head."""
    compare_schedule(wl.get_spec("dllm_8k"), check_every=1)


@pytest.mark.parametrize("name, groups", [
    ("dllm_64k_b4", [(0, 0), (3, 7)]),
    ("dllm_ctx_200k", [(0, 0), (0, 7)]),
    ("dllm_ctx_800k", [(0, 3)]),
    ("dllm_8k_nb4", [(0, 0), (0, 5)]),
    ("sparse_32k_d40", [(0, 0), (0, 6)]),
    ("video_1560", [(0, 0), (0, 13), (0, 23)]),
    ("sparse_32k_k2048", [(0, 0), (0, 5)]),
    ("dllm_8k_lock", [(0, 0), (0, 3)]),
    ("sparse_32k_mass", [(0, 0), (0, 6)]),
])
def test_full_size_sampled_heads(name, groups):
    """Full-size workloads; the oracle recomputes only the sampled (b, kv-head) groups."""
    spec = wl.get_spec(name)
    compare_schedule(spec, groups=groups, check_every=1)


@pytest.mark.parametrize("sparse", [False, True])
def test_step_changed_prefix_recomputes(sparse):
    """fb_step on a longer prefix without a new block (tau off, so the stale
    cache would otherwise be reused): the step recomputes, as the oracle's, and
    both outputs agree; then a step on the same prefix reuses again."""
    B, Hq, Hkv, D, Nb, Lp = 1, 8, 2, 128, 32, 1200
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, Lp, "bf16", seed=71)
    sel = wl.random_selection(B, Hq, Lp - 200, 64, seed=72) if sparse else None
    qd, kind, vind, kpd, vpd = q.cuda(), kin.cuda(), vin.cuda(), kp.cuda(), vp.cuda()
    o = torch.empty(B, Hq, Nb, D, device="cuda")
    lse = torch.empty(B, Hq, Nb, device="cuda")
    layer = fb.FlashBlockLayer(qd, kind, kpd, o, max_prefix=Lp, sparse=sparse, max_sel_k=64)
    ref = orc.FlashBlockOracle(B, Hq, Hkv, D, Nb)
    q64, k64, v64, kp64, vp64 = (orc.to64(t) for t in (q, kin, vin, kp, vp))
    seld = None if sel is None else sel.cuda()
    seln = None if sel is None else sel.numpy()
    layer.begin_block()
    for plen, expect in ((Lp - 200, True), (Lp - 200, False), (Lp, True), (Lp, False)):
        layer.step(qd, kind, vind, kpd, vpd, plen, 0, fb.FB_TAU_OFF, o, lse, sel=seld)
        r = ref.step(q64, k64, v64, kp64, vp64, plen, 0, None, seln)
        assert layer.last_recomputed() == r.recompute == expect
        assert_o_close(o, r.o, TOL["bf16"], f"prefix {plen}")
        assert_lse_close(lse, r.lse, TOL["bf16"], f"prefix {plen}")
    layer.close()
    assert fb.fb_get_device_status() == fb.FB_OK


@pytest.mark.parametrize("k", [0, 1, 50, 640])
def test_select_mass_all_tied_takes_the_first_keys(k):
    """Zero queries give every key the same mass bit for bit (each query's
    probabilities are all 2^-log2(n)), so the top k are the first k keys."""
    B, Hq, Hkv, D, Nb, Lp = 1, 8, 2, 128, 32, 640
    q = torch.zeros(B, Hq, Nb, D, dtype=torch.bfloat16, device="cuda")
    kp = wl.tensor((B, Hkv, Lp, D), 81, 1.0, "bf16").cuda()
    vp = wl.tensor((B, Hkv, Lp, D), 82, 1.0, "bf16").cuda()
    o = torch.empty(B, Hq, Nb, D, device="cuda")
    desc = fb.make_desc(q, kp[:, :, :Nb], kp, o)
    sel = torch.full((B, Hq, k), -1, dtype=torch.int32, device="cuda")
    mass = torch.empty(B, Hq, Lp, device="cuda")
    ws = torch.empty(fb.fb_select_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
    fb.fb_select_mass(desc, q, kp, vp, Lp, k, sel, ws, mass_out=mass)
    assert fb.fb_get_device_status() == fb.FB_OK
    assert torch.all(mass == mass[0, 0, 0])
    assert abs(float(mass[0, 0, 0]) - Nb / Lp) < 1e-6 * Nb / Lp * 10
    assert torch.equal(sel.cpu(), torch.arange(k, dtype=torch.int32).expand(B, Hq, k))


@pytest.mark.parametrize("shape", [(1, 8, 2, 128, 32, 3000, 300), (2, 32, 8, 128, 16, 4100, 4100),
                                   (1, 4, 4, 128, 32, 129, 7)], ids=lambda s: "x".join(map(str, s)))
def test_select_mass_against_the_oracle(shape):
    """fb_select_mass: masses within 2e-5 of the fp64 oracle's, and the top-k
    equal to the oracle's outside the near-tie band at the k-th mass."""
    from _gpu_common import MASS_TOL
    B, Hq, Hkv, D, Nb, Lp, k = shape
    q, kin, vin, kp, vp = _mk(B, Hq, Hkv, D, Nb, Lp, "bf16", seed=91, std=0.5)
    qd, kpd, vpd = q.cuda(), kp.cuda(), vp.cuda()
    o = torch.empty(B, Hq, Nb, D, device="cuda")
    desc = fb.make_desc(qd, kin.cuda(), kpd, o)
    sel = torch.empty(B, Hq, k, dtype=torch.int32, device="cuda")
    mass = torch.empty(B, Hq, Lp, device="cuda")
    ws = torch.empty(fb.fb_select_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
    fb.fb_select_mass(desc, qd, kpd, vpd, Lp, k, sel, ws, mass_out=mass)
    assert fb.fb_get_device_status() == fb.FB_OK
    M = orc.attention_mass(orc.to64(q), orc.to64(kp), Lp, 1 / np.sqrt(D))
    gm = mass.double().cpu().numpy()
    assert np.max(np.abs(gm - M) / M.max(axis=2, keepdims=True)) <= MASS_TOL
    g_sel = sel.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            m = M[b, h]
            kth = np.sort(m)[::-1][k - 1]
            band = MASS_TOL * m.max()
            assert np.all(np.diff(g_sel[b, h]) > 0)
            assert np.isin(np.flatnonzero(m > kth + band), g_sel[b, h]).all()
            assert not np.isin(np.flatnonzero(m < kth - band), g_sel[b, h]).any()
