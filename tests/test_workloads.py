"""The seeded input generator: determinism, shapes, value model (CPU only)."""
import numpy as np
import torch

from block_diffusion_attention_flashblock_b200 import workloads as wl


def test_deterministic_and_bf16_exact():
    spec = wl.get_spec("dllm_8k", prefix0=300, blocks=2, steps=3)
    a = list(wl.Workload(spec).schedule())
    b = list(wl.Workload(spec).schedule())
    assert len(a) == 6
    for x, y in zip(a, b):
        assert x.M == y.M and torch.equal(x.q, y.q) and torch.equal(x.kin, y.kin)
        assert x.q.dtype == torch.bfloat16 and x.q.shape == (1, 32, 32, 128)
        assert x.kin.shape == (1, 8, 32, 128)
    assert [s.prefix_len for s in a] == [300] * 3 + [332] * 3
    kp, vp = wl.Workload(spec).prefix_kv()
    assert kp.shape == (1, 8, 300 + 64, 128) and torch.all(kp[:, :, 300:] == 0)
    assert abs(kp[:, :, :300].float().std().item() - 0.5) < 0.01


def test_only_M_tokens_change():
    spec = wl.get_spec("dllm_8k", prefix0=64, blocks=1, steps=6)
    prev = None
    for st in wl.Workload(spec).schedule():
        if prev is not None:
            changed = (st.q != prev.q).any(dim=-1).any(dim=1)[0]       # [Nb]
            assert int(changed.sum()) <= st.M
            assert torch.equal((st.kin != prev.kin).any(-1).any(1)[0] & ~changed,
                               torch.zeros_like(changed))
        prev = st


def test_video_every_token_changes_per_head_sigma():
    spec = wl.get_spec("video_1560", prefix0=100, Nb=40, steps=2, Hq=4, Hkv=4)
    w = wl.Workload(spec)
    st = list(w.schedule())
    assert st[1].M == spec.Nb
    sig = w.head_sigmas(0)
    d = (st[1].q.float() - st[0].q.float()).std(dim=(0, 2, 3)).numpy()
    assert np.allclose(d, sig, rtol=0.15)


def test_selection_top_k_ascending_ties_low_index():
    spec = wl.get_spec("sparse_32k_k2048", prefix0=500, sel_k=37, Hq=4, Hkv=1)
    sel = wl.Workload(spec).selection(0, 500).numpy()
    assert sel.shape == (1, 4, 37) and sel.dtype == np.int32
    g = wl._rng(spec, wl._T_SCORE, 0)
    score = g.random((4, 500), dtype=np.float32)
    for h in range(4):
        s = sel[0, h]
        assert np.all(np.diff(s) > 0)
        kth = np.sort(score[h])[::-1][36]
        assert np.all(score[h][s] >= kth)
        assert (score[h] > kth).sum() <= 37


def test_sweep_workloads_restate_their_recipe():
    # context sweep: the long-context layer at B = 1 from 100k to 800k tokens
    for n in (100, 200, 400, 800):
        s = wl.get_spec(f"dllm_ctx_{n}k")
        assert (s.B, s.Hq, s.Hkv, s.D, s.Nb, s.steps, s.tau) == (1, 32, 8, 128, 64, 16, 16)
        assert s.prefix0 == n * 1000 and s.m_model == ("binomial", 64, 0.1)
    # sparse density: the selected fraction of the 32k prefix
    for pct in (20, 30, 40):
        s = wl.get_spec(f"sparse_32k_d{pct}")
        assert s.sel_k == 32768 * pct // 100 and s.prefix0 == 32768 and s.tau == 8
    # small blocks: 4 tokens, at most 4 change per step, tau 2
    s = wl.get_spec("dllm_8k_nb4")
    assert s.Nb == 4 and s.tau == 2 and s.m_model == ("binomial", 4, 0.15)
    w = wl.Workload(wl.get_spec("dllm_8k_nb4", prefix0=64, blocks=2))
    steps = list(w.schedule())
    assert len(steps) == 16 and all(0 <= st.M <= 4 for st in steps)
    assert steps[0].q.shape == (1, 32, 4, 128)


def test_distinct_seeds_per_workload():
    seeds = [s.seed for s in wl.SPECS.values()]
    assert len(seeds) == len(set(seeds))
