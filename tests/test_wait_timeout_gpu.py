"""An expired barrier wait reports FB_ETIMEOUT and leaves the device usable.

Every mbarrier wait in the sm_100a kernels is bounded by a global-timer limit
(fb_debug_set_wait_limit_ns, default two seconds).  Here the limit is set to
one millisecond and the stall hook (fb_debug_set_stall) makes each tcgen05
and small in-block kernel first wait on a barrier that nothing completes, so
that wait runs out: the CTA records FB_ETIMEOUT in the device status word,
the other roles of the CTA see the failure and stop, and every CTA waits
(with its own one-second floor) for the copies and MMAs it started, frees its
tensor memory and returns.  Nothing faults, traps or hangs.  Afterwards the
same calls without the hook must match the oracle, which shows the context is
intact.
"""
import numpy as np
import pytest
import torch

from block_diffusion_attention_flashblock_b200 import fb
from block_diffusion_attention_flashblock_b200 import workloads as wl
from oracle import flashblock_oracle as orc

from _gpu_common import TOL, assert_lse_close, assert_o_close

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.mark.gpu
@pytest.mark.parametrize("rows", [0, 64], ids=["inblock-auto", "inblock-warp-per-rows"])
@pytest.mark.parametrize("Nb", [32, 64], ids=["split-kernel", "paired-kernel"])
def test_expired_wait_reports_timeout_and_the_device_recovers(Nb, rows):
    # dLLM-like shapes: the prefix pass runs on a tcgen05 kernel (TMA + MMA
    # barriers; with blocks of 64 the KV head's 256 query rows make two tiles
    # and the paired stream-K kernel runs) and the in-block merge on the small
    # kernel (bulk-copy barriers)
    B, Hq, Hkv, D, Lp = 1, 8, 2, 128, 2048
    q = wl.tensor((B, Hq, Nb, D), 41, 1.0, "bf16")
    kin = wl.tensor((B, Hkv, Nb, D), 42, 1.0, "bf16")
    vin = wl.tensor((B, Hkv, Nb, D), 43, 1.0, "bf16")
    kp = wl.tensor((B, Hkv, Lp, D), 44, 1.0, "bf16")
    vp = wl.tensor((B, Hkv, Lp, D), 45, 1.0, "bf16")
    qd, kind, vind, kpd, vpd = (t.cuda() for t in (q, kin, vin, kp, vp))
    a = torch.empty(B, Hq, Nb, D, device="cuda")
    l = torch.empty(B, Hq, Nb, device="cuda")
    o = torch.empty(B, Hq, Nb, D, device="cuda")
    lse = torch.empty(B, Hq, Nb, device="cuda")
    desc = fb.make_desc(qd, kind, kpd, o)
    ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")

    assert fb.fb_get_device_status() == fb.FB_OK
    try:
        fb.fb_debug_set_inblock_rows(rows)   # 64: the warp-per-rows small-block kernel
        fb.fb_debug_set_wait_limit_ns(1_000_000)
        fb.fb_debug_set_stall(True)
        fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, a, l, ws)
        status_prefix = fb.fb_get_device_status()
        fb.fb_attn_inblock(desc, qd, kind, vind, o, lse, [a], [l])
        status = fb.fb_get_device_status()
    finally:
        fb.fb_debug_set_stall(False)
        fb.fb_debug_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert status_prefix == fb.FB_ETIMEOUT, fb.status_string(status_prefix)
    assert status == fb.FB_ETIMEOUT, fb.status_string(status)

    # the status word was cleared by the read, and the context still works
    try:
        fb.fb_attn_outblock(desc, qd, kpd, vpd, Lp, a, l, ws)
        fb.fb_attn_inblock(desc, qd, kind, vind, o, lse, [a], [l])
    finally:
        fb.fb_debug_set_inblock_rows(0)
    assert fb.fb_get_device_status() == fb.FB_OK
    sc = 1.0 / np.sqrt(D)
    O, L = orc.full_attention(orc.to64(q), orc.to64(kin), orc.to64(vin), orc.to64(kp), orc.to64(vp), Lp, sc)
    assert_o_close(o, O, TOL["bf16"], "O after recovery")
    assert_lse_close(lse, L, TOL["bf16"], "LSE after recovery")
