"""fb_attn_outblock_noalloc: block-external attention for callers that cannot
allocate device memory (their host framework owns the pool, or they may not
allocate while serving).  Its split-KV scratch is a fixed array inside the
library, so the test checks it against fb_attn_outblock with caller scratch,
and against the fp64 oracle, on two calls in a row (the second call reuses
whatever the first left in the array), and that a call needing more than the
array is refused.

This file sorts last so that a run stopping at the first failure has run every
other test before it; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from block_diffusion_attention_flashblock_b200 import fb
from block_diffusion_attention_flashblock_b200 import workloads as wl
from oracle import flashblock_oracle as orc

from _gpu_common import TOL, assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, Nb, Lp, seed):
    q = wl.tensor((B, Hq, Nb, 128), seed, 0.5).cuda()
    kin = torch.empty(B, Hkv, Nb, 128, dtype=torch.bfloat16, device="cuda")
    kp = wl.tensor((B, Hkv, Lp + 32, 128), seed + 1, 0.5).cuda()
    vp = wl.tensor((B, Hkv, Lp + 32, 128), seed + 2, 0.5).cuda()
    return q, kin, kp, vp


@pytest.mark.parametrize("shape", [(1, 32, 8, 32, 8192), (2, 16, 4, 64, 3000), (1, 4, 4, 32, 700)],
                         ids=lambda s: "x".join(map(str, s)))
def test_noalloc_matches_scratch_version_twice(shape):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, Hq, Hkv, Nb, Lp = shape
    for call, seed in enumerate((101, 202)):       # two calls in a row, different inputs
        q, kin, kp, vp = _inputs(B, Hq, Hkv, Nb, Lp, seed)
        a_ref = torch.empty(B, Hq, Nb, 128, device="cuda"); l_ref = torch.empty(B, Hq, Nb, device="cuda")
        desc = fb.make_desc(q, kin, kp, a_ref)
        ws = torch.empty(fb.fb_outblock_workspace_bytes(desc, Lp), dtype=torch.uint8, device="cuda")
        fb.fb_attn_outblock(desc, q, kp, vp, Lp, a_ref, l_ref, ws)
        a = torch.full_like(a_ref, float("nan")); l = torch.full_like(l_ref, float("nan"))
        fb.fb_attn_outblock_noalloc(desc, q, kp, vp, Lp, a, l)
        torch.cuda.synchronize()
        assert fb.fb_get_device_status() == fb.FB_OK
        assert_o_close(a, a_ref.double().cpu().numpy(), TOL["bf16"], f"A_out, call {call}")
        assert_lse_close(l, l_ref.double().cpu().numpy(), TOL["bf16"], f"L_out, call {call}")
        # and independently against the fp64 oracle on the same inputs
        A, L = orc.outblock(orc.to64(q.cpu()), orc.to64(kp.cpu()), orc.to64(vp.cpu()), Lp, 1 / np.sqrt(128))
        assert_o_close(a, A, TOL["bf16"], f"A_out vs oracle, call {call}")
        assert_lse_close(l, L, TOL["bf16"], f"L_out vs oracle, call {call}")


def test_noalloc_refuses_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # 4 x 32 heads x 1024 queries: one split partial alone exceeds the array
    q = torch.empty(4, 32, 1024, 128, dtype=torch.bfloat16, device="cuda")
    kin = torch.empty(4, 8, 1024, 128, dtype=torch.bfloat16, device="cuda")
    kp = torch.empty(4, 8, 4096, 128, dtype=torch.bfloat16, device="cuda")
    a = torch.empty(4, 32, 1024, 128, device="cuda"); l = torch.empty(4, 32, 1024, device="cuda")
    desc = fb.make_desc(q, kin, kp, a)
    assert fb.fb_outblock_workspace_bytes(desc, 4096) > fb.FB_NOALLOC_SCRATCH_BYTES
    with pytest.raises(fb.FbError) as e:
        fb.fb_attn_outblock_noalloc(desc, q, kp, kp, 4096, a, l)
    assert e.value.status == fb.FB_ENOSPACE
