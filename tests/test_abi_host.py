"""The C-ABI library on the host (no GPU needed): it loads, exports every
function include/fb.h declares, and rejects bad arguments with the documented
status before any launch.  Pointers here are fake addresses that are never
dereferenced: every call below must fail its host-side checks first."""
import ctypes as C

import pytest
import torch

from block_diffusion_attention_flashblock_b200 import fb, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return fb.lib()


def test_exports_every_declared_symbol(L):
    names = fb.header_functions()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(names) == set(fb._SIGS), "binding and header disagree"


def test_status_strings(L):
    for s in range(9):
        assert fb.status_string(s).startswith("FB_")
    assert fb.status_string(FB := fb.FB_ETIMEOUT).startswith("FB_ETIMEOUT")
    assert L.fb_version() >> 16 == 1


def _desc(**kw):
    q = torch.empty(1, 8, 32, 128, dtype=torch.bfloat16)
    kin = torch.empty(1, 2, 32, 128, dtype=torch.bfloat16)
    kp = torch.empty(1, 2, 512, 128, dtype=torch.bfloat16)
    d = fb.make_desc(q, kin, kp, q)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced


def _outblock(L, d, q=FAKE, kp=FAKE, vp=FAKE, plen=256, sel=None, sel_k=0, a=FAKE, l=FAKE,
              ar=None, lr=None, ws=FAKE, wsb=1 << 30):
    return L.fb_attn_outblock(C.byref(d), q, kp, vp, plen, sel, sel_k, a, l, ar, lr, ws, wsb, None)


def test_outblock_argument_checks(L):
    assert L.fb_attn_outblock(None, FAKE, FAKE, FAKE, 1, None, 0, FAKE, FAKE, None, None, FAKE, 1, None) \
        == fb.FB_EINVAL
    assert _outblock(L, _desc(D=96)) == fb.FB_EUNSUPPORTED
    assert _outblock(L, _desc(Hkv=3)) == fb.FB_EINVAL
    assert _outblock(L, _desc(in_dtype=7)) == fb.FB_EDTYPE
    assert _outblock(L, _desc(B=0)) == fb.FB_EINVAL
    d = _desc(); d.q_strides[2] = 100        # 200 bytes: not a multiple of 16
    assert _outblock(L, d) == fb.FB_EALIGN
    assert _outblock(L, _desc(), q=FAKE + 8) == fb.FB_EALIGN
    assert _outblock(L, _desc(), q=None) == fb.FB_EINVAL
    assert _outblock(L, _desc(), plen=513) == fb.FB_EINVAL          # beyond kp_capacity
    assert _outblock(L, _desc(), plen=-1) == fb.FB_EINVAL
    assert _outblock(L, _desc(), sel=FAKE, sel_k=300) == fb.FB_EINVAL   # sel_k > prefix
    assert _outblock(L, _desc(), ar=FAKE, lr=FAKE) == fb.FB_EINVAL      # residual without sel
    assert _outblock(L, _desc(), wsb=16) == fb.FB_ENOSPACE
    assert _outblock(L, _desc(), ws=None) == fb.FB_ENOSPACE
    assert _outblock(L, _desc(scale=-1.0)) == fb.FB_EINVAL


def test_workspace_sizes_grow_with_prefix(L):
    d = _desc()
    n1 = fb.fb_outblock_workspace_bytes(d, 64)
    n2 = fb.fb_outblock_workspace_bytes(d, 1 << 16)
    assert 0 < n1 <= n2
    assert fb.fb_outblock_workspace_bytes(d, 1 << 16, 2048) >= n2


def test_inblock_merge_append_checks(L):
    d = _desc()
    ptrs = (C.c_void_p * 8)(*[FAKE] * 8)
    assert L.fb_attn_inblock(C.byref(d), FAKE, FAKE, FAKE, 8, ptrs, ptrs, FAKE, None, None) == fb.FB_EINVAL
    assert L.fb_attn_inblock(C.byref(d), FAKE, FAKE, FAKE, -1, ptrs, ptrs, FAKE, None, None) == fb.FB_EINVAL
    assert L.fb_attn_inblock(C.byref(d), FAKE, None, FAKE, 0, None, None, FAKE, None, None) == fb.FB_EINVAL
    bad = (C.c_void_p * 1)(FAKE + 4)
    assert L.fb_attn_inblock(C.byref(d), FAKE, FAKE, FAKE, 1, bad, bad, FAKE, None, None) == fb.FB_EALIGN
    assert L.fb_merge(C.byref(d), 0, ptrs, ptrs, FAKE, None, None) == fb.FB_EINVAL
    assert L.fb_merge(C.byref(d), 9, ptrs, ptrs, FAKE, None, None) == fb.FB_EINVAL
    assert L.fb_kv_append(C.byref(d), FAKE, FAKE, 500, FAKE, FAKE, None) == fb.FB_EINVAL  # 500+32 > 512
    assert L.fb_kv_append(C.byref(d), FAKE, FAKE, 0, FAKE + 2, FAKE, None) == fb.FB_EALIGN


def test_cache_and_step_checks(L):
    d = _desc()
    n = fb.fb_cache_workspace_bytes(d, 0, 512)
    assert n > 0
    h = C.c_void_p(0)
    assert L.fb_cache_create(C.byref(d), 0, 512, 0, FAKE, n - 1, None, C.byref(h)) == fb.FB_ENOSPACE
    assert L.fb_cache_create(C.byref(d), 0, 512, 0, FAKE + 16, n, None, C.byref(h)) == fb.FB_EALIGN
    assert L.fb_cache_create(C.byref(d), 64, 512, 0, FAKE, n, None, C.byref(h)) == fb.FB_EINVAL
    assert L.fb_cache_create(C.byref(d), 0, 512, 0, FAKE, n, None, C.byref(h)) == fb.FB_OK
    a = fb.fb_step_args()
    a.q = a.kin = a.vin = a.kp = a.vp = a.o = FAKE
    a.prefix_len, a.M, a.tau = 256, 0, 4
    a.sel, a.sel_k = FAKE, 16
    assert L.fb_step(h, C.byref(a), None) == fb.FB_ESTATE          # sparse step, dense handle
    a.sel, a.sel_k = None, 0
    a.gamma = FAKE
    assert L.fb_step(h, C.byref(a), None) == fb.FB_ESTATE          # gamma step, no gamma state
    a.gamma = None
    a.prefix_len = 4096
    assert L.fb_step(h, C.byref(a), None) == fb.FB_EINVAL          # beyond max_prefix
    a.prefix_len = 256; a.M = -1
    assert L.fb_step(h, C.byref(a), None) == fb.FB_EINVAL
    a.M = 0; a.o = FAKE + 1
    assert L.fb_step(h, C.byref(a), None) == fb.FB_EALIGN
    r = C.c_int32(-1)
    assert L.fb_cache_last_step(h, C.byref(r)) == fb.FB_OK and r.value == 0
    assert L.fb_cache_begin_block(h, None) == fb.FB_OK
    assert L.fb_cache_destroy(h) == fb.FB_OK
    assert L.fb_cache_destroy(None) == fb.FB_EINVAL


def test_active_subset_step_checks(L):
    """fb_step with an active-query list: the flag, the count and the list's
    alignment are checked before any launch."""
    d = _desc()
    h = C.c_void_p(0)
    n = fb.fb_cache_workspace_bytes(d, 0, 512)
    assert L.fb_cache_create(C.byref(d), 0, 512, 0, FAKE, n, None, C.byref(h)) == fb.FB_OK
    a = fb.fb_step_args()
    a.q = a.kin = a.vin = a.kp = a.vp = a.o = FAKE
    a.prefix_len, a.M, a.tau = 256, 0, 4
    a.active, a.n_active = FAKE, 8
    assert L.fb_step(h, C.byref(a), None) == fb.FB_ESTATE          # no FB_CACHE_ACTIVE
    assert L.fb_cache_destroy(h) == fb.FB_OK
    flags = fb.FB_CACHE_ACTIVE | fb.FB_CACHE_SPARSE
    n2 = fb.fb_cache_workspace_bytes(d, flags, 512, 64)
    assert n2 > fb.fb_cache_workspace_bytes(d, fb.FB_CACHE_SPARSE, 512, 64)   # room for the compact block
    assert L.fb_cache_create(C.byref(d), flags, 512, 64, FAKE, n2, None, C.byref(h)) == fb.FB_OK
    for bad in (0, 33, -1):
        a.n_active = bad
        assert L.fb_step(h, C.byref(a), None) == fb.FB_EINVAL
    a.n_active = 8
    a.active = FAKE + 4
    assert L.fb_step(h, C.byref(a), None) == fb.FB_EALIGN
    a.active = FAKE
    a.sel, a.sel_k = FAKE, 16
    assert L.fb_step(h, C.byref(a), None) == fb.FB_EUNSUPPORTED     # with a sparse selection
    assert L.fb_cache_destroy(h) == fb.FB_OK


def _select(L, d, plen=256, k=16, sel=FAKE, ws=FAKE, wsb=1 << 30, mass=None):
    return L.fb_select_mass(C.byref(d), FAKE, FAKE, FAKE, plen, k, sel, mass, ws, wsb, None)


def test_select_mass_checks(L):
    d = _desc()
    assert fb.fb_select_workspace_bytes(d, 512) >= fb.fb_outblock_workspace_bytes(d, 512)
    assert _select(L, d, k=257) == fb.FB_EINVAL          # k > prefix
    assert _select(L, d, k=-1) == fb.FB_EINVAL
    assert _select(L, d, plen=0, k=0) == fb.FB_EINVAL
    assert _select(L, d, plen=513) == fb.FB_EINVAL       # beyond kp_capacity
    assert _select(L, d, sel=FAKE + 4) == fb.FB_EALIGN
    assert _select(L, d, wsb=64) == fb.FB_ENOSPACE
    assert _select(L, d, sel=None) == fb.FB_EINVAL       # k > 0 needs somewhere to write
    # the KV head's G * Nb = 4 * 64 query rows do not fit one 128-row tile
    q = torch.empty(1, 8, 64, 128, dtype=torch.bfloat16)
    d64 = fb.make_desc(q, torch.empty(1, 2, 64, 128, dtype=torch.bfloat16),
                       torch.empty(1, 2, 512, 128, dtype=torch.bfloat16), q)
    assert _select(L, d64) == fb.FB_EUNSUPPORTED
    assert _select(L, _desc(in_dtype=fb.FB_F32, out_dtype=fb.FB_F32)) in (fb.FB_EUNSUPPORTED, fb.FB_EALIGN)


def test_debug_hooks_validate_and_reset(L):
    assert L.fb_debug_set_prefix_kernel(5) == fb.FB_EINVAL
    assert L.fb_debug_set_prefix_kernel(-1) == fb.FB_EINVAL
    for which in (4, 3, 2, 1, 0):
        assert L.fb_debug_set_prefix_kernel(which) == fb.FB_OK
    for on in (0, 1):
        assert L.fb_debug_set_pdl(on) == fb.FB_OK
        assert L.fb_debug_set_stall(on) == fb.FB_OK
    assert L.fb_debug_set_stall(0) == fb.FB_OK
    assert L.fb_debug_set_wait_limit_ns(2_000_000_000) == fb.FB_OK
    for rows in (2, 8, 48, 128, -1):
        assert L.fb_debug_set_inblock_rows(rows) == fb.FB_EINVAL
    for rows in (1, 16, 32, 64, 0):
        assert L.fb_debug_set_inblock_rows(rows) == fb.FB_OK
