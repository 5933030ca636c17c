"""ctypes binding of libfb (include/fb.h), same names as the C ABI.

Argument marshalling only: tensors become device pointers and strides, the
current torch stream becomes the cudaStream_t; every step of the computation
runs in libfb's kernels.  Loading fails loudly if libfb.so has not been built.

Source of the method: "FlashBlock: Attention Caching for Efficient
Long-Context Block Diffusion" (summary sections "Mécanisme Central" and
"Stratégies de Réutilisation Adaptatives").
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfb.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "fb.h")

FB_OK, FB_EINVAL, FB_EALIGN, FB_EDTYPE, FB_EUNSUPPORTED = 0, 1, 2, 3, 4
FB_ESTATE, FB_ECUDA, FB_ETIMEOUT, FB_ENOSPACE = 5, 6, 7, 8
FB_F32, FB_BF16 = 0, 1
FB_MAX_PARTS = 8
FB_TAU_OFF = 2**31 - 1
FB_CACHE_SPARSE, FB_CACHE_GAMMA, FB_CACHE_ACTIVE = 1, 2, 4


class FbError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class fb_attn_desc(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("D", C.c_int32),
                ("Nb", C.c_int32), ("in_dtype", C.c_int32), ("out_dtype", C.c_int32),
                ("scale", C.c_float), ("kp_capacity", C.c_int64),
                ("q_strides", C.c_int64 * 3), ("kin_strides", C.c_int64 * 3),
                ("kp_strides", C.c_int64 * 3), ("o_strides", C.c_int64 * 3)]


class fb_step_args(C.Structure):
    _fields_ = [("q", C.c_void_p), ("kin", C.c_void_p), ("vin", C.c_void_p),
                ("kp", C.c_void_p), ("vp", C.c_void_p), ("prefix_len", C.c_int64),
                ("M", C.c_int32), ("tau", C.c_int32), ("gamma", C.c_void_p),
                ("sel", C.c_void_p), ("sel_k", C.c_int32), ("o", C.c_void_p),
                ("lse", C.c_void_p), ("reuse_out", C.c_void_p), ("sim_out", C.c_void_p),
                ("active", C.c_void_p), ("n_active", C.c_int32)]


_P = C.c_void_p
_SIGS = {
    "fb_status_string": (C.c_char_p, [C.c_int]),
    "fb_version": (C.c_int32, []),
    "fb_outblock_workspace_bytes": (C.c_int, [_P, C.c_int64, C.c_int32, C.POINTER(C.c_size_t)]),
    "fb_attn_outblock": (C.c_int, [_P, _P, _P, _P, C.c_int64, _P, C.c_int32, _P, _P, _P, _P, _P,
                                   C.c_size_t, _P]),
    "fb_attn_outblock_noalloc": (C.c_int, [_P, _P, _P, _P, C.c_int64, _P, _P, _P]),
    "fb_attn_inblock": (C.c_int, [_P, _P, _P, _P, C.c_int32, _P, _P, _P, _P, _P]),
    "fb_select_workspace_bytes": (C.c_int, [_P, C.c_int64, C.POINTER(C.c_size_t)]),
    "fb_select_mass": (C.c_int, [_P, _P, _P, _P, C.c_int64, C.c_int32, _P, _P, _P, C.c_size_t, _P]),
    "fb_merge": (C.c_int, [_P, C.c_int32, _P, _P, _P, _P, _P]),
    "fb_kv_append": (C.c_int, [_P, _P, _P, C.c_int64, _P, _P, _P]),
    "fb_cache_workspace_bytes": (C.c_int, [_P, C.c_int32, C.c_int64, C.c_int32, C.POINTER(C.c_size_t)]),
    "fb_cache_create": (C.c_int, [_P, C.c_int32, C.c_int64, C.c_int32, _P, C.c_size_t, _P,
                                  C.POINTER(C.c_void_p)]),
    "fb_cache_destroy": (C.c_int, [_P]),
    "fb_cache_begin_block": (C.c_int, [_P, _P]),
    "fb_step": (C.c_int, [_P, _P, _P]),
    "fb_cache_last_step": (C.c_int, [_P, C.POINTER(C.c_int32)]),
    "fb_get_device_status": (C.c_int, [_P, C.POINTER(C.c_int)]),
    "fb_debug_set_wait_limit_ns": (C.c_int, [C.c_uint64]),
    "fb_debug_set_pdl": (C.c_int, [C.c_int32]),
    "fb_debug_set_inblock_loads": (C.c_int, [C.c_int32]),
    "fb_debug_set_inblock_rows": (C.c_int, [C.c_int32]),
    "fb_debug_set_inblock_kernel": (C.c_int, [C.c_int32]),
    "fb_debug_set_stall": (C.c_int, [C.c_int32]),
    "fb_profile_enable": (C.c_int, [C.c_int32]),
    "fb_debug_set_prefix_kernel": (C.c_int, [C.c_int32]),
    "fb_profile_read": (C.c_int, [C.c_int32, _P, _P, _P]),
}

_lib = None


def lib() -> C.CDLL:
    """Load libfb.so once; raise if it is missing (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfb.so is not built ({LIB_PATH}); run "
                               "`python -m block_diffusion_attention_flashblock_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of the functions include/fb.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fb_[a-z0-9_]+)\s*\(", src)))


def status_string(s: int) -> str:
    return lib().fb_status_string(int(s)).decode()


def _check(st: int, what: str):
    if st != FB_OK:
        raise FbError(st, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return FB_F32
    if dt == torch.bfloat16:
        return FB_BF16
    raise FbError(FB_EDTYPE, f"dtype {dt}")


def make_desc(q: torch.Tensor, kin: torch.Tensor, kp: torch.Tensor, o: torch.Tensor,
              scale: float = 0.0) -> fb_attn_desc:
    """Descriptor from tensors Q [B,Hq,Nb,D], K_in [B,Hkv,Nb,D], K_p [B,Hkv,cap,D], O [B,Hq,Nb,D]."""
    B, Hq, Nb, D = q.shape
    d = fb_attn_desc()
    d.B, d.Hq, d.Hkv, d.D, d.Nb = B, Hq, kin.shape[1], D, Nb
    d.in_dtype = _dtype_code(q.dtype)
    d.out_dtype = _dtype_code(o.dtype)
    d.scale = float(scale)
    d.kp_capacity = kp.shape[2]
    for name, t in (("q_strides", q), ("kin_strides", kin), ("kp_strides", kp), ("o_strides", o)):
        if t.stride(3) != 1:
            raise FbError(FB_EINVAL, f"{name}: head dimension must be contiguous")
        setattr(d, name, (C.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2)))
    return d


def _parts(a_parts: Sequence[torch.Tensor], l_parts: Sequence[torch.Tensor]):
    n = len(a_parts)
    A = (C.c_void_p * max(n, 1))(*[t.data_ptr() for t in a_parts])
    Lp = (C.c_void_p * max(n, 1))(*[t.data_ptr() for t in l_parts])
    return n, A, Lp


# --------------------------------------------------------------- C calls ---
def fb_outblock_workspace_bytes(desc: fb_attn_desc, prefix_len: int, sel_k: int = 0) -> int:
    n = C.c_size_t(0)
    _check(lib().fb_outblock_workspace_bytes(C.byref(desc), prefix_len, sel_k, C.byref(n)),
           "fb_outblock_workspace_bytes")
    return n.value


def _sel_ptr(sel: Optional[torch.Tensor]) -> Optional[int]:
    """A selection list marks a sparse call even when it is empty (k = 0): an
    empty tensor has no storage, so pass the address of a one-element stand-in."""
    if sel is None:
        return None
    if sel.numel() == 0:
        global _EMPTY_SEL
        if _EMPTY_SEL is None or _EMPTY_SEL.device != sel.device:
            _EMPTY_SEL = torch.zeros(4, dtype=torch.int32, device=sel.device)
        return _EMPTY_SEL.data_ptr()
    return sel.data_ptr()


_EMPTY_SEL = None


def fb_attn_outblock(desc, q, kp, vp, prefix_len, a_out, l_out, ws, sel=None, sel_k=0,
                     a_res=None, l_res=None, stream=None):
    _check(lib().fb_attn_outblock(C.byref(desc), _ptr(q), _ptr(kp), _ptr(vp), prefix_len, _sel_ptr(sel),
                                  sel_k, _ptr(a_out), _ptr(l_out), _ptr(a_res), _ptr(l_res), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "fb_attn_outblock")


FB_NOALLOC_SCRATCH_BYTES = 64 << 20


def fb_attn_outblock_noalloc(desc, q, kp, vp, prefix_len, a_out, l_out, stream=None):
    """fb_attn_outblock (dense) with its scratch in the library's fixed array."""
    _check(lib().fb_attn_outblock_noalloc(C.byref(desc), _ptr(q), _ptr(kp), _ptr(vp), prefix_len,
                                          _ptr(a_out), _ptr(l_out), _stream(stream)),
           "fb_attn_outblock_noalloc")


def fb_select_workspace_bytes(desc, prefix_len: int) -> int:
    n = C.c_size_t(0)
    _check(lib().fb_select_workspace_bytes(C.byref(desc), prefix_len, C.byref(n)), "fb_select_workspace_bytes")
    return n.value


def fb_select_mass(desc, q, kp, vp, prefix_len, k, sel_out, ws, mass_out=None, stream=None):
    """Top-k prefix keys per (b, query head) by attention mass into sel_out [B, Hq, k]."""
    _check(lib().fb_select_mass(C.byref(desc), _ptr(q), _ptr(kp), _ptr(vp), prefix_len, k, _ptr(sel_out),
                                _ptr(mass_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "fb_select_mass")


def fb_attn_inblock(desc, q, kin, vin, o, lse=None, a_parts=(), l_parts=(), stream=None):
    n, A, Lp = _parts(a_parts, l_parts)
    _check(lib().fb_attn_inblock(C.byref(desc), _ptr(q), _ptr(kin), _ptr(vin), n, A, Lp, _ptr(o),
                                 _ptr(lse), _stream(stream)), "fb_attn_inblock")


def fb_merge(desc, a_parts, l_parts, o, lse=None, stream=None):
    n, A, Lp = _parts(a_parts, l_parts)
    _check(lib().fb_merge(C.byref(desc), n, A, Lp, _ptr(o), _ptr(lse), _stream(stream)), "fb_merge")


def fb_kv_append(desc, kp, vp, prefix_len, kin, vin, stream=None):
    _check(lib().fb_kv_append(C.byref(desc), _ptr(kp), _ptr(vp), prefix_len, _ptr(kin), _ptr(vin),
                              _stream(stream)), "fb_kv_append")


def fb_cache_workspace_bytes(desc, flags, max_prefix, max_sel_k=0) -> int:
    n = C.c_size_t(0)
    _check(lib().fb_cache_workspace_bytes(C.byref(desc), flags, max_prefix, max_sel_k, C.byref(n)),
           "fb_cache_workspace_bytes")
    return n.value


def fb_cache_create(desc, flags, max_prefix, max_sel_k, dev_mem: torch.Tensor, stream=None):
    h = C.c_void_p(0)
    _check(lib().fb_cache_create(C.byref(desc), flags, max_prefix, max_sel_k, _ptr(dev_mem),
                                 dev_mem.numel() * dev_mem.element_size(), _stream(stream), C.byref(h)),
           "fb_cache_create")
    return h


def fb_cache_destroy(h):
    _check(lib().fb_cache_destroy(h), "fb_cache_destroy")


def fb_cache_begin_block(h, stream=None):
    _check(lib().fb_cache_begin_block(h, _stream(stream)), "fb_cache_begin_block")


def fb_step(h, q, kin, vin, kp, vp, prefix_len, M, tau, o, lse=None, gamma=None, sel=None,
            reuse_out=None, sim_out=None, stream=None, active=None):
    """active: optional device int32 [B, n_active] block positions still unlocked."""
    a = fb_step_args()
    a.active = _ptr(active)
    a.n_active = 0 if active is None else active.shape[-1]
    a.q, a.kin, a.vin, a.kp, a.vp = _ptr(q), _ptr(kin), _ptr(vin), _ptr(kp), _ptr(vp)
    a.prefix_len, a.M, a.tau = prefix_len, M, tau
    a.gamma, a.sel = _ptr(gamma), _sel_ptr(sel)
    a.sel_k = 0 if sel is None else sel.shape[-1]
    a.o, a.lse, a.reuse_out, a.sim_out = _ptr(o), _ptr(lse), _ptr(reuse_out), _ptr(sim_out)
    _check(lib().fb_step(h, C.byref(a), _stream(stream)), "fb_step")


def fb_cache_last_step(h) -> int:
    r = C.c_int32(0)
    _check(lib().fb_cache_last_step(h, C.byref(r)), "fb_cache_last_step")
    return r.value


def fb_get_device_status(stream=None) -> int:
    s = C.c_int(0)
    _check(lib().fb_get_device_status(_stream(stream), C.byref(s)), "fb_get_device_status")
    return s.value


PREFIX_AUTO, PREFIX_GENERIC, PREFIX_TC, PREFIX_TC_NO_CLUSTER, PREFIX_TC_CLUSTER = 0, 1, 2, 3, 4


def fb_debug_set_prefix_kernel(which: int):
    _check(lib().fb_debug_set_prefix_kernel(which), "fb_debug_set_prefix_kernel")


def fb_debug_set_wait_limit_ns(ns: int):
    _check(lib().fb_debug_set_wait_limit_ns(ns), "fb_debug_set_wait_limit_ns")


def fb_debug_set_pdl(on: bool):
    _check(lib().fb_debug_set_pdl(1 if on else 0), "fb_debug_set_pdl")


def fb_debug_set_inblock_kernel(which: int):
    _check(lib().fb_debug_set_inblock_kernel(which), "fb_debug_set_inblock_kernel")


def fb_debug_set_inblock_loads(bulk: bool):
    _check(lib().fb_debug_set_inblock_loads(1 if bulk else 0), "fb_debug_set_inblock_loads")


def fb_debug_set_inblock_rows(rows: int):
    _check(lib().fb_debug_set_inblock_rows(int(rows)), "fb_debug_set_inblock_rows")


def fb_debug_set_stall(on: bool):
    _check(lib().fb_debug_set_stall(1 if on else 0), "fb_debug_set_stall")


FB_PROFILE_KINDS = 3
PROFILE_KIND_NAMES = ("prefix_attention", "inblock_merge", "aux")


def fb_profile_enable(on: bool):
    _check(lib().fb_profile_enable(1 if on else 0), "fb_profile_enable")


def fb_profile_read(reset: bool = True):
    """Per kernel kind: (launches, total event-timed ms, algorithmic bytes)."""
    n = (C.c_int64 * FB_PROFILE_KINDS)()
    ms = (C.c_double * FB_PROFILE_KINDS)()
    by = (C.c_double * FB_PROFILE_KINDS)()
    _check(lib().fb_profile_read(1 if reset else 0, n, ms, by), "fb_profile_read")
    return {PROFILE_KIND_NAMES[k]: (n[k], ms[k], by[k]) for k in range(FB_PROFILE_KINDS)}


# ------------------------------------------------------- a stateful layer ---
class FlashBlockLayer:
    """One attention layer's FlashBlock state: a cache handle over a device buffer.

    Thin convenience over fb_cache_* / fb_step; all work is in libfb.
    """

    def __init__(self, q_like, kin_like, kp, o_like, max_prefix, gamma=False, sparse=False,
                 max_sel_k=0, scale=0.0, active=False):
        self.desc = make_desc(q_like, kin_like, kp, o_like, scale)
        self.flags = ((FB_CACHE_GAMMA if gamma else 0) | (FB_CACHE_SPARSE if sparse else 0)
                      | (FB_CACHE_ACTIVE if active else 0))
        nbytes = fb_cache_workspace_bytes(self.desc, self.flags, max_prefix, max_sel_k)
        self.mem = torch.empty(nbytes, dtype=torch.uint8, device=kp.device)
        self.handle = fb_cache_create(self.desc, self.flags, max_prefix, max_sel_k, self.mem)

    def begin_block(self):
        fb_cache_begin_block(self.handle)

    def step(self, q, kin, vin, kp, vp, prefix_len, M, tau, o, lse=None, gamma=None, sel=None,
             reuse_out=None, sim_out=None, active=None):
        fb_step(self.handle, q, kin, vin, kp, vp, prefix_len, M, tau, o, lse, gamma, sel,
                reuse_out, sim_out, active=active)

    def last_recomputed(self) -> bool:
        return bool(fb_cache_last_step(self.handle))

    def close(self):
        if self.handle is not None:
            fb_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
