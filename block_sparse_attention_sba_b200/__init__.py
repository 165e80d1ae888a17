"""Python binding of libsba (training-free Top-p block-sparse attention, B200).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libsba.so``; torch provides device memory and streams. The functions
``sba_*`` mirror the C ABI in ``include/sba.h`` one to one (same names, same
argument order, torch tensors in place of device pointers, ``stream`` taken
from torch's current stream when omitted). ``Plan`` and ``SparseAttention``
are conveniences built only from those calls.

Importing fails loudly when the library has not been built; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsba.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python block_sparse_attention_sba_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

SBA_OK = 0
SBA_ERR_INVALID_ARG = -1
SBA_ERR_UNSUPPORTED = -2
SBA_ERR_CUDA = -3
SBA_ERR_CAPACITY = -4
SBA_ERR_DEVICE_TIMEOUT = -5
SBA_ERR_DEVICE_CHECK = -6
SBA_F32 = 0
SBA_BF16 = 1
SBA_SCHED_LPT = 0
SBA_SCHED_HEAD_MAJOR = 1
SBA_ORDER_CUBE = 0
SBA_ORDER_HILBERT = 1

EXPORTED = ["sba_plan_create", "sba_plan_destroy", "sba_plan_query", "sba_workspace_init",
            "sba_reorder", "sba_unreorder", "sba_build_mask", "sba_attention",
            "sba_check_device_status", "sba_debug_timeout_probe", "sba_debug_exp2_poly",
            "sba_perm_export",
            "sba_attention_grid_size", "sba_status_string", "sba_last_error",
            "sba_build_mask_noalloc", "sba_build_stripe_mask", "sba_smooth_v",
            "sba_attention_lowbit", "sba_noalloc_status"]


class sba_geometry(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
                ("Hh", ctypes.c_int32), ("W", ctypes.c_int32), ("d", ctypes.c_int32),
                ("ct", ctypes.c_int32), ("ch", ctypes.c_int32), ("cw", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("sB", ctypes.c_int64), ("sH", ctypes.c_int64),
                ("sN", ctypes.c_int64), ("order", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class sba_stripe(ctypes.Structure):
    """One head's stripe-mask parameters (see sba_build_stripe_mask in sba.h)."""
    _fields_ = [("Tw", ctypes.c_int32), ("To", ctypes.c_int32), ("Ts", ctypes.c_int32),
                ("Sw", ctypes.c_int32), ("So", ctypes.c_int32), ("Ss", ctypes.c_int32)]


class sba_plan_info(ctypes.Structure):
    _fields_ = [("nT", ctypes.c_int32), ("nH", ctypes.c_int32), ("nW", ctypes.c_int32),
                ("nb", ctypes.c_int32), ("bs", ctypes.c_int32), ("Npad", ctypes.c_int32),
                ("rows", ctypes.c_int32), ("words", ctypes.c_int32), ("max_nnz", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_size_t)]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_sig = {
    "sba_plan_create": [ctypes.POINTER(sba_geometry), ctypes.POINTER(_vp)],
    "sba_plan_destroy": [_vp],
    "sba_plan_query": [_vp, ctypes.POINTER(sba_plan_info)],
    "sba_workspace_init": [_vp, _vp, _vp],
    "sba_reorder": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "sba_unreorder": [_vp, _vp, _vp, _vp, _vp],
    "sba_build_mask": [_vp, _vp, _vp, ctypes.POINTER(ctypes.c_float), _i32, _vp, _vp, _vp, _vp,
                       _vp, _vp, _vp],
    "sba_attention": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp],
    "sba_build_mask_noalloc": [_vp, _vp, _vp, ctypes.POINTER(ctypes.c_float), _i32, _vp, _vp, _vp,
                               _vp, _vp, _vp],
    "sba_build_stripe_mask": [_vp, ctypes.POINTER(sba_stripe), _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "sba_smooth_v": [_vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "sba_attention_lowbit": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "sba_check_device_status": [_vp, _vp, _vp],
    "sba_noalloc_status": [_vp],
    "sba_debug_timeout_probe": [_vp, _vp, ctypes.c_uint64, _vp],
    "sba_debug_exp2_poly": [_vp, _vp, ctypes.c_int64, _vp],
    "sba_perm_export": [_vp, ctypes.POINTER(ctypes.c_int32)],
    "sba_attention_grid_size": [],
    "sba_status_string": [_i32],
    "sba_last_error": [],
}
for _name, _args in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _i32
_lib.sba_plan_destroy.restype = None
_lib.sba_status_string.restype = ctypes.c_char_p
_lib.sba_last_error.restype = ctypes.c_char_p


class SbaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.sba_last_error().decode()
        super().__init__(f"{where}: {_lib.sba_status_string(status).decode()} ({msg})")


def _check(status: int, where: str) -> int:
    if status != SBA_OK:
        raise SbaError(status, where)
    return status


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------- raw C ABI

_plan_heads = {}  # plan handle -> H (the C side reads top_p[0..H-1])


def sba_plan_create(geom: sba_geometry) -> int:
    h = _vp()
    _check(_lib.sba_plan_create(ctypes.byref(geom), ctypes.byref(h)), "sba_plan_create")
    _plan_heads[h.value] = int(geom.H)
    return h.value


def sba_plan_destroy(plan: int) -> None:
    _plan_heads.pop(plan, None)
    _lib.sba_plan_destroy(plan)


def sba_plan_query(plan: int) -> sba_plan_info:
    info = sba_plan_info()
    _check(_lib.sba_plan_query(plan, ctypes.byref(info)), "sba_plan_query")
    return info


def sba_workspace_init(plan: int, workspace, stream=None) -> None:
    _check(_lib.sba_workspace_init(plan, _ptr(workspace), _stream(stream)), "sba_workspace_init")


def sba_reorder(plan: int, q, k, v, qt, kt, vt, workspace=None, stream=None) -> None:
    _check(_lib.sba_reorder(plan, _ptr(q), _ptr(k), _ptr(v), _ptr(qt), _ptr(kt), _ptr(vt),
                            _ptr(workspace), _stream(stream)), "sba_reorder")


def sba_unreorder(plan: int, ot, o, workspace=None, stream=None) -> None:
    _check(_lib.sba_unreorder(plan, _ptr(ot), _ptr(o), _ptr(workspace), _stream(stream)),
           "sba_unreorder")


def _top_p_array(plan: int, top_p: Sequence[float]):
    """ctypes float array of one Top-p value per head (the C side reads H of
    them, so a shorter sequence is refused here instead of read past)."""
    H = _plan_heads.get(plan)
    if H is None:
        raise ValueError("unknown plan handle (create plans with sba_plan_create)")
    if len(top_p) != H:
        raise ValueError(f"top_p has {len(top_p)} values; the plan has H = {H} heads")
    return (ctypes.c_float * H)(*[float(x) for x in top_p])


def sba_build_mask(plan: int, qt, kt, top_p: Sequence[float], top_k: int, bitmask, row_cnt,
                   row_ptr, col_idx, work_order, workspace, stream=None) -> None:
    arr = _top_p_array(plan, top_p)
    _check(_lib.sba_build_mask(plan, _ptr(qt), _ptr(kt), arr, int(top_k), _ptr(bitmask),
                               _ptr(row_cnt), _ptr(row_ptr), _ptr(col_idx), _ptr(work_order),
                               _ptr(workspace), _stream(stream)), "sba_build_mask")


def sba_build_mask_noalloc(plan: int, qt, kt, top_p: Sequence[float], top_k: int, bitmask,
                           row_cnt, row_ptr, col_idx, work_order, stream=None) -> None:
    """sba_build_mask without a workspace: the library's static scratch is used
    instead (see include/sba.h for the size limit and the sharing rules)."""
    arr = _top_p_array(plan, top_p)
    _check(_lib.sba_build_mask_noalloc(plan, _ptr(qt), _ptr(kt), arr, int(top_k), _ptr(bitmask),
                                       _ptr(row_cnt), _ptr(row_ptr), _ptr(col_idx),
                                       _ptr(work_order), _stream(stream)), "sba_build_mask_noalloc")


def sba_build_stripe_mask(plan: int, params, bitmask, row_cnt, row_ptr, col_idx, work_order,
                          workspace, stream=None) -> None:
    """params: one (Tw, To, Ts, Sw, So, Ss) per head."""
    arr = (sba_stripe * len(params))(*[sba_stripe(*[int(x) for x in prm]) for prm in params])
    _check(_lib.sba_build_stripe_mask(plan, arr, _ptr(bitmask), _ptr(row_cnt), _ptr(row_ptr),
                                      _ptr(col_idx), _ptr(work_order), _ptr(workspace),
                                      _stream(stream)), "sba_build_stripe_mask")


def sba_smooth_v(plan: int, vt, vq, vmean, vexp, workspace, stream=None) -> None:
    _check(_lib.sba_smooth_v(plan, _ptr(vt), _ptr(vq), _ptr(vmean), _ptr(vexp), _ptr(workspace),
                             _stream(stream)), "sba_smooth_v")


def sba_attention_lowbit(plan: int, qt, kt, vq, vmean, vexp, row_ptr, col_idx, work_order, ot,
                         lse=None, trace=None, workspace=None, stream=None) -> None:
    _check(_lib.sba_attention_lowbit(plan, _ptr(qt), _ptr(kt), _ptr(vq), _ptr(vmean), _ptr(vexp),
                                     _ptr(row_ptr), _ptr(col_idx), _ptr(work_order), _ptr(ot),
                                     _ptr(lse), _ptr(trace), _ptr(workspace), _stream(stream)),
           "sba_attention_lowbit")


def sba_attention(plan: int, qt, kt, vt, row_ptr, col_idx, work_order, ot, lse=None,
                  sched: int = SBA_SCHED_LPT, trace=None, workspace=None, stream=None) -> None:
    _check(_lib.sba_attention(plan, _ptr(qt), _ptr(kt), _ptr(vt), _ptr(row_ptr), _ptr(col_idx),
                              _ptr(work_order), _ptr(ot), _ptr(lse), int(sched), _ptr(trace),
                              _ptr(workspace), _stream(stream)), "sba_attention")


def sba_noalloc_status(stream=None) -> int:
    """Status of sba_build_mask_noalloc's static scratch (syncs; does not
    raise on device-side errors)."""
    return _lib.sba_noalloc_status(_stream(stream))


def sba_check_device_status(plan: int, workspace, stream=None) -> int:
    """Returns the status code (does not raise on device-side errors)."""
    return _lib.sba_check_device_status(plan, _ptr(workspace), _stream(stream))


def sba_debug_exp2_poly(x, y, stream=None) -> None:
    """y = 2^x through the attention softmax's FMA-pipe exponential (fp32
    device tensors of equal length)."""
    import torch
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise SbaError(SBA_ERR_INVALID_ARG, "x and y must be fp32 tensors of equal length")
    _check(_lib.sba_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "sba_debug_exp2_poly")


def sba_debug_timeout_probe(plan: int, workspace, timeout_ns: int, stream=None) -> None:
    _check(_lib.sba_debug_timeout_probe(plan, _ptr(workspace), int(timeout_ns), _stream(stream)),
           "sba_debug_timeout_probe")


def sba_perm_export(plan: int, N: int):
    out = (ctypes.c_int32 * N)()
    _check(_lib.sba_perm_export(plan, out), "sba_perm_export")
    return list(out)


def sba_attention_grid_size() -> int:
    return _lib.sba_attention_grid_size()


def sba_status_string(status: int) -> str:
    return _lib.sba_status_string(status).decode()


def sba_last_error() -> str:
    return _lib.sba_last_error().decode()


# ------------------------------------------------------------- conveniences

class Plan:
    """Owns an sba_plan for one geometry. Strides are those of a [B, H, N, d]
    view of q/k/v/o (d contiguous)."""

    def __init__(self, B: int, H: int, T: int, Hh: int, W: int, d: int, cube,
                 dtype: str = "bf16", strides: Optional[Sequence[int]] = None,
                 order: str = "cube"):
        N = T * Hh * W
        if strides is None:
            strides = (H * N * d, N * d, d)
        self.geom = sba_geometry(B, H, T, Hh, W, d, cube[0], cube[1], cube[2],
                                 SBA_BF16 if dtype == "bf16" else SBA_F32,
                                 int(strides[0]), int(strides[1]), int(strides[2]),
                                 SBA_ORDER_HILBERT if order == "hilbert" else SBA_ORDER_CUBE, 0)
        self.order = order
        self.handle = sba_plan_create(self.geom)
        self.info = sba_plan_query(self.handle)
        self.B, self.H, self.T, self.Hh, self.W, self.d = B, H, T, Hh, W, d
        self.N = N
        self.dtype = dtype

    @classmethod
    def for_tensor(cls, q, T: int, Hh: int, W: int, cube, order: str = "cube") -> "Plan":
        B, H, N, d = q.shape
        assert N == T * Hh * W and q.stride(3) == 1
        import torch
        dt = "bf16" if q.dtype == torch.bfloat16 else "f32"
        return cls(B, H, T, Hh, W, d, cube, dt, (q.stride(0), q.stride(1), q.stride(2)), order)

    def __del__(self):
        h = getattr(self, "handle", None)
        if not h:
            return
        self.handle = None
        try:
            sba_plan_destroy(h)
        except (TypeError, AttributeError):
            # interpreter shutdown: the module's globals are already cleared
            # and the process releases the library with everything else
            pass


class SparseAttention:
    """Device buffers for one plan plus the four calls in order:
    reorder -> build_mask -> attention -> unreorder."""

    def __init__(self, plan: Plan, device="cuda", nnz_capacity: Optional[int] = None):
        import torch
        self.plan = plan
        inf = plan.info
        dt = torch.bfloat16 if plan.dtype == "bf16" else torch.float32
        B, H, d = plan.B, plan.H, plan.d
        mk = lambda *s, dtype=dt: torch.empty(*s, dtype=dtype, device=device)
        self.qt, self.kt, self.vt, self.ot = (mk(B, H, inf.Npad, d) for _ in range(4))
        self.bitmask = mk(inf.rows, inf.words, dtype=torch.int32)
        self.row_cnt = mk(inf.rows, dtype=torch.int32)
        self.row_ptr = mk(inf.rows + 1, dtype=torch.int32)
        self.col_idx = mk(nnz_capacity or inf.max_nnz, dtype=torch.int32)
        self.work_order = mk(inf.rows, dtype=torch.int32)
        self.lse = mk(B, H, inf.Npad, dtype=torch.float32)
        self.workspace = torch.zeros(inf.workspace_bytes, dtype=torch.uint8, device=device)
        if torch.cuda.is_available():
            sba_workspace_init(plan.handle, self.workspace)

    def __call__(self, q, k, v, top_p, top_k: int, o=None, sched: int = SBA_SCHED_LPT,
                 trace=None, stream=None):
        import torch
        p = self.plan
        h = p.handle
        if o is None:
            o = torch.empty_like(q)
        top_p = list(top_p) if len(top_p) == p.H else [float(top_p[0])] * p.H
        sba_reorder(h, q, k, v, self.qt, self.kt, self.vt, self.workspace, stream)
        sba_build_mask(h, self.qt, self.kt, top_p, top_k, self.bitmask, self.row_cnt,
                       self.row_ptr, self.col_idx, self.work_order, self.workspace, stream)
        sba_attention(h, self.qt, self.kt, self.vt, self.row_ptr, self.col_idx, self.work_order,
                      self.ot, self.lse, sched, trace, self.workspace, stream)
        sba_unreorder(h, self.ot, o, self.workspace, stream)
        return o

    def stripe(self, q, k, v, params, o=None, sched: int = SBA_SCHED_LPT, trace=None,
               stream=None):
        """The same path with a stripe mask (one (Tw, To, Ts, Sw, So, Ss) per
        head, or one for all heads) in place of Top-p routing."""
        import torch
        p = self.plan
        h = p.handle
        if o is None:
            o = torch.empty_like(q)
        params = list(params) if len(params) == p.H else [tuple(params[0])] * p.H
        sba_reorder(h, q, k, v, self.qt, self.kt, self.vt, self.workspace, stream)
        sba_build_stripe_mask(h, params, self.bitmask, self.row_cnt, self.row_ptr, self.col_idx,
                              self.work_order, self.workspace, stream)
        sba_attention(h, self.qt, self.kt, self.vt, self.row_ptr, self.col_idx, self.work_order,
                      self.ot, self.lse, sched, trace, self.workspace, stream)
        sba_unreorder(h, self.ot, o, self.workspace, stream)
        return o

    def lowbit(self, q, k, v, top_p, top_k: int, o=None, trace=None, stream=None):
        """The same path with the low-bit P.V product: values smoothed and
        quantised by sba_smooth_v, attention by sba_attention_lowbit."""
        import torch
        p = self.plan
        h = p.handle
        inf = p.info
        dev = self.qt.device
        if not hasattr(self, "vq"):
            self.vq = torch.empty(p.B, p.H, inf.nb, p.d, inf.bs, dtype=torch.uint8, device=dev)
            self.vmean = torch.empty(p.B, p.H, inf.nb, p.d, dtype=torch.float32, device=dev)
            self.vexp = torch.empty(p.B, p.H, dtype=torch.int32, device=dev)
        if o is None:
            o = torch.empty_like(q)
        top_p = list(top_p) if len(top_p) == p.H else [float(top_p[0])] * p.H
        sba_reorder(h, q, k, v, self.qt, self.kt, self.vt, self.workspace, stream)
        sba_build_mask(h, self.qt, self.kt, top_p, top_k, self.bitmask, self.row_cnt,
                       self.row_ptr, self.col_idx, self.work_order, self.workspace, stream)
        sba_smooth_v(h, self.vt, self.vq, self.vmean, self.vexp, self.workspace, stream)
        sba_attention_lowbit(h, self.qt, self.kt, self.vq, self.vmean, self.vexp, self.row_ptr,
                             self.col_idx, self.work_order, self.ot, self.lse, trace,
                             self.workspace, stream)
        sba_unreorder(h, self.ot, o, self.workspace, stream)
        return o

    def check(self, stream=None) -> int:
        return sba_check_device_status(self.plan.handle, self.workspace, stream)
