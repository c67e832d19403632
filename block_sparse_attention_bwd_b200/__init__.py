"""Python binding of libspattn (exact block-sparse attention on B200).

Argument marshalling only: every step of the forward and backward passes
runs in the CUDA kernels of ``libspattn.so`` behind the C ABI declared in
``include/spattn.h``.  PyTorch supplies device memory and the current CUDA
stream.  There is no fallback: if the library is missing, importing this
package raises.

Names follow the C ABI: :class:`Plan` wraps ``spattn_plan``;
:func:`spattn_fwd`, :func:`spattn_bwd` and :func:`spattn_check` call the
entry points of the same names.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspattn.so")

SPATTN_OK = 0
SPATTN_ERR_INVALID_ARG, SPATTN_ERR_UNSUPPORTED, SPATTN_ERR_OOM, SPATTN_ERR_CUDA = 1, 2, 3, 4
SPATTN_ERR_TIMEOUT, SPATTN_ERR_DEVICE = 5, 6
STATUS_NAMES = {
    0: "SPATTN_OK",
    1: "SPATTN_ERR_INVALID_ARG",
    2: "SPATTN_ERR_UNSUPPORTED",
    3: "SPATTN_ERR_OOM",
    4: "SPATTN_ERR_CUDA",
    5: "SPATTN_ERR_TIMEOUT",
    6: "SPATTN_ERR_DEVICE",
}

ENTRY_POINTS = (
    "spattn_plan", "spattn_fwd", "spattn_bwd", "spattn_bwd_noalloc", "spattn_check", "spattn_plan_stats", "spattn_profile",
    "spattn_profile_read", "spattn_plan_pages", "spattn_plan_qblocks", "spattn_plan_work", "spattn_plan_destroy",
    "spattn_status_string", "spattn_wait_selftest", "spattn_plan_set_graph_device", "spattn_plan_entry_heads",
    "spattn_quantize_fp8", "spattn_fwd_fp8",
)


class SpattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_lib().spattn_status_string(status).decode()})")


class _Layout(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("q_slots", ctypes.c_int64), ("kv_slots", ctypes.c_int64),
        ("q_group", ctypes.POINTER(ctypes.c_int32)), ("kv_group", ctypes.POINTER(ctypes.c_int32)),
        ("n_q_groups", ctypes.c_int32), ("n_kv_groups", ctypes.c_int32), ("scale", ctypes.c_float),
        ("kv_heads", ctypes.c_int32), ("graph_batches", ctypes.c_int32),
    ]


class _Graph(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.POINTER(ctypes.c_int64)), ("kv_groups", ctypes.POINTER(ctypes.c_int32))]


class _Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "useful_pairs", "physical_pairs_fwd", "physical_pairs_dkdv", "physical_pairs_dq", "bsa_pairs",
        "n_work_fwd", "n_work_dkdv", "n_entries_fwd", "n_entries_dkdv", "device_bytes", "launches_fwd",
        "launches_bwd")] + [("plan_ms", ctypes.c_double)]


class _KernelTimes(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * 5), ("launches", ctypes.c_int64 * 5)]


KERNEL_NAMES = ("fwd", "fill", "delta", "dkdv", "dq")


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        I32, I64 = ctypes.c_int32, ctypes.c_int64
        lib.spattn_plan.argtypes = [ctypes.POINTER(_Layout), ctypes.POINTER(_Graph), ctypes.POINTER(P)]
        lib.spattn_fwd.argtypes = [P, P, P, P, P, P, P]
        lib.spattn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P]
        lib.spattn_quantize_fp8.argtypes = [P, I64, I64, ctypes.c_int, P, P, P]
        lib.spattn_fwd_fp8.argtypes = [P, P, P, P, P, P, P, P, P]
        lib.spattn_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, P]
        lib.spattn_check.argtypes = [P, P]
        lib.spattn_wait_selftest.argtypes = [P, I64, P]
        lib.spattn_plan_set_graph_device.argtypes = [P, P, P, I64, P]
        lib.spattn_plan_stats.argtypes = [P, ctypes.POINTER(_Stats)]
        lib.spattn_plan_pages.argtypes = [P, I32, I64, ctypes.POINTER(ctypes.POINTER(I32)), ctypes.POINTER(I64)]
        lib.spattn_plan_qblocks.argtypes = [P, I32, I64, ctypes.POINTER(ctypes.POINTER(I32)), ctypes.POINTER(I64)]
        lib.spattn_plan_work.argtypes = [P, I32, ctypes.POINTER(ctypes.POINTER(I32)), ctypes.POINTER(I64),
                                         ctypes.POINTER(ctypes.POINTER(I32)), ctypes.POINTER(ctypes.POINTER(ctypes.c_uint64)),
                                         ctypes.POINTER(I64)]
        lib.spattn_plan_entry_heads.argtypes = [P, I32, ctypes.POINTER(ctypes.POINTER(ctypes.c_uint16)),
                                                ctypes.POINTER(I64)]
        lib.spattn_profile.argtypes = [P, ctypes.c_int]
        lib.spattn_profile_read.argtypes = [P, ctypes.POINTER(_KernelTimes)]
        lib.spattn_plan_destroy.argtypes = [P]
        lib.spattn_plan_destroy.restype = None
        lib.spattn_status_string.argtypes = [ctypes.c_int]
        lib.spattn_status_string.restype = ctypes.c_char_p
        for name in ENTRY_POINTS:
            if name not in ("spattn_plan_destroy", "spattn_status_string"):
                getattr(lib, name).restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _check(status: int, where: str):
    if status != SPATTN_OK:
        raise SpattnError(status, where)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


class Plan:
    """Owning wrapper of ``spattn_plan_t``.

    ``q_group`` / ``kv_group``: int32 per slot (-1 = padded).  ``row_ptr`` /
    ``kv_groups``: CSR over (head, query group) of allowed key groups.
    The plan lives on the current CUDA device.
    """

    def __init__(self, q_group, kv_group, n_q_groups, n_kv_groups, row_ptr, kv_groups, *, batch, heads,
                 head_dim, scale=0.0, kv_heads=0, graph_batches=1):
        qg, kg = _i32(q_group), _i32(kv_group)
        rp = np.ascontiguousarray(row_ptr, dtype=np.int64)
        cols = _i32(kv_groups) if len(kv_groups) else np.zeros(1, np.int32)
        self._keep = (qg, kg, rp, cols)
        lay = _Layout(batch, heads, head_dim, qg.size, kg.size,
                      qg.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), kg.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                      int(n_q_groups), int(n_kv_groups), float(scale), int(kv_heads), int(graph_batches))
        gr = _Graph(rp.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), cols.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
        h = ctypes.c_void_p()
        _check(_lib().spattn_plan(ctypes.byref(lay), ctypes.byref(gr), ctypes.byref(h)), "spattn_plan")
        self.handle = h
        self.batch, self.heads, self.head_dim = batch, heads, head_dim
        self.kv_heads = heads if kv_heads == 0 else kv_heads
        self.q_slots, self.kv_slots = qg.size, kg.size
        self._keep = None

    @classmethod
    def from_problem(cls, problem, batch: Optional[int] = None):
        b = problem.batch if batch is None else batch
        gb = getattr(problem, "graph_batches", 1)
        if gb != 1 and b != problem.batch:
            raise ValueError("a problem with one graph per batch entry has a fixed batch")
        return cls(problem.q_group, problem.kv_group, problem.n_q_groups, problem.n_kv_groups, problem.row_ptr,
                   problem.kv_groups, batch=b, heads=problem.heads, head_dim=problem.head_dim, scale=problem.scale,
                   kv_heads=getattr(problem, "kv_heads", 0) or 0, graph_batches=gb)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _lib().spattn_plan_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_graph_device(self, row_ptr, kv_groups, stream=None):
        """Re-plan on the GPU for a new graph: ``row_ptr`` int64 and
        ``kv_groups`` int32, contiguous CUDA tensors in the spattn_graph
        format (spattn_plan_set_graph_device)."""
        import torch

        if row_ptr.dtype != torch.int64 or not row_ptr.is_cuda or not row_ptr.is_contiguous():
            raise ValueError("row_ptr: expected a contiguous CUDA int64 tensor")
        if kv_groups.dtype != torch.int32 or not kv_groups.is_cuda or not kv_groups.is_contiguous():
            raise ValueError("kv_groups: expected a contiguous CUDA int32 tensor")
        _check(_lib().spattn_plan_set_graph_device(self.handle, _ptr(row_ptr), _ptr(kv_groups), kv_groups.numel(),
                                                   _stream_handle(stream)), "spattn_plan_set_graph_device")

    def stats(self) -> dict:
        s = _Stats()
        _check(_lib().spattn_plan_stats(self.handle, ctypes.byref(s)), "spattn_plan_stats")
        return {n: getattr(s, n) for n, _ in _Stats._fields_}

    def profile(self, enable: bool):
        """Start / stop recording per-kernel CUDA events in fwd / bwd calls (clears the record)."""
        _check(_lib().spattn_profile(self.handle, 1 if enable else 0), "spattn_profile")

    def profile_read(self) -> dict:
        """{kernel: (summed ms, launches)} of the recorded launches; clears the record."""
        t = _KernelTimes()
        _check(_lib().spattn_profile_read(self.handle, ctypes.byref(t)), "spattn_profile_read")
        return {n: (t.ms[i], t.launches[i]) for i, n in enumerate(KERNEL_NAMES)}

    def pages(self, head: int, qblock: int) -> np.ndarray:
        ptr = ctypes.POINTER(ctypes.c_int32)()
        n = ctypes.c_int64()
        _check(_lib().spattn_plan_pages(self.handle, head, qblock, ctypes.byref(ptr), ctypes.byref(n)), "spattn_plan_pages")
        return np.ctypeslib.as_array(ptr, shape=(n.value,)).copy() if n.value else np.zeros(0, np.int32)

    def qblocks(self, head: int, page: int) -> np.ndarray:
        ptr = ctypes.POINTER(ctypes.c_int32)()
        n = ctypes.c_int64()
        _check(_lib().spattn_plan_qblocks(self.handle, head, page, ctypes.byref(ptr), ctypes.byref(n)), "spattn_plan_qblocks")
        return np.ctypeslib.as_array(ptr, shape=(n.value,)).copy() if n.value else np.zeros(0, np.int32)

    def entry_heads(self, which: int) -> np.ndarray:
        """Per entry of work list ``which``: its query head relative to the item's K/V head group."""
        return _entry_heads(self, which)

    def work(self, which: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """(work [n, 32] int32, pages [e] int32, masks [e, 2] uint64) of pass ``which`` (0 query-owned, 1
        key-owned); segment s of entry e is bits 16 (s % 4) of masks[e, s // 4]."""
        w = ctypes.POINTER(ctypes.c_int32)()
        p = ctypes.POINTER(ctypes.c_int32)()
        m = ctypes.POINTER(ctypes.c_uint64)()
        nw, ne = ctypes.c_int64(), ctypes.c_int64()
        _check(_lib().spattn_plan_work(self.handle, which, ctypes.byref(w), ctypes.byref(nw), ctypes.byref(p),
                                       ctypes.byref(m), ctypes.byref(ne)), "spattn_plan_work")
        work = np.ctypeslib.as_array(w, shape=(nw.value * 32,)).reshape(-1, 32).copy() if nw.value else np.zeros((0, 32), np.int32)
        pages = np.ctypeslib.as_array(p, shape=(ne.value,)).copy() if ne.value else np.zeros(0, np.int32)
        masks = (np.ctypeslib.as_array(m, shape=(2 * ne.value,)).reshape(-1, 2).copy() if ne.value
                 else np.zeros((0, 2), np.uint64))
        return work, pages, masks


def _entry_heads(plan, which):
    h = ctypes.POINTER(ctypes.c_uint16)()
    n = ctypes.c_int64()
    _check(_lib().spattn_plan_entry_heads(plan.handle, which, ctypes.byref(h), ctypes.byref(n)),
           "spattn_plan_entry_heads")
    return np.ctypeslib.as_array(h, shape=(n.value,)).copy() if n.value else np.zeros(0, np.uint16)


def _stream_handle(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _need(t, name, shape, dtype):
    import torch

    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) \
            or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of shape {tuple(shape)}")


def spattn_fwd(q, k, v, plan: Plan, o=None, lse=None, stream=None):
    """O [B,H,Sq,D] bf16 and LSE [B,H,Sq] fp32 for the plan's sparse graph."""
    import torch

    qs = (plan.batch, plan.heads, plan.q_slots, plan.head_dim)
    ks = (plan.batch, plan.kv_heads, plan.kv_slots, plan.head_dim)
    _need(q, "q", qs, torch.bfloat16)
    _need(k, "k", ks, torch.bfloat16)
    _need(v, "v", ks, torch.bfloat16)
    if o is None:
        o = torch.empty(qs, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(qs[:3], dtype=torch.float32, device=q.device)
    _need(o, "o", qs, torch.bfloat16)
    _need(lse, "lse", qs[:3], torch.float32)
    _check(_lib().spattn_fwd(_ptr(q), _ptr(k), _ptr(v), plan.handle, _ptr(o), _ptr(lse), _stream_handle(stream)),
           "spattn_fwd")
    return o, lse


def quantize_fp8(x, stream=None):
    """E4M3 codes (uint8, same shape) and per-(batch, head) descale factors
    (float32 [B, H]) of a bf16 tensor [B, H, S, D], one slice per (batch, head)."""
    import torch

    if x.dim() != 4 or x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("quantize_fp8: x must be a contiguous CUDA bf16 tensor [B, H, S, D]")
    B, H, S, D = x.shape
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    descale = torch.empty((B, H), dtype=torch.float32, device=x.device)
    _check(_lib().spattn_quantize_fp8(_ptr(x), B * H, S, D, _ptr(x8), _ptr(descale), _stream_handle(stream)),
           "spattn_quantize_fp8")
    return x8, descale


def spattn_fwd_fp8(q8, k8, q_descale, k_descale, v, plan: Plan, o=None, lse=None, stream=None):
    """O and LSE of attention over the dequantised E4M3 Q and K (see quantize_fp8)."""
    import torch

    qs = (plan.batch, plan.heads, plan.q_slots, plan.head_dim)
    ks = (plan.batch, plan.kv_heads, plan.kv_slots, plan.head_dim)
    _need(q8, "q8", qs, torch.uint8)
    _need(k8, "k8", ks, torch.uint8)
    _need(v, "v", ks, torch.bfloat16)
    _need(q_descale, "q_descale", qs[:2], torch.float32)
    _need(k_descale, "k_descale", ks[:2], torch.float32)
    if o is None:
        o = torch.empty(qs, dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty(qs[:3], dtype=torch.float32, device=q8.device)
    _need(o, "o", qs, torch.bfloat16)
    _need(lse, "lse", qs[:3], torch.float32)
    _check(_lib().spattn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(q_descale), _ptr(k_descale), _ptr(v), plan.handle, _ptr(o),
                                 _ptr(lse), _stream_handle(stream)), "spattn_fwd_fp8")
    return o, lse


def spattn_bwd(q, k, v, o, lse, do, plan: Plan, dq=None, dk=None, dv=None, stream=None):
    """dQ, dK, dV (bf16) given the forward's O and LSE and the loss gradient dO."""
    import torch

    qs = (plan.batch, plan.heads, plan.q_slots, plan.head_dim)
    ks = (plan.batch, plan.kv_heads, plan.kv_slots, plan.head_dim)
    for t, nm, sh in ((q, "q", qs), (k, "k", ks), (v, "v", ks), (o, "o", qs), (do, "do", qs)):
        _need(t, nm, sh, torch.bfloat16)
    _need(lse, "lse", qs[:3], torch.float32)
    dq = torch.empty(qs, dtype=torch.bfloat16, device=q.device) if dq is None else dq
    dk = torch.empty(ks, dtype=torch.bfloat16, device=q.device) if dk is None else dk
    dv = torch.empty(ks, dtype=torch.bfloat16, device=q.device) if dv is None else dv
    _need(dq, "dq", qs, torch.bfloat16)
    _need(dk, "dk", ks, torch.bfloat16)
    _need(dv, "dv", ks, torch.bfloat16)
    _check(_lib().spattn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), plan.handle, _ptr(dq), _ptr(dk),
                             _ptr(dv), _stream_handle(stream)), "spattn_bwd")
    return dq, dk, dv


def spattn_check(plan: Plan, stream=None):
    """Synchronise the stream and raise if a kernel recorded a device-side error."""
    _check(_lib().spattn_check(plan.handle, _stream_handle(stream)), "spattn_check")


def spattn_wait_selftest(plan: Plan, deadline_cycles: int, stream=None) -> int:
    """Run the bounded-wait failure self-test; returns the following spattn_check status."""
    _check(_lib().spattn_wait_selftest(plan.handle, int(deadline_cycles), _stream_handle(stream)),
           "spattn_wait_selftest")
    return _lib().spattn_check(plan.handle, _stream_handle(stream))


def load_library():
    """Load libspattn.so (raises ImportError when it has not been built)."""
    return _lib()
