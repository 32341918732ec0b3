"""Routed mixture-of-experts layer for NVIDIA B200 (sm_100a).

A thin ctypes binding of the C ABI in ``include/moe.h`` (``libmoe_b200.so``,
built in-tree by ``mixture_experts_layer_31_b200.build``).  The functions below
carry the ABI's names and only marshal arguments; every step of the layer runs
in the library's CUDA kernels.  ``MoELayer`` is a convenience wrapper that keeps
device tensors (PyTorch is used for device memory and streams only).

There is no CPU fallback: the first call into the library raises ImportError
when ``libmoe_b200.so`` is not built, and calls on a machine without a CUDA
device fail with MOE_ERR_CUDA.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

# enums (mirror include/moe.h)
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = 0, 1, 2, 3, 4
MOE_ROUTER_SIGMOID_BIAS, MOE_ROUTER_SOFTMAX = 0, 1
MOE_W_F32, MOE_W_BF16, MOE_W_INT8_ROW, MOE_W_INT4_B32, MOE_W_INT4_B128 = 0, 1, 2, 3, 4
MOE_X_F32, MOE_X_BF16 = 0, 1
MOE_ACT_SILU, MOE_ACT_GELU_TANH = 0, 1
MOE_PATH_AUTO, MOE_PATH_GEMV, MOE_PATH_GEMM = 0, 1, 2
MOE_FLAG_BAD_EXPERT_INDEX, MOE_FLAG_TOO_FEW_ACTIVE, MOE_FLAG_NONFINITE_LOGIT = 1, 2, 4

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA"}
WFMT = {"f32": MOE_W_F32, "bf16": MOE_W_BF16, "int8": MOE_W_INT8_ROW, "int4": MOE_W_INT4_B32,
        "int4b128": MOE_W_INT4_B128}
ACT = {"silu": MOE_ACT_SILU, "gelu_tanh": MOE_ACT_GELU_TANH}
XFMT = {"f32": MOE_X_F32, "bf16": MOE_X_BF16}
ROUTER = {"sigmoid": MOE_ROUTER_SIGMOID_BIAS, "softmax": MOE_ROUTER_SOFTMAX}

EXPORTS = ("moe_workspace_size", "moe_route", "moe_route_logits", "moe_forward", "moe_layer_forward", "moe_forward_noalloc",
           "moe_block_workspace_size",
           "moe_forward_block", "moe_expert_counts",
           "moe_cover_set", "moe_selftest_bounded_wait", "moe_last_error", "moe_device_flags", "moe_launch_count",
           "moe_stage_timing", "moe_stage_times", "moe_stage_timing_only")


def _header_scratch_bytes() -> int:
    """MOE_NOALLOC_SCRATCH_BYTES as include/moe.h defines it (the one definition;
    the library is compiled from the same header)."""
    import re
    hdr = os.path.join(os.path.dirname(_HERE), "include", "moe.h")
    with open(hdr) as f:
        m = re.search(r"#define\s+MOE_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    if m is None:
        raise ImportError("MOE_NOALLOC_SCRATCH_BYTES not found in %s" % hdr)
    return int(m.group(1)) << int(m.group(2))


MOE_NOALLOC_SCRATCH_BYTES = _header_scratch_bytes()


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, str(status)), message))
        self.status = status


class moe_desc(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("router", ctypes.c_int32), ("act", ctypes.c_int32), ("wfmt", ctypes.c_int32),
        ("xfmt", ctypes.c_int32), ("path", ctypes.c_int32), ("scale", ctypes.c_float),
        ("W_r", ctypes.c_void_p), ("b", ctypes.c_void_p), ("expert_mask", ctypes.c_void_p),
        ("W_gate", ctypes.c_void_p), ("W_up", ctypes.c_void_p), ("W_down", ctypes.c_void_p),
        ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
    ]


class moe_shared_expert(ctypes.Structure):
    _fields_ = [("I", ctypes.c_int32), ("wfmt", ctypes.c_int32), ("W_gate", ctypes.c_void_p),
                ("W_up", ctypes.c_void_p), ("W_down", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
                ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p)]


class moe_stage_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_float)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmoe_b200.so is not built; run `python -m mixture_experts_layer_31_b200.build` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(moe_desc)
    lib.moe_workspace_size.argtypes = [D, i32, ctypes.POINTER(sz)]
    lib.moe_route.argtypes = [D, vp, i32, vp, vp, vp, sz, vp]
    lib.moe_forward.argtypes = [D, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.moe_route_logits.argtypes = [D, vp, i32, vp, vp, sz, vp]
    lib.moe_forward_noalloc.argtypes = [D, vp, i32, vp, vp, vp, vp]
    lib.moe_layer_forward.argtypes = [D, vp, i32, vp, vp, vp, vp, sz, vp]
    SH = ctypes.POINTER(moe_shared_expert)
    lib.moe_block_workspace_size.argtypes = [D, SH, i32, ctypes.POINTER(sz)]
    lib.moe_forward_block.argtypes = [D, SH, vp, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_expert_counts.argtypes = [D, vp, i32, vp, vp]
    lib.moe_cover_set.argtypes = [vp, i32, ctypes.c_double, vp, vp, ctypes.POINTER(i32)]
    lib.moe_selftest_bounded_wait.argtypes = [vp]
    lib.moe_selftest_bounded_wait.restype = ctypes.c_int
    lib.moe_last_error.argtypes = []
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_device_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    lib.moe_launch_count.argtypes = []
    lib.moe_launch_count.restype = ctypes.c_uint64
    lib.moe_stage_timing.argtypes = [i32]
    lib.moe_stage_times.argtypes = [ctypes.POINTER(moe_stage_time), i32, ctypes.POINTER(i32)]
    lib.moe_stage_timing_only.argtypes = [ctypes.c_char_p]
    for f in ("moe_workspace_size", "moe_route", "moe_route_logits", "moe_forward", "moe_layer_forward", "moe_forward_noalloc",
              "moe_block_workspace_size",
              "moe_forward_block", "moe_expert_counts",
              "moe_cover_set", "moe_device_flags", "moe_stage_timing", "moe_stage_times", "moe_stage_timing_only"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (loaded on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error().decode())


# ---------------------------------------------------------------- ABI functions

def moe_workspace_size(desc: moe_desc, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(desc), int(T), ctypes.byref(n)))
    return n.value


def moe_route(desc: moe_desc, x: int, T: int, topk_idx: int, topk_w: int, workspace: int, ws_bytes: int,
              stream: int = 0) -> None:
    _check(lib().moe_route(ctypes.byref(desc), x, int(T), topk_idx, topk_w, workspace, int(ws_bytes), stream))


def moe_route_logits(desc: moe_desc, x: int, T: int, logits: int, workspace: int, ws_bytes: int,
                     stream: int = 0) -> None:
    """logits [T, E] fp32: the router logits exactly as moe_route ranks them."""
    _check(lib().moe_route_logits(ctypes.byref(desc), x, int(T), logits, workspace, int(ws_bytes), stream))


def moe_forward(desc: moe_desc, x: int, T: int, topk_idx: int, topk_w: int, y: int, workspace: int,
                ws_bytes: int, stream: int = 0) -> None:
    _check(lib().moe_forward(ctypes.byref(desc), x, int(T), topk_idx, topk_w, y, workspace, int(ws_bytes), stream))


def moe_layer_forward(desc: moe_desc, x: int, T: int, topk_idx: int, topk_w: int, y: int, workspace: int,
                      ws_bytes: int, stream: int = 0) -> None:
    """moe_route + moe_forward in one call (topk_idx / topk_w are written)."""
    _check(lib().moe_layer_forward(ctypes.byref(desc), x, int(T), topk_idx, topk_w, y, workspace, int(ws_bytes),
                                   stream))


def moe_forward_noalloc(desc: moe_desc, x: int, T: int, topk_idx: int, topk_w: int, y: int,
                        stream: int = 0) -> None:
    """moe_forward with the library's static scratch instead of a workspace, for
    callers that cannot allocate device memory (see include/moe.h)."""
    _check(lib().moe_forward_noalloc(ctypes.byref(desc), x, int(T), topk_idx, topk_w, y, stream))


def moe_block_workspace_size(desc: moe_desc, shared: Optional["moe_shared_expert"], T: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_block_workspace_size(ctypes.byref(desc), ctypes.byref(shared) if shared else None, int(T),
                                          ctypes.byref(n)))
    return n.value


def moe_forward_block(desc: moe_desc, shared: Optional["moe_shared_expert"], x: int, T: int, topk_idx: int,
                      topk_w: int, residual: Optional[int], y: int, workspace: int, ws_bytes: int,
                      stream: int = 0) -> None:
    """y = routed experts + shared expert (if any) + residual (if any)."""
    _check(lib().moe_forward_block(ctypes.byref(desc), ctypes.byref(shared) if shared else None, x, int(T),
                                   topk_idx, topk_w, residual, y, workspace, int(ws_bytes), stream))


def moe_expert_counts(desc: moe_desc, topk_idx: int, T: int, counts: int, stream: int = 0) -> None:
    """counts[e] (device uint64 [E]) += entries of topk_idx [T, k] equal to e."""
    _check(lib().moe_expert_counts(ctypes.byref(desc), topk_idx, int(T), counts, stream))


def moe_cover_set(counts, cover: float):
    """Host utility: (keep [E] uint8, new_index [E] int32, n_keep) for the smallest
    expert set whose counts (host array [E]) reach cover * total."""
    import numpy as np
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    E = c.size
    keep = np.empty(E, np.uint8)
    new_index = np.empty(E, np.int32)
    n = ctypes.c_int32(0)
    _check(lib().moe_cover_set(c.ctypes.data, int(E), float(cover), keep.ctypes.data, new_index.ctypes.data,
                               ctypes.byref(n)))
    return keep, new_index, int(n.value)


def moe_selftest_bounded_wait(stream: int = 0) -> None:
    """Launch the bounded-wait self-test (raises MOE_FLAG_TIMEOUT on the device after ~2 s)."""
    _check(lib().moe_selftest_bounded_wait(stream))


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_device_flags(clear: bool = False) -> int:
    v = ctypes.c_uint32(0)
    _check(lib().moe_device_flags(ctypes.byref(v), 1 if clear else 0))
    return v.value


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


def moe_stage_timing(enable: bool) -> None:
    _check(lib().moe_stage_timing(1 if enable else 0))


def moe_stage_timing_only(name=None) -> None:
    """Time only the launches of kernel `name` (None: every launch again)."""
    _check(lib().moe_stage_timing_only(None if not name else name.encode()))


def moe_stage_times() -> dict:
    """{kernel name: (launches, total ms)} since the previous call."""
    cap = 64
    buf = (moe_stage_time * cap)()
    n = ctypes.c_int32(0)
    _check(lib().moe_stage_times(buf, cap, ctypes.byref(n)))
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n.value, cap))}


# ---------------------------------------------------------------- convenience wrapper

class MoELayer:
    """Device-resident layer: holds the weights as torch CUDA tensors, a reusable
    workspace, and calls moe_route / moe_forward on the current torch stream."""

    def __init__(self, *, H, I, E, k, router, scale, wfmt, xfmt, W_r, W_gate, W_up, W_down, b=None,
                 expert_mask=None, s_gate=None, s_up=None, s_down=None, path=MOE_PATH_AUTO, device="cuda",
                 act="silu", I_s=0, Ws_gate=None, Ws_up=None, Ws_down=None, ss_gate=None, ss_up=None,
                 ss_down=None):
        import torch
        lib()  # fail loudly now if the CUDA library is missing
        self.torch = torch
        self.device = torch.device(device)

        def dev(a):
            if a is None:
                return None
            if not isinstance(a, torch.Tensor):
                import numpy as np
                a = np.ascontiguousarray(a)
                if a.dtype == np.uint16:  # bf16 bit patterns
                    a = a.view(np.int16)
                a = torch.from_numpy(a)
            return a.contiguous().to(self.device)

        self.tensors = dict(W_r=dev(W_r), b=dev(b), expert_mask=dev(expert_mask), W_gate=dev(W_gate),
                            W_up=dev(W_up), W_down=dev(W_down), s_gate=dev(s_gate), s_up=dev(s_up),
                            s_down=dev(s_down))
        d = moe_desc()
        d.H, d.I, d.E, d.k = int(H), int(I), int(E), int(k)
        d.router = ROUTER[router] if isinstance(router, str) else int(router)
        d.act = ACT[act] if isinstance(act, str) else int(act)
        d.wfmt = WFMT[wfmt] if isinstance(wfmt, str) else int(wfmt)
        d.xfmt = XFMT[xfmt] if isinstance(xfmt, str) else int(xfmt)
        d.path = int(path)
        d.scale = float(scale)
        for name, t in self.tensors.items():
            setattr(d, name, None if t is None else t.data_ptr())
        self.desc = d
        self._ws = None
        self._ws_T = -1
        self.shared = None
        if I_s:
            self.shared_tensors = dict(W_gate=dev(Ws_gate), W_up=dev(Ws_up), W_down=dev(Ws_down),
                                       s_gate=dev(ss_gate), s_up=dev(ss_up), s_down=dev(ss_down))
            sh = moe_shared_expert()
            sh.I, sh.wfmt = int(I_s), d.wfmt
            for name, t in self.shared_tensors.items():
                setattr(sh, name, None if t is None else t.data_ptr())
            self.shared = sh
        self._bws = None
        self._bws_T = -1

    @property
    def x_dtype(self):
        return self.torch.bfloat16 if self.desc.xfmt == MOE_X_BF16 else self.torch.float32

    def workspace(self, T: int):
        if self._ws is None or self._ws_T < T:
            n = moe_workspace_size(self.desc, T)
            self._ws = self.torch.empty(max(n, 256), dtype=self.torch.uint8, device=self.device)
            self._ws_T = T
        return self._ws

    def _stream(self):
        return self.torch.cuda.current_stream(self.device).cuda_stream

    def route(self, x, out: Optional[Tuple] = None):
        T = x.shape[0]
        if out is None:
            idx = self.torch.empty((T, self.desc.k), dtype=self.torch.int32, device=self.device)
            w = self.torch.empty((T, self.desc.k), dtype=self.torch.float32, device=self.device)
        else:
            idx, w = out
        ws = self.workspace(T)
        moe_route(self.desc, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), ws.data_ptr(), ws.numel(), self._stream())
        return idx, w

    def route_logits(self, x, out=None):
        """The router logits [T, E] fp32 that route() ranks (moe_route_logits)."""
        T = x.shape[0]
        logits = out if out is not None else self.torch.empty((T, self.desc.E), dtype=self.torch.float32,
                                                                device=self.device)
        ws = self.workspace(T)
        moe_route_logits(self.desc, x.data_ptr(), T, logits.data_ptr(), ws.data_ptr(), ws.numel(), self._stream())
        return logits

    def forward(self, x, idx, w, y=None):
        T = x.shape[0]
        if y is None:
            y = self.torch.empty((T, self.desc.H), dtype=self.x_dtype, device=self.device)
        ws = self.workspace(T)
        moe_forward(self.desc, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), y.data_ptr(), ws.data_ptr(),
                    ws.numel(), self._stream())
        return y

    def __call__(self, x):
        idx, w = self.route(x)
        return self.forward(x, idx, w), idx, w

    def layer(self, x, out=None):
        """Route and forward in one call (moe_layer_forward): (y, idx, w)."""
        T = x.shape[0]
        if out is None:
            idx = self.torch.empty((T, self.desc.k), dtype=self.torch.int32, device=self.device)
            w = self.torch.empty((T, self.desc.k), dtype=self.torch.float32, device=self.device)
            y = self.torch.empty((T, self.desc.H), dtype=self.x_dtype, device=self.device)
        else:
            y, idx, w = out
        ws = self.workspace(T)
        moe_layer_forward(self.desc, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), y.data_ptr(), ws.data_ptr(),
                          ws.numel(), self._stream())
        return y, idx, w

    def block_workspace(self, T: int):
        if self._bws is None or self._bws_T != T:
            n = moe_block_workspace_size(self.desc, self.shared, T)
            self._bws = self.torch.empty(max(n, 256), dtype=self.torch.uint8, device=self.device)
            self._bws_T = T
        return self._bws

    def block(self, x, idx, w, residual=None, y=None):
        """The MoE block: routed experts + the shared expert (if the layer has one) +
        residual (if given, [T, H] in x's dtype; y may be residual itself)."""
        T = x.shape[0]
        if y is None:
            y = self.torch.empty((T, self.desc.H), dtype=self.x_dtype, device=self.device)
        ws = self.block_workspace(T)
        moe_forward_block(self.desc, self.shared, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(),
                          None if residual is None else residual.data_ptr(), y.data_ptr(), ws.data_ptr(),
                          ws.numel(), self._stream())
        return y

    def expert_counts(self, idx, counts=None):
        """Accumulate per-expert routing counts of idx [T, k] into counts (a device
        uint64 tensor [E], created zeroed when None) and return it."""
        if counts is None:
            counts = self.torch.zeros(self.desc.E, dtype=self.torch.uint64, device=self.device)
        moe_expert_counts(self.desc, idx.data_ptr(), idx.shape[0], counts.data_ptr(), self._stream())
        return counts
