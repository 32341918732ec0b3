"""fp64 CPU oracle for the routed mixture-of-experts layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``mixture_experts_layer_31_b200`` never does: it has no CPU path.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, index-order sums,
``-ffp-contract=off``); this module compiles it and marshals numpy arrays.  The
C functions are single-threaded and obviously sequential; the Python wrappers
split tokens over threads (ctypes releases the GIL during the call), which does
not change any result because tokens are independent.

Routing follows the Kimi-Linear LiteRT-LM details page (Conversion notes,
mixture-of-experts bullet) and the Qwen3-30B-A3B LiteRT-LM card (Conversion
Notes); the expert FFN and combine follow the same passages.  See the header of
``moe_oracle.c`` for the step-by-step citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

GATE, UP, DOWN = 0, 1, 2
_WFMT = {"f32": 0, "bf16": 1, "int8": 2, "int4": 3, "int4b128": 4}
_ACT = {"silu": 0, "gelu_tanh": 1}
_XFMT = {"f32": 0, "bf16": 1}
_ROUTER = {"sigmoid": 0, "softmax": 1}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("router", ctypes.c_int32), ("wfmt", ctypes.c_int32), ("xfmt", ctypes.c_int32),
        ("act", ctypes.c_int32), ("scale", ctypes.c_double),
        ("W_r", ctypes.c_void_p), ("b", ctypes.c_void_p), ("mask", ctypes.c_void_p),
        ("W_gate", ctypes.c_void_p), ("W_up", ctypes.c_void_p), ("W_down", ctypes.c_void_p),
        ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, vp, i64, i32 = ctypes.POINTER(_Layer), ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_weight.argtypes = [P, i32, i64, i64, i64]
        lib.oracle_weight.restype = ctypes.c_double
        lib.oracle_router_logits.argtypes = [P, vp, i64, i64, vp]
        lib.oracle_keys.argtypes = [P, vp, vp]
        lib.oracle_select.argtypes = [P, vp, vp, vp, vp]
        lib.oracle_route.argtypes = [P, vp, i64, i64, vp, vp, vp]
        lib.oracle_expert.argtypes = [P, i64, vp, vp]
        lib.oracle_combine.argtypes = [P, vp, i64, i64, vp, vp, vp]
        lib.oracle_forward.argtypes = [P, vp, i64, i64, vp, vp, vp, vp]
        lib.oracle_block.argtypes = [P, P, vp, vp, i64, i64, vp, vp, vp]
        lib.oracle_expert_counts.argtypes = [vp, i64, ctypes.c_int32, vp]
        lib.oracle_cover_set.argtypes = [vp, ctypes.c_int32, ctypes.c_double, vp, vp, vp]
        for f in ("oracle_router_logits", "oracle_keys", "oracle_select", "oracle_route",
                  "oracle_expert", "oracle_combine", "oracle_forward", "oracle_block", "oracle_expert_counts",
                  "oracle_cover_set"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]) -> Optional[int]:
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


class Oracle:
    """Binds one synthetic Problem (see ``synth.Problem``) to the C oracle."""

    def __init__(self, prob, nthreads: Optional[int] = None):
        self.prob = prob
        self.nthreads = int(nthreads) if nthreads else max(1, os.cpu_count() or 1)
        self._keep = [prob.x, prob.W_r, prob.b, prob.mask, prob.W_gate, prob.W_up, prob.W_down,
                      prob.s_gate, prob.s_up, prob.s_down]
        L = _Layer()
        L.H, L.I, L.E, L.k = prob.H, prob.I, prob.E, prob.k
        L.router, L.wfmt, L.xfmt = _ROUTER[prob.router], _WFMT[prob.wfmt], _XFMT[prob.xfmt]
        L.act = _ACT[getattr(prob, "act", "silu")]
        L.scale = float(prob.scale)
        L.W_r, L.b, L.mask = _p(prob.W_r), _p(prob.b), _p(prob.mask)
        L.W_gate, L.W_up, L.W_down = _p(prob.W_gate), _p(prob.W_up), _p(prob.W_down)
        L.s_gate, L.s_up, L.s_down = _p(prob.s_gate), _p(prob.s_up), _p(prob.s_down)
        self.L = L
        self.S = None  # the shared expert as a one-expert layer, when the problem has one
        if getattr(prob, "I_s", 0):
            self._keep += [prob.Ws_gate, prob.Ws_up, prob.Ws_down, prob.ss_gate, prob.ss_up, prob.ss_down]
            S = _Layer()
            S.H, S.I, S.E, S.k = prob.H, prob.I_s, 1, 1
            S.router, S.wfmt, S.xfmt, S.act = L.router, L.wfmt, L.xfmt, L.act
            S.scale = 1.0
            S.W_gate, S.W_up, S.W_down = _p(prob.Ws_gate), _p(prob.Ws_up), _p(prob.Ws_down)
            S.s_gate, S.s_up, S.s_down = _p(prob.ss_gate), _p(prob.ss_up), _p(prob.ss_down)
            self.S = S
        self.lib = _load()

    # -- helpers --------------------------------------------------------------
    def _split(self, tokens: Sequence[int]):
        n = len(tokens)
        nt = max(1, min(self.nthreads, n))
        return [tokens[n * i // nt: n * (i + 1) // nt] for i in range(nt)]

    def _x(self):
        return _p(self.prob.x)

    # -- single pieces ----------------------------------------------------------
    def weight(self, which: int, e: int, row: int, col: int) -> float:
        return self.lib.oracle_weight(ctypes.byref(self.L), which, e, row, col)

    def logits(self, tokens: Sequence[int]) -> np.ndarray:
        tokens = list(tokens)
        out = np.empty((len(tokens), self.prob.E), np.float64)
        pos = {t: i for i, t in enumerate(tokens)}

        def run_part(part):
            for t in part:
                rc = self.lib.oracle_router_logits(ctypes.byref(self.L), self._x(), t, t + 1,
                                                   out[pos[t]:].ctypes.data)
                assert rc == 0
            return 0

        with ThreadPoolExecutor(self.nthreads) as ex:
            list(ex.map(run_part, self._split(tokens)))
        return out

    def keys(self, logits_row: np.ndarray) -> np.ndarray:
        lr = np.ascontiguousarray(logits_row, np.float64)
        k = np.empty(self.prob.E, np.float64)
        assert self.lib.oracle_keys(ctypes.byref(self.L), _p(lr), _p(k)) == 0
        return k

    def select(self, logits_row: np.ndarray):
        lr = np.ascontiguousarray(logits_row, np.float64)
        idx = np.empty(self.prob.k, np.int32)
        w = np.empty(self.prob.k, np.float64)
        m = np.empty(1, np.float64)
        rc = self.lib.oracle_select(ctypes.byref(self.L), _p(lr), _p(idx), _p(w), _p(m))
        if rc != 0:
            raise ValueError("oracle_select rejected the problem (k > active experts?)")
        return idx, w, float(m[0])

    def expert(self, e: int, xt: np.ndarray) -> np.ndarray:
        xt = np.ascontiguousarray(xt, np.float64)
        o = np.empty(self.prob.H, np.float64)
        assert self.lib.oracle_expert(ctypes.byref(self.L), e, _p(xt), _p(o)) == 0
        return o

    # -- whole layer --------------------------------------------------------------
    def route(self, tokens: Optional[Sequence[int]] = None):
        """(idx [n,k] int32, w [n,k] f64, margin [n] f64) for the given tokens (default: all)."""
        tokens = list(range(self.prob.T)) if tokens is None else [int(t) for t in tokens]
        n, k = len(tokens), self.prob.k
        idx = np.empty((n, k), np.int32)
        w = np.empty((n, k), np.float64)
        margin = np.empty(n, np.float64)
        pos = {t: i for i, t in enumerate(tokens)}

        def run_part(part):
            for t in part:
                i = pos[t]
                rc = self.lib.oracle_route(ctypes.byref(self.L), self._x(), t, t + 1,
                                           idx[i:].ctypes.data, w[i:].ctypes.data, margin[i:].ctypes.data)
                if rc != 0:
                    raise ValueError("oracle_route rejected the problem")
            return 0

        with ThreadPoolExecutor(self.nthreads) as ex:
            list(ex.map(run_part, self._split(tokens)))
        return idx, w, margin

    def combine(self, tokens: Sequence[int], idx: np.ndarray, w: np.ndarray) -> np.ndarray:
        """y [n,H] fp64 for the given tokens under a given routing (idx/w rows follow `tokens`)."""
        tokens = [int(t) for t in tokens]
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        y = np.empty((len(tokens), self.prob.H), np.float64)
        pos = {t: i for i, t in enumerate(tokens)}

        def run_part(part):
            for t in part:
                i = pos[t]
                rc = self.lib.oracle_combine(ctypes.byref(self.L), self._x(), t, t + 1,
                                             idx[i:].ctypes.data, w[i:].ctypes.data, y[i:].ctypes.data)
                assert rc == 0
            return 0

        with ThreadPoolExecutor(self.nthreads) as ex:
            list(ex.map(run_part, self._split(tokens)))
        return y

    def block(self, tokens: Sequence[int], idx: np.ndarray, w: np.ndarray) -> np.ndarray:
        """The MoE block y [n,H] fp64 under a given routing: routed sum + shared expert
        (if the problem has one) + residual (if it has one)."""
        tokens = [int(t) for t in tokens]
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        y = np.empty((len(tokens), self.prob.H), np.float64)
        pos = {t: i for i, t in enumerate(tokens)}
        Sp = ctypes.byref(self.S) if self.S is not None else None
        res = _p(getattr(self.prob, "residual", None))

        def run_part(part):
            for t in part:
                i = pos[t]
                rc = self.lib.oracle_block(ctypes.byref(self.L), Sp, self._x(), res, t, t + 1,
                                           idx[i:].ctypes.data, w[i:].ctypes.data, y[i:].ctypes.data)
                assert rc == 0
            return 0

        with ThreadPoolExecutor(self.nthreads) as ex:
            list(ex.map(run_part, self._split(tokens)))
        return y

    def forward(self, tokens: Optional[Sequence[int]] = None):
        """(y [n,H] f64, idx, w, margin) for the given tokens (default: all)."""
        tokens = list(range(self.prob.T)) if tokens is None else [int(t) for t in tokens]
        idx, w, margin = self.route(tokens)
        return self.combine(tokens, idx, w), idx, w, margin


# -- routing statistics (CMF code specialist page, How it was made: Calibrate and Defrag) --

def expert_counts(idx: np.ndarray, E: int, counts: Optional[np.ndarray] = None) -> np.ndarray:
    """counts[e] += number of routing entries equal to e (entries outside [0, E) skipped)."""
    idx = np.ascontiguousarray(idx, np.int32)
    counts = np.zeros(E, np.uint64) if counts is None else counts
    assert counts.dtype == np.uint64 and counts.flags["C_CONTIGUOUS"] and counts.size == E
    assert _load().oracle_expert_counts(_p(idx), idx.size, int(E), _p(counts)) == 0
    return counts


def cover_set(counts: np.ndarray, cover: float):
    """(keep [E] uint8, new_index [E] int32, n_keep): the smallest expert set whose
    counts reach cover * total, renumbered into a dense prefix."""
    counts = np.ascontiguousarray(counts, np.uint64)
    E = counts.size
    keep = np.empty(E, np.uint8)
    new_index = np.empty(E, np.int32)
    n = np.empty(1, np.int32)
    rc = _load().oracle_cover_set(_p(counts), int(E), float(cover), _p(keep), _p(new_index), _p(n))
    if rc != 0:
        raise ValueError("oracle_cover_set rejected its arguments")
    return keep, new_index, int(n[0])
