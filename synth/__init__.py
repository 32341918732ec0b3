"""Seeded synthetic inputs for the routed mixture-of-experts layer.

This package only *makes inputs*: activations, router weights and bias, the
expert mask, and expert weights in the stored formats the layer reads (fp32,
bf16, int8 per output row, int4 block-32).  It contains none of the layer's
arithmetic, so the fp64 oracle (``oracle/``) and the CUDA library both consume
its arrays without sharing method code.  The random streams and storage
encoders are implemented in ``synth.c`` (counter-based SplitMix64, Box-Muller,
round-to-nearest-even bf16, the two weight encoders).

The workloads follow the shapes and distributions the pages describe:

* Kimi-Linear-48B-A3B routed layer: 256 routed experts, 8 chosen per token,
  sigmoid scores with a selection bias, weights renormalised and scaled by
  2.446, expert intermediate dim 2048 (LiteRT-LM details page, Conversion
  notes, mixture-of-experts bullet; APEX GGUF card, Method).
* Qwen3-30B-A3B routed layer: 128 experts, 8 used per token, softmax router,
  top-8 renormalised (Qwen3 LiteRT-LM card, intro and Conversion Notes).
* Skewed routing with an expert mask: the top 64 of 256 experts carry 73% of
  the routing mass; about 160 of 256 experts kept (CMF code specialist page,
  Calibrate and Defrag steps).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

# stream ids: one independent random stream per tensor
S_X, S_WR, S_B, S_WG, S_WU, S_WD, S_MASK, S_RANK = 1, 2, 3, 4, 5, 6, 7, 8
S_SG, S_SU, S_SD, S_RES = 9, 10, 11, 12  # shared expert gate/up/down, residual stream

WFMT = {"f32": 0, "bf16": 1, "int8": 2, "int4": 3, "int4b128": 4}
ACT = {"silu": 0, "gelu_tanh": 1}
INT4_BLOCK = {"int4": 32, "int4b128": 128}
XFMT = {"f32": 0, "bf16": 1}
ROUTER = {"sigmoid": 0, "softmax": 1}


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, IEEE fp, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-pthread",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        sz, u64, dbl, i32 = ctypes.c_size_t, ctypes.c_uint64, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        for name, args in {
            "synth_normal_f32": [vp, sz, u64, u64, dbl, dbl, i32],
            "synth_normal_bf16": [vp, sz, u64, u64, dbl, dbl, i32],
            "synth_uniform_f32": [vp, sz, u64, u64, dbl, dbl, i32],
            "synth_uniform_f64": [vp, sz, u64, u64, dbl, dbl],
            "synth_int8_rows": [vp, vp, sz, sz, u64, u64, dbl, i32],
            "synth_int4_blocks": [vp, vp, sz, sz, u64, u64, dbl, i32],
            "synth_int4_blocks_b": [vp, vp, sz, sz, sz, u64, u64, dbl, i32],
        }.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.synth_draw_u64.argtypes = [u64, u64, u64]
        lib.synth_draw_u64.restype = u64
        _lib = lib
    return _lib


def _threads(n: Optional[int]) -> int:
    return int(n) if n else max(1, os.cpu_count() or 1)


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_f32(shape, seed, stream, mean=0.0, std=1.0, nthreads=None) -> np.ndarray:
    a = np.empty(shape, np.float32)
    assert _load().synth_normal_f32(_ptr(a), a.size, seed, stream, mean, std, _threads(nthreads)) == 0
    return a


def normal_bf16(shape, seed, stream, mean=0.0, std=1.0, nthreads=None) -> np.ndarray:
    """bf16 values as uint16 bit patterns (N(mean, std) in fp32, then round-to-nearest-even)."""
    a = np.empty(shape, np.uint16)
    assert _load().synth_normal_bf16(_ptr(a), a.size, seed, stream, mean, std, _threads(nthreads)) == 0
    return a


def uniform_f32(shape, seed, stream, lo, hi, nthreads=None) -> np.ndarray:
    a = np.empty(shape, np.float32)
    assert _load().synth_uniform_f32(_ptr(a), a.size, seed, stream, lo, hi, _threads(nthreads)) == 0
    return a


def uniform_f64(n, seed, stream, lo=0.0, hi=1.0) -> np.ndarray:
    a = np.empty(n, np.float64)
    assert _load().synth_uniform_f64(_ptr(a), a.size, seed, stream, lo, hi) == 0
    return a


def int8_rows(rows, cols, seed, stream, std, nthreads=None):
    """N(0, std) matrix [rows, cols] stored int8 with one fp32 scale per row."""
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    assert _load().synth_int8_rows(_ptr(q), _ptr(s), rows, cols, seed, stream, std, _threads(nthreads)) == 0
    return q, s


def int4_blocks(rows, cols, seed, stream, std, nthreads=None, block=32):
    """N(0, std) matrix [rows, cols] stored as int4 nibbles [rows, cols/2] + scales [rows, cols/block]."""
    q = np.empty((rows, cols // 2), np.uint8)
    s = np.empty((rows, cols // block), np.float32)
    assert _load().synth_int4_blocks_b(_ptr(q), _ptr(s), rows, cols, block, seed, stream, std,
                                       _threads(nthreads)) == 0
    return q, s


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (for building test inputs)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# workloads

# Skew constant for the masked, Zipf-like workload: b_e = SKEW_C * (-ln(rank_e + 1))
# over the active experts.  Chosen by tests/golden/calibrate_skew.py (which runs
# only the oracle's router) so that the 64 highest-bias experts receive 0.73 of
# the (token, slot) selections; the realised share is stored beside it in
# tests/golden/skew_calibration.json and re-checked on a token sample by the tests.
SKEW_C = 0.05844

CONFIGS: Dict[int, dict] = {
    1: dict(workload="tiny-fp32-sigmoid", T=16, H=256, E=16, k=4, I=128, router="sigmoid",
            scale=2.446, wfmt="f32", xfmt="f32", x_std=1.0, w_std="fan_in", wr_std="fan_in",
            bias=("uniform", -0.1, 0.1), n_active=None),
    2: dict(workload="kimi-decode-bf16", T=32, H=2304, E=256, k=8, I=2048, router="sigmoid",
            scale=2.446, wfmt="bf16", xfmt="bf16", x_std=1.0, w_std=0.02, wr_std=0.02,
            wr_bf16=True, bias=("normal", 0.0, 0.05), n_active=None),
    3: dict(workload="kimi-prefill-int8", T=4096, H=2304, E=256, k=8, I=2048, router="sigmoid",
            scale=2.446, wfmt="int8", xfmt="bf16", x_std=1.0, w_std=0.02, wr_std=0.02,
            bias=("normal", 0.0, 0.05), n_active=None),
    4: dict(workload="qwen3-int4-softmax", T=1024, H=2048, E=128, k=8, I=768, router="softmax",
            scale=1.0, wfmt="int4", xfmt="bf16", x_std=1.0, w_std=0.02, wr_std=0.02,
            bias=None, n_active=None),
    5: dict(workload="kimi-skewed-masked-int8", T=16384, H=2304, E=256, k=8, I=2048,
            router="sigmoid", scale=2.446, wfmt="int8", xfmt="bf16", x_std=1.0, w_std=0.02,
            wr_std=0.02, bias=("skew", SKEW_C), n_active=160),
}


def config(cfg_id: int, **overrides) -> dict:
    c = dict(CONFIGS[cfg_id])
    c.update(overrides)
    c["cfg_id"] = cfg_id
    c.setdefault("seed", 1000 + cfg_id)
    return c


@dataclasses.dataclass
class Problem:
    """One layer instance in the stored formats (all numpy, C-contiguous)."""
    cfg: dict
    T: int
    H: int
    I: int
    E: int
    k: int
    router: str
    scale: float
    wfmt: str
    xfmt: str
    x: np.ndarray            # [T,H] f32, or uint16 bf16 bits
    W_r: np.ndarray          # [E,H] f32
    b: Optional[np.ndarray]  # [E] f32
    mask: Optional[np.ndarray]  # [E] uint8 (1 = active)
    W_gate: np.ndarray       # [E,I,H] (int4: [E,I,H/2] uint8)
    W_up: np.ndarray
    W_down: np.ndarray       # [E,H,I] (int4: [E,H,I/2] uint8)
    s_gate: Optional[np.ndarray] = None  # int8 [E,I]; int4 [E,I,H/32]
    s_up: Optional[np.ndarray] = None
    s_down: Optional[np.ndarray] = None  # int8 [E,H]; int4 [E,H,I/32] (int4b128: I/128)
    act: str = "silu"                    # gated activation: "silu" or "gelu_tanh"
    # shared expert (one dense gated FFN over every token, weight 1), stored like one
    # routed expert ([1, I_s, H] / [1, H, I_s] and scales), and the residual stream
    # [T, H] in x's format -- present only when the workload asks for them
    I_s: int = 0
    Ws_gate: Optional[np.ndarray] = None
    Ws_up: Optional[np.ndarray] = None
    Ws_down: Optional[np.ndarray] = None
    ss_gate: Optional[np.ndarray] = None
    ss_up: Optional[np.ndarray] = None
    ss_down: Optional[np.ndarray] = None
    residual: Optional[np.ndarray] = None

    def weight_bytes_per_expert(self) -> int:
        n = 0
        for a in (self.W_gate, self.W_up, self.W_down):
            n += a.nbytes // self.E
        for s in (self.s_gate, self.s_up, self.s_down):
            if s is not None:
                n += s.nbytes // self.E
        return n


def _expert_weights(fmt, E, rows, cols, seed, stream, std, nthreads):
    if fmt == "f32":
        return normal_f32((E, rows, cols), seed, stream, 0.0, std, nthreads), None
    if fmt == "bf16":
        return normal_bf16((E, rows, cols), seed, stream, 0.0, std, nthreads), None
    if fmt == "int8":
        q, s = int8_rows(E * rows, cols, seed, stream, std, nthreads)
        return q.reshape(E, rows, cols), s.reshape(E, rows)
    if fmt in INT4_BLOCK:
        B = INT4_BLOCK[fmt]
        q, s = int4_blocks(E * rows, cols, seed, stream, std, nthreads, block=B)
        return q.reshape(E, rows, cols // 2), s.reshape(E, rows, cols // B)
    raise ValueError(fmt)


def active_mask(cfg: dict) -> Optional[np.ndarray]:
    """Seeded random subset of n_active experts (1 = active), or None."""
    if not cfg.get("n_active"):
        return None
    E, n = cfg["E"], cfg["n_active"]
    u = uniform_f64(E, cfg["seed"], S_MASK)
    keep = np.argsort(u, kind="stable")[:n]
    m = np.zeros(E, np.uint8)
    m[keep] = 1
    return m


def skew_ranks(cfg: dict, mask: np.ndarray) -> np.ndarray:
    """Seeded rank of each active expert (0 = highest bias); -1 for masked experts
    (no mask: every expert is active)."""
    E = cfg["E"]
    u = uniform_f64(E, cfg["seed"], S_RANK)
    act = np.arange(E) if mask is None else np.nonzero(mask)[0]
    order = act[np.argsort(u[act], kind="stable")]
    r = np.full(E, -1, np.int64)
    r[order] = np.arange(len(order))
    return r


def skew_bias(cfg: dict, mask: np.ndarray, c: float) -> np.ndarray:
    r = skew_ranks(cfg, mask)
    b = np.zeros(cfg["E"], np.float32)
    act = r >= 0
    b[act] = (c * -np.log(r[act] + 1.0)).astype(np.float32)
    return b


def make_problem(cfg_id: int, nthreads: Optional[int] = None, replica: int = 0, **overrides) -> Problem:
    """Generate the seeded inputs of one workload (shapes may be overridden for small cases).

    ``replica`` r > 0 draws a different token batch x (seed + 1e6 * r) for the same
    layer weights -- one batch per data-parallel replica."""
    c = config(cfg_id, **overrides)
    T, H, E, k, I, seed = c["T"], c["H"], c["E"], c["k"], c["I"], c["seed"]
    x_seed = seed + 1_000_000 * int(replica)
    if c["xfmt"] == "bf16":
        x = normal_bf16((T, H), x_seed, S_X, 0.0, c["x_std"], nthreads)
    else:
        x = normal_f32((T, H), x_seed, S_X, 0.0, c["x_std"], nthreads)
    wr_std = 1.0 / math.sqrt(H) if c["wr_std"] == "fan_in" else c["wr_std"]
    if c.get("wr_bf16"):
        W_r = bf16_bits_to_f32(normal_bf16((E, H), seed, S_WR, 0.0, wr_std, nthreads)).copy()
    else:
        W_r = normal_f32((E, H), seed, S_WR, 0.0, wr_std, nthreads)
    mask = active_mask(c)
    bias = c.get("bias")
    if bias is None:
        b = None
    elif bias[0] == "uniform":
        b = uniform_f32((E,), seed, S_B, bias[1], bias[2])
    elif bias[0] == "normal":
        b = normal_f32((E,), seed, S_B, bias[1], bias[2])
    elif bias[0] == "skew":
        b = skew_bias(c, mask, bias[1])
    else:
        raise ValueError(bias)
    g_std = 1.0 / math.sqrt(H) if c["w_std"] == "fan_in" else c["w_std"]
    d_std = 1.0 / math.sqrt(I) if c["w_std"] == "fan_in" else c["w_std"]
    W_gate, s_gate = _expert_weights(c["wfmt"], E, I, H, seed, S_WG, g_std, nthreads)
    W_up, s_up = _expert_weights(c["wfmt"], E, I, H, seed, S_WU, g_std, nthreads)
    W_down, s_down = _expert_weights(c["wfmt"], E, H, I, seed, S_WD, d_std, nthreads)
    extra = {}
    I_s = int(c.get("shared") or 0)  # shared expert's intermediate size (0: none)
    if I_s:
        ds_std = 1.0 / math.sqrt(I_s) if c["w_std"] == "fan_in" else c["w_std"]
        extra["I_s"] = I_s
        extra["Ws_gate"], extra["ss_gate"] = _expert_weights(c["wfmt"], 1, I_s, H, seed, S_SG, g_std, nthreads)
        extra["Ws_up"], extra["ss_up"] = _expert_weights(c["wfmt"], 1, I_s, H, seed, S_SU, g_std, nthreads)
        extra["Ws_down"], extra["ss_down"] = _expert_weights(c["wfmt"], 1, H, I_s, seed, S_SD, ds_std, nthreads)
    if c.get("residual"):
        if c["xfmt"] == "bf16":
            extra["residual"] = normal_bf16((T, H), x_seed, S_RES, 0.0, c["x_std"], nthreads)
        else:
            extra["residual"] = normal_f32((T, H), x_seed, S_RES, 0.0, c["x_std"], nthreads)
    return Problem(cfg=c, T=T, H=H, I=I, E=E, k=k, router=c["router"], scale=float(c["scale"]),
                   wfmt=c["wfmt"], xfmt=c["xfmt"], x=x, W_r=W_r, b=b, mask=mask,
                   W_gate=W_gate, W_up=W_up, W_down=W_down,
                   s_gate=s_gate, s_up=s_up, s_down=s_down, act=c.get("act", "silu"), **extra)
