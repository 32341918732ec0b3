"""Shared test helpers: building small problems from explicit arrays, and
independent textbook references (numpy / torch library routines) used to pin
the oracle.  Nothing here imports the CUDA library."""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import synth


def problem_from_arrays(x, W_r, W_gate, W_up, W_down, k, scale, router="sigmoid", b=None,
                        mask=None, wfmt="f32", xfmt="f32", s_gate=None, s_up=None, s_down=None):
    E, H = W_r.shape
    I = W_gate.shape[1]
    c = dict(workload="explicit", T=x.shape[0], H=H, E=E, k=k, I=I, router=router, scale=scale,
             wfmt=wfmt, xfmt=xfmt, cfg_id=0, seed=0)
    f = lambda a, dt=None: None if a is None else np.ascontiguousarray(a if dt is None else np.asarray(a, dt))
    return synth.Problem(cfg=c, T=x.shape[0], H=H, I=I, E=E, k=k, router=router, scale=float(scale),
                         wfmt=wfmt, xfmt=xfmt, x=f(x), W_r=f(W_r, np.float32), b=f(b, np.float32),
                         mask=f(mask, np.uint8), W_gate=f(W_gate), W_up=f(W_up), W_down=f(W_down),
                         s_gate=f(s_gate, np.float32), s_up=f(s_up, np.float32),
                         s_down=f(s_down, np.float32))


def dense_weights(prob, which, shared=False):
    """Dequantised expert matrices as float64 [E, rows, cols] (the shared expert's as
    [1, rows, cols] when shared), decoded with numpy."""
    if shared:
        W = {"gate": prob.Ws_gate, "up": prob.Ws_up, "down": prob.Ws_down}[which]
        S = {"gate": prob.ss_gate, "up": prob.ss_up, "down": prob.ss_down}[which]
    else:
        W = {"gate": prob.W_gate, "up": prob.W_up, "down": prob.W_down}[which]
        S = {"gate": prob.s_gate, "up": prob.s_up, "down": prob.s_down}[which]
    if prob.wfmt == "f32":
        return W.astype(np.float64)
    if prob.wfmt == "bf16":
        return synth.bf16_bits_to_f32(W).astype(np.float64)
    if prob.wfmt == "int8":
        return W.astype(np.float64) * S[..., None].astype(np.float64)
    if prob.wfmt in ("int4", "int4b128"):
        block = 32 if prob.wfmt == "int4" else 128
        lo = (W & 0xF).astype(np.int64)
        hi = (W >> 4).astype(np.int64)
        lo = np.where(lo >= 8, lo - 16, lo)
        hi = np.where(hi >= 8, hi - 16, hi)
        q = np.empty(W.shape[:-1] + (W.shape[-1] * 2,), np.float64)
        q[..., 0::2] = lo
        q[..., 1::2] = hi
        return q * np.repeat(S.astype(np.float64), block, axis=-1)
    raise ValueError(prob.wfmt)


def dense_x(prob, a=None):
    a = prob.x if a is None else a
    if prob.xfmt == "bf16":
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return a.astype(np.float64)


def textbook_swiglu(x, Wg, Wu, Wd, act="silu"):
    """torch library gated FFN in fp64: Wd (act(Wg x) * (Wu x)) for rows of x, with act
    torch's silu or its tanh-approximated gelu."""
    x = torch.as_tensor(x, dtype=torch.float64)
    g = F.linear(x, torch.as_tensor(Wg))
    a = F.silu(g) if act == "silu" else F.gelu(g, approximate="tanh")
    return F.linear(a * F.linear(x, torch.as_tensor(Wu)), torch.as_tensor(Wd)).numpy()


def ln_expr(s: str) -> float:
    """Evaluate the tiny expressions used in the hand-example fixture."""
    s = s.replace(" ", "")
    if "/" in s and "ln" not in s:
        a, b = s.split("/")
        return float(a) / float(b)
    neg = s.startswith("-")
    s = s.lstrip("-")
    if s.endswith("ln3") or s.endswith("ln2"):
        base = math.log(3.0) if s.endswith("ln3") else math.log(2.0)
        coef = s[:-3]
        v = (float(coef) if coef else 1.0) * base
    else:
        v = float(s)
    return -v if neg else v
