"""Helpers for the GPU parity tests: upload a synthetic problem, run the CUDA
library through its C ABI, and judge the result against the fp64 oracle.

Judgement (the pages' checks, restated for a CUDA path):
  * top-k indices equal the oracle's bit for bit wherever the oracle's margin
    between the k-th and (k+1)-th key exceeds 1e-4; near-ties are counted, and
    for them the GPU's choice must still be a valid top-k within 1e-4;
  * routing weights match the oracle's to fp32 accuracy where indices match;
  * y is compared with the oracle's combine under the GPU's own routing (so
    near-tie tokens are judged too): ||y - y_ref||_2 / ||y_ref||_2 within the
    stated tolerance (1e-5 for the all-fp32 layer, 5e-3 with bf16 activations).
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_31_b200 as moe
import oracle

MARGIN = 1e-4
TOL_F32 = 1e-5
TOL_BF16 = 5e-3


def tolerance(prob) -> float:
    return TOL_F32 if (prob.xfmt == "f32" and prob.wfmt == "f32") else TOL_BF16


def layer_from_problem(prob, path=moe.MOE_PATH_AUTO) -> moe.MoELayer:
    return moe.MoELayer(H=prob.H, I=prob.I, E=prob.E, k=prob.k, router=prob.router, scale=prob.scale,
                        wfmt=prob.wfmt, xfmt=prob.xfmt, W_r=prob.W_r, b=prob.b, expert_mask=prob.mask,
                        W_gate=prob.W_gate, W_up=prob.W_up, W_down=prob.W_down, s_gate=prob.s_gate,
                        s_up=prob.s_up, s_down=prob.s_down, path=path, act=prob.act, I_s=prob.I_s,
                        Ws_gate=prob.Ws_gate, Ws_up=prob.Ws_up, Ws_down=prob.Ws_down, ss_gate=prob.ss_gate,
                        ss_up=prob.ss_up, ss_down=prob.ss_down)


def x_to_device(prob, a=None) -> torch.Tensor:
    """x (or another [T, H] array in x's format, e.g. the residual) on the GPU."""
    a = prob.x if a is None else a
    if prob.xfmt == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def run(prob, path=moe.MOE_PATH_AUTO, layer=None):
    layer = layer or layer_from_problem(prob, path)
    x = x_to_device(prob)
    y, idx, w = layer(x)
    torch.cuda.synchronize()
    return layer, x, y, idx, w


def judge(prob, y, idx, w, tokens=None, orc=None, tol=None):
    """Assert parity with the oracle on `tokens` (default: all); returns a report dict."""
    tokens = np.arange(prob.T) if tokens is None else np.asarray(tokens)
    orc = orc or oracle.Oracle(prob)
    idx_ref, w_ref, margin = orc.route(tokens)
    gi = idx.cpu().numpy()[tokens]
    gw = w.cpu().numpy()[tokens].astype(np.float64)
    clear = margin > MARGIN
    mism = np.nonzero(clear & (gi != idx_ref).any(1))[0]
    assert mism.size == 0, "index mismatch above the margin at tokens %s" % tokens[mism][:10]
    if clear.any():
        np.testing.assert_allclose(gw[clear], w_ref[clear], rtol=2e-4, atol=1e-6)
    active = np.ones(prob.E, bool) if prob.mask is None else prob.mask.astype(bool)
    near = np.nonzero(~clear)[0]
    if near.size:
        lg = orc.logits(tokens[near])
        for j, i in enumerate(near):
            keys = orc.keys(lg[j])
            sel = gi[i]
            assert len(set(sel.tolist())) == prob.k and active[sel].all()
            rest = np.setdiff1d(np.nonzero(active)[0], sel)
            if rest.size:
                assert keys[sel].min() >= keys[rest].max() - MARGIN
    y_ref = orc.combine(tokens, gi, gw)
    yg = y.double().cpu().numpy()[tokens]
    rel = float(np.linalg.norm(yg - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    tol = tolerance(prob) if tol is None else tol
    assert rel <= tol, "relative L2 error %.3e above %.1e" % (rel, tol)
    return dict(tokens=int(tokens.size), near_ties=int(near.size), rel_l2=rel)


def judge_block(prob, y, idx, w, tokens=None, orc=None, tol=None):
    """Block output (routed + shared + residual) against the oracle's block under the
    GPU's own routing, which judge() has already held to the routing rules."""
    tokens = np.arange(prob.T) if tokens is None else np.asarray(tokens)
    orc = orc or oracle.Oracle(prob)
    gi = idx.cpu().numpy()[tokens]
    gw = w.cpu().numpy()[tokens].astype(np.float64)
    y_ref = orc.block(tokens, gi, gw)
    yg = y.double().cpu().numpy()[tokens]
    rel = float(np.linalg.norm(yg - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    tol = tolerance(prob) if tol is None else tol
    assert rel <= tol, "block: relative L2 error %.3e above %.1e" % (rel, tol)
    return dict(tokens=int(tokens.size), rel_l2=rel)
