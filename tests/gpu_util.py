"""Helpers for the GPU parity tests: upload a synthetic problem, run the CUDA
library through its C ABI, and judge the result against the fp64 oracle.

Judgement (the pages' checks, restated for a CUDA path):
  * routing.  The GPU ranks fp32 router logits; the oracle ranks exact (fp64)
    ones.  With the GPU's own logits in hand (moe_route_logits), the test
    measures per token delta_t = max_e |l_gpu - l_exact| and first checks it
    against a worst-case fp32 bound (3H * 2^-23 * sum_h |W_r[e,h] x[t,h]|: the
    logits really are fp32-accurate).  Wherever the exact gap between the k-th
    and (k+1)-th key exceeds twice the key error that delta_t allows, no fp32
    ranking can differ from the exact one, so the GPU's experts must equal the
    oracle's bit for bit (in slot order too where every gap among the first
    k+1 keys is resolved).  Every token -- near-ties included -- must hold the
    top k of the GPU's own fp32 keys.  The pages' margin rule is kept on top:
    wherever the oracle's k-th/(k+1)-th key margin exceeds 1e-4 the indices
    match exactly; tokens at or below it are counted as near-ties (probability
    domain for the softmax router), and the tokens fp32 cannot resolve are
    counted separately;
  * routing weights match the oracle's to fp32 accuracy where indices match;
  * y is compared with the oracle's combine under the GPU's own routing (so
    near-tie tokens are judged too): ||y - y_ref||_2 / ||y_ref||_2 over the
    judged tokens within the stated tolerance (1e-5 for the all-fp32 layer, 5e-3
    with bf16 activations), and every single token within twice that.
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_31_b200 as moe
import oracle
from helpers import dense_x

MARGIN = 1e-4
TOL_F32 = 1e-5
TOL_BF16 = 5e-3
TOKEN_FACTOR = 2.0  # per-token relative L2 bound, as a multiple of the whole-tensor bar
KEY_ROUNDING = 2.0 ** -20  # fp32 rounding of sigmoid(l) + b on the GPU (a few ulp of a key <= 2)


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


def gpu_logits(layer, x) -> np.ndarray:
    """The router logits the GPU ranked for x (moe_route_logits), as float32 [T, E]."""
    lg = layer.route_logits(x)
    torch.cuda.synchronize()
    return lg.cpu().numpy()


# ------------------------------------------------------------------ which tokens reach which work units

def chunk_tokens(T: int, k: int, E: int) -> int:
    """Token chunk of the grouped GEMMs' work units for a batch of T tokens: T
    rounded up to 16, at most 256, and 128 when the average expert gets at most
    96 pairs (the tiling rule of the library's tensor-core path)."""
    t = min(256, (max(T, 1) + 15) // 16 * 16)
    if t > 128 and T * k <= 96 * E:
        t = 128
    return t


def _pick_positions(start: int, n: int, chunk: int, box: int = 32):
    """Positions (relative to an expert's first sorted pair) that touch every
    work unit of an expert with n pairs: in each chunk its first, middle and last
    pair and one pair in every `box`-row token box, alternating between the two
    16-column halves that the epilogue's two warp groups drain."""
    pos = []
    for c0 in range(0, n, chunk):
        m = min(chunk, n - c0)
        pos += [c0, c0 + m // 2, c0 + m - 1]
        for b, b0 in enumerate(range(0, m, box)):
            off = min(b0 + 16 * (b % 2) + 7, m - 1)
            pos.append(c0 + off)
    return [start + p for p in pos]


def unit_cover_tokens(idx: np.ndarray, E: int, T: int, k: int, chunk=None):
    """Tokens whose outputs, checked in full, reach every (expert, token chunk) work
    unit of the routed grouped GEMMs (every row block of a unit lands in every
    checked token's output row).  The expert-sorted order is the library's: pairs
    t*k + slot, stably by expert.  Returns (tokens, number of units)."""
    chunk = chunk or chunk_tokens(T, k, E)
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    pairs = np.nonzero(valid)[0]
    order = pairs[np.argsort(flat[pairs], kind="stable")]
    counts = np.bincount(flat[pairs], minlength=E)
    offs = np.concatenate([[0], np.cumsum(counts)])
    picks, units = [], 0
    for e in np.nonzero(counts)[0]:
        units += (counts[e] + chunk - 1) // chunk
        picks += _pick_positions(int(offs[e]), int(counts[e]), chunk)
    toks = np.unique(order[np.asarray(picks, dtype=np.int64)] // k)
    return toks, int(units)


def dense_cover_tokens(T: int, chunk: int):
    """The same for a dense problem (the shared expert: every token in order)."""
    return np.unique(np.asarray(_pick_positions(0, T, chunk), dtype=np.int64))


# ------------------------------------------------------------------ judging

def _keys_f32(prob, lg: np.ndarray, active: np.ndarray) -> np.ndarray:
    """The GPU's keys from its fp32 logits, recomputed in fp32: sigmoid(l) + b, or l
    itself (the softmax router ranks the logits, whose order is the softmax's)."""
    lg = lg.astype(np.float32)
    if prob.router == "sigmoid":
        one = np.float32(1.0)
        key = one / (one + np.exp(-lg))
        if prob.b is not None:
            key = key + prob.b.astype(np.float32)
    else:
        key = lg.copy()
    key = key.astype(np.float64)
    key[:, ~active] = -np.inf
    return key


def _check_routing(prob, gi, gw, tokens, orc, lg):
    """The routing rules of the module docstring; returns counts for the report."""
    k, E = prob.k, prob.E
    active = np.ones(E, bool) if prob.mask is None else prob.mask.astype(bool)
    n_act = int(active.sum())
    idx_ref, w_ref, margin = orc.route(tokens)
    rep = dict(near_ties=int((margin <= MARGIN).sum()))
    # every token: k distinct active experts
    for i in range(len(tokens)):
        sel = gi[i]
        assert len(set(sel.tolist())) == k and (sel >= 0).all() and active[sel].all(), \
            "token %d: invalid selection %s" % (tokens[i], sel)
    # the pages' rule: indices exact above the 1e-4 margin
    clear = margin > MARGIN
    mism = np.nonzero(clear & (np.sort(gi, 1) != np.sort(idx_ref, 1)).any(1))[0]
    assert mism.size == 0, "index mismatch above the margin at tokens %s" % tokens[mism][:10]
    if lg is None:
        if clear.any():
            np.testing.assert_allclose(gw[clear], w_ref[clear], rtol=2e-4, atol=1e-6)
        return rep
    lo = orc.logits(tokens)  # exact logits, fp64
    err = np.abs(lg.astype(np.float64) - lo)
    err[:, ~active] = 0.0
    # the logits are fp32-accurate: within a worst-case fp32 summation bound
    sabs = np.abs(dense_x(prob)[tokens]) @ np.abs(prob.W_r.astype(np.float64)).T
    bound = 3.0 * prob.H * 2.0 ** -23 * sabs + 1e-30
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert (err <= bound).all(), "logit error %.3e above its fp32 bound %.3e (token %d, expert %d)" % (
        err[worst], bound[worst], tokens[worst[0]], worst[1])
    delta = err.max(1)
    dkey = 0.25 * delta + KEY_ROUNDING if prob.router == "sigmoid" else delta
    # exact keys in the domain the GPU ranks in (sigmoid + bias, or the logits)
    if prob.router == "sigmoid":
        ekey = np.stack([orc.keys(row) for row in lo])
    else:
        ekey = lo.copy()
    ekey[:, ~active] = -np.inf
    order = np.lexsort((np.broadcast_to(np.arange(E), ekey.shape), -ekey), axis=1)[:, :min(k + 1, n_act)]
    top = np.take_along_axis(ekey, order, 1)
    gaps = top[:, :-1] - top[:, 1:] if top.shape[1] > k else np.concatenate(
        [top[:, :-1] - top[:, 1:], np.full((len(tokens), 1), np.inf)], 1)
    set_ok = gaps[:, k - 1] > 2.0 * dkey
    order_ok = gaps[:, :k].min(1) > 2.0 * dkey
    bad = np.nonzero(set_ok & (np.sort(gi, 1) != np.sort(order[:, :k], 1)).any(1))[0]
    assert bad.size == 0, "experts differ from the exact top-k where fp32 resolves it: tokens %s" % tokens[bad][:10]
    bad = np.nonzero(order_ok & (gi != order[:, :k]).any(1))[0]
    assert bad.size == 0, "slot order differs where fp32 resolves it: tokens %s" % tokens[bad][:10]
    if order_ok.any():
        np.testing.assert_allclose(gw[order_ok], w_ref[order_ok], rtol=2e-4, atol=1e-6)
    # every token holds the top k of the GPU's own keys
    gkey = _keys_f32(prob, lg, active)
    finite_max = np.where(np.isfinite(gkey), np.abs(gkey), 0.0).max(1)
    slack = 16 * np.spacing(finite_max.astype(np.float32)).astype(np.float64) \
        if prob.router == "sigmoid" else np.zeros(len(tokens))
    for i in range(len(tokens)):
        rest = np.ones(E, bool)
        rest[gi[i]] = False
        rest &= active
        if rest.any():
            assert gkey[i, gi[i]].min() >= gkey[i, rest].max() - slack[i], \
                "token %d: selection is not the top k of the GPU's own keys" % tokens[i]
    rep.update(fp32_unresolved=int((~set_ok).sum()), exact_set=int(set_ok.sum()),
               max_logit_err=float(delta.max()), max_logit_err_over_bound=float((err / bound).max()))
    return rep


def judge(prob, y, idx, w, tokens=None, orc=None, tol=None, logits=None):
    """Assert parity with the oracle on `tokens` (default: all); returns a report dict.

    logits: the GPU's router logits for all T tokens (gpu_logits), which turn on
    the fp32-resolution index rule; without them only the 1e-4 margin rule runs."""
    tokens = np.arange(prob.T) if tokens is None else np.asarray(tokens)
    orc = orc or oracle.Oracle(prob)
    gi = idx.cpu().numpy()[tokens]
    gw = w.cpu().numpy()[tokens].astype(np.float64)
    rep = _check_routing(prob, gi, gw, tokens, orc, None if logits is None else np.asarray(logits)[tokens])
    y_ref = orc.combine(tokens, gi, gw)
    yg = y.double().cpu().numpy()[tokens]
    rep.update(_check_output(prob, yg, y_ref, tokens, tol))
    return rep


def _check_output(prob, yg, y_ref, tokens, tol, what="y"):
    tol = tolerance(prob) if tol is None else tol
    rel = float(np.linalg.norm(yg - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    assert rel <= tol, "%s: relative L2 error %.3e above %.1e" % (what, rel, tol)
    per = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-300)
    wt = int(np.argmax(per))
    assert per[wt] <= TOKEN_FACTOR * tol, "%s: token %d relative L2 error %.3e above %.1e" % (
        what, tokens[wt], per[wt], TOKEN_FACTOR * tol)
    return dict(tokens=int(len(tokens)), rel_l2=rel, worst_token_rel_l2=float(per[wt]), worst_token=int(tokens[wt]))


def judge_block(prob, y, idx, w, tokens=None, orc=None, tol=None):
    """Block output (routed + shared + residual) against the oracle's block under the
    GPU's own routing, which judge() has already held to the routing rules."""
    tokens = np.arange(prob.T) if tokens is None else np.asarray(tokens)
    orc = orc or oracle.Oracle(prob)
    gi = idx.cpu().numpy()[tokens]
    gw = w.cpu().numpy()[tokens].astype(np.float64)
    y_ref = orc.block(tokens, gi, gw)
    yg = y.double().cpu().numpy()[tokens]
    return _check_output(prob, yg, y_ref, tokens, tol, what="block")
