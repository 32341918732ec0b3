"""Pins for the fp64 oracle: each test checks it against something other than
itself -- hand-derived closed forms, brute force over all subsets, the torch
library SwiGLU, the encoders' error bound against the real-valued weights, and
the invariants the pages state (renormalised weights sum to the scale; masking
experts equals slicing them out; only routed experts contribute)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from helpers import dense_weights, dense_x, ln_expr, problem_from_arrays, textbook_swiglu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _hand_problem(case):
    mat = lambda m: np.array([[ln_expr(v) for v in row] for row in m], np.float64)
    W_r = mat(case["W_r"]).astype(np.float32)
    Wg = np.stack([mat(m) for m in case["W_gate"]]).astype(np.float32)
    Wu = np.stack([mat(m) for m in case["W_up"]]).astype(np.float32)
    Wd = np.stack([mat(m) for m in case["W_down"]]).astype(np.float32)
    x = np.array([case["x"]], np.float32)
    return problem_from_arrays(x, W_r, Wg, Wu, Wd, k=case["k"], scale=case["scale"],
                               router=case["router"], b=case.get("b"))


@pytest.mark.parametrize("name", ["sigmoid_bias", "softmax"])
def test_hand_examples(name):
    """Closed forms derived by hand from the pages' definition (tests/golden/hand_examples.json).
    float32 storage of ln-values limits agreement to ~1e-7 relative."""
    case = json.load(open(GOLDEN))[name]
    prob = _hand_problem(case)
    y, idx, w, margin = oracle.Oracle(prob, nthreads=1).forward()
    ev = lambda v: ln_expr(v) if isinstance(v, str) else float(v)
    assert idx[0].tolist() == case["expect_idx"]
    np.testing.assert_allclose(w[0], [ev(v) for v in case["expect_w"]], rtol=1e-6)
    assert margin[0] == pytest.approx(ev(case["expect_margin"]), rel=1e-6)
    np.testing.assert_allclose(y[0] / math.log(3.0), case["expect_y_over_ln3"], rtol=1e-6, atol=1e-6)


def _random_problem(seed, E=7, H=12, I=5, T=6, k=3, router="sigmoid", wfmt="f32", mask=None, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    W_r = rng.standard_normal((E, H)).astype(np.float32) * 0.5
    Wg = rng.standard_normal((E, I, H)).astype(np.float32) / math.sqrt(H)
    Wu = rng.standard_normal((E, I, H)).astype(np.float32) / math.sqrt(H)
    Wd = rng.standard_normal((E, H, I)).astype(np.float32) / math.sqrt(I)
    b = rng.uniform(-0.3, 0.3, E).astype(np.float32) if (bias and router == "sigmoid") else None
    return problem_from_arrays(x, W_r, Wg, Wu, Wd, k=k, scale=2.446 if router == "sigmoid" else 1.0,
                               router=router, b=b, mask=mask)


@pytest.mark.parametrize("router", ["sigmoid", "softmax"])
@pytest.mark.parametrize("seed", range(4))
def test_topk_brute_force(router, seed):
    """Selection equals the unique k-subset that dominates every unselected expert,
    found by enumerating all subsets; keys computed with scipy (expit / softmax)."""
    mask = None
    if seed % 2:
        mask = np.ones(7, np.uint8)
        mask[[1, 4]] = 0
    prob = _random_problem(seed, router=router, mask=mask)
    orc = oracle.Oracle(prob, nthreads=1)
    _, idx, w, margin = orc.forward()
    x64 = prob.x.astype(np.float64)
    logits = x64 @ prob.W_r.astype(np.float64).T
    active = [e for e in range(prob.E) if mask is None or mask[e]]
    for t in range(prob.T):
        if router == "sigmoid":
            score = scipy.special.expit(logits[t])
            key = score + (prob.b.astype(np.float64) if prob.b is not None else 0.0)
        else:
            p = np.zeros(prob.E)
            p[active] = scipy.special.softmax(logits[t][active])
            key = score = p
        winners = []
        for S in itertools.combinations(active, prob.k):
            rest = [e for e in active if e not in S]
            if all((key[i], -i) > (key[j], -j) for i in S for j in rest):
                winners.append(set(S))
        assert len(winners) == 1
        assert set(idx[t].tolist()) == winners[0]
        order = sorted(winners[0], key=lambda e: (-key[e], e))
        assert idx[t].tolist() == order
        ref_w = score[order] / score[order].sum() * prob.scale
        np.testing.assert_allclose(w[t], ref_w, rtol=1e-12)
        rest = sorted(set(active) - winners[0], key=lambda e: (-key[e], e))
        assert margin[t] == pytest.approx(key[order[-1]] - key[rest[0]], rel=1e-9, abs=1e-15)


@pytest.mark.parametrize("cfg_id", [1, 4])
def test_weights_sum_to_scale(cfg_id):
    """Renormalised weights sum to the scale factor (2.446 Kimi, 1 Qwen3)."""
    prob = synth.make_problem(cfg_id, T=24, H=256, I=128, E=min(32, synth.CONFIGS[cfg_id]["E"]))
    _, w, _ = oracle.Oracle(prob).route()
    np.testing.assert_allclose(w.sum(1), prob.scale, rtol=1e-12)
    assert (w > 0).all()


def test_k1_weight_is_scale():
    prob = _random_problem(11, k=1)
    _, idx, w, _ = oracle.Oracle(prob, nthreads=1).forward()
    assert (w == np.float64(2.446)).all()


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("wfmt", ["f32", "bf16", "int8", "int4", "int4b128"])
@pytest.mark.parametrize("xfmt", ["f32", "bf16"])
def test_single_expert_reduces_to_dense_swiglu(wfmt, xfmt, act):
    """k = E = 1: the layer is scale * act(W_gate x) * (W_up x) through W_down, checked
    against torch's silu / tanh-gelu and linear on independently decoded weights, for
    every stored weight format and both activations."""
    n = 128 if wfmt == "int4b128" else 64
    prob = synth.make_problem(1, T=5, H=n, I=n, E=1, k=1, wfmt=wfmt, xfmt=xfmt, seed=77,
                              w_std=0.05, bias=None, act=act)
    y, idx, w, _ = oracle.Oracle(prob).forward()
    assert (idx == 0).all()
    ref = prob.scale * textbook_swiglu(dense_x(prob), dense_weights(prob, "gate")[0],
                                       dense_weights(prob, "up")[0], dense_weights(prob, "down")[0], act)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_activations_differ_where_they_should():
    """The activation attribute reaches the expert: SiLU and tanh-GELU give different
    outputs on the same layer, and both vanish with the gate weights."""
    a = synth.make_problem(1, T=3, H=64, I=64, E=4, k=2, seed=78)
    b = synth.make_problem(1, T=3, H=64, I=64, E=4, k=2, seed=78, act="gelu_tanh")
    ya, ia, _, _ = oracle.Oracle(a, nthreads=1).forward()
    yb, ib, _, _ = oracle.Oracle(b, nthreads=1).forward()
    assert (ia == ib).all()
    assert np.abs(ya - yb).max() > 1e-3 * np.abs(ya).max()


@pytest.mark.parametrize("router", ["sigmoid", "softmax"])
def test_all_experts_selected_is_dense_mixture(router):
    """k = E: y = sum_e w_e SwiGLU_e(x) with w_e the scores renormalised over all experts."""
    prob = _random_problem(5, E=4, k=4, router=router, T=3)
    y, _, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    x = prob.x.astype(np.float64)
    logits = x @ prob.W_r.astype(np.float64).T
    r = scipy.special.expit(logits) if router == "sigmoid" else scipy.special.softmax(logits, axis=1)
    wts = r / r.sum(1, keepdims=True) * prob.scale
    ref = sum(wts[:, e:e + 1] * textbook_swiglu(x, dense_weights(prob, "gate")[e], dense_weights(prob, "up")[e],
                                                dense_weights(prob, "down")[e]) for e in range(prob.E))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_identical_experts_give_scaled_swiglu():
    prob = _random_problem(6, E=6, k=3)
    for W in (prob.W_gate, prob.W_up, prob.W_down):
        W[:] = W[0]
    y, _, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    x = prob.x.astype(np.float64)
    ref = prob.scale * textbook_swiglu(x, prob.W_gate[0].astype(np.float64), prob.W_up[0].astype(np.float64),
                                       prob.W_down[0].astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_zero_input_and_zero_gate():
    prob = _random_problem(7)
    prob.x[:] = 0
    y, _, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    assert (y == 0).all()
    prob = _random_problem(8)
    prob.W_gate[:] = 0
    y, _, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    assert (y == 0).all()


@pytest.mark.parametrize("router", ["sigmoid", "softmax"])
def test_mask_equals_slice(router):
    """The pages' defrag invariant: masking experts is bit-identical to slicing the
    router rows, the selection bias and the experts into a dense prefix."""
    prob = synth.make_problem(5, T=40, H=128, I=64, E=24, n_active=11, router=router,
                              bias=("skew", 0.2) if router == "sigmoid" else None, seed=31)
    act = np.nonzero(prob.mask)[0]
    sl = problem_from_arrays(
        prob.x, prob.W_r[act], prob.W_gate[act], prob.W_up[act], prob.W_down[act], k=prob.k,
        scale=prob.scale, router=router, b=None if prob.b is None else prob.b[act], wfmt=prob.wfmt,
        xfmt=prob.xfmt, s_gate=prob.s_gate[act], s_up=prob.s_up[act], s_down=prob.s_down[act])
    y1, i1, w1, m1 = oracle.Oracle(prob).forward()
    y2, i2, w2, m2 = oracle.Oracle(sl).forward()
    assert (act[i2] == i1).all()
    assert np.array_equal(w1, w2) and np.array_equal(y1, y2) and np.array_equal(m1, m2)
    assert prob.mask[i1].all()


def test_expert_relabelling_invariance():
    prob = _random_problem(9, E=7, T=8)
    perm = np.random.default_rng(1).permutation(prob.E)
    q = problem_from_arrays(prob.x, prob.W_r[perm], prob.W_gate[perm], prob.W_up[perm], prob.W_down[perm],
                            k=prob.k, scale=prob.scale, b=prob.b[perm])
    y1, i1, _, m1 = oracle.Oracle(prob, nthreads=1).forward()
    y2, i2, _, _ = oracle.Oracle(q, nthreads=1).forward()
    ok = m1 > 1e-9
    assert (perm[i2[ok]] == i1[ok]).all()
    np.testing.assert_allclose(y2[ok], y1[ok], rtol=1e-12, atol=1e-14)


def test_token_permutation_equivariance():
    prob = _random_problem(10, T=9)
    perm = np.random.default_rng(2).permutation(prob.T)
    q = problem_from_arrays(prob.x[perm], prob.W_r, prob.W_gate, prob.W_up, prob.W_down, k=prob.k,
                            scale=prob.scale, b=prob.b)
    y1, _, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    y2, _, _, _ = oracle.Oracle(q, nthreads=1).forward()
    assert np.array_equal(y2, y1[perm])


def test_softmax_denominator_cancels():
    """Renormalising the softmax over the selected experts equals a softmax of the
    selected logits alone (the full denominator cancels)."""
    prob = _random_problem(12, E=9, k=4, router="softmax", T=10)
    _, idx, w, _ = oracle.Oracle(prob, nthreads=1).forward()
    logits = prob.x.astype(np.float64) @ prob.W_r.astype(np.float64).T
    for t in range(prob.T):
        np.testing.assert_allclose(w[t], scipy.special.softmax(logits[t][idx[t]]), rtol=1e-12)


@pytest.mark.parametrize("wfmt", ["int8", "int4", "int4b128", "bf16"])
def test_oracle_dequantisation_matches_real_weights(wfmt):
    """The oracle's decode of each stored format lies within half a quantisation step
    of the real-valued weight the encoder started from (regenerated from the same
    random stream); bf16 within half an ulp."""
    H, I, E = (128, 256, 3) if wfmt == "int4b128" else (64, 96, 3)
    prob = synth.make_problem(3, T=2, H=H, I=I, E=E, wfmt=wfmt, seed=5)
    orc = oracle.Oracle(prob, nthreads=1)
    for which, name, rows, cols in ((0, "gate", I, H), (2, "down", H, I)):
        stream = synth.S_WG if which == 0 else synth.S_WD
        real = synth.normal_f32((E, rows, cols), prob.cfg["seed"], stream, 0.0, 0.02).astype(np.float64)
        rng = np.random.default_rng(which)
        for _ in range(300):
            e, r, c = rng.integers(E), rng.integers(rows), rng.integers(cols)
            v = orc.weight(which, int(e), int(r), int(c))
            if wfmt == "int8":
                s = float(getattr(prob, "s_" + name)[e, r])
                assert abs(v - real[e, r, c]) <= s / 2 * (1 + 1e-6)
                assert abs(v / s - round(v / s)) < 1e-9 and abs(v / s) <= 127
            elif wfmt in ("int4", "int4b128"):
                s = float(getattr(prob, "s_" + name)[e, r, c // (32 if wfmt == "int4" else 128)])
                assert s >= 2.0 ** -14
                assert abs(v - real[e, r, c]) <= s / 2 * (1 + 1e-6)
                assert -8 <= round(v / s) <= 7
            else:
                assert abs(v - real[e, r, c]) <= abs(real[e, r, c]) * 2.0 ** -8


@pytest.mark.parametrize("router", ["sigmoid", "softmax"])
def test_exact_ties_break_to_lower_index(router):
    """Equal keys (duplicated router rows, equal bias) resolve to the lower expert
    index, and the output slots follow (key descending, index ascending)."""
    prob = _random_problem(13, E=8, k=3, router=router, T=4, bias=False)
    prob.W_r[:] = prob.W_r[0]           # every key equal
    prob.W_r[5] = prob.W_r[0] * 0       # expert 5 differs (logit 0)
    _, idx, _, margin = oracle.Oracle(prob, nthreads=1).forward()
    logits = prob.x.astype(np.float64) @ prob.W_r[0].astype(np.float64)
    for t in range(prob.T):
        if logits[t] > 0:    # the seven tied experts beat expert 5
            assert idx[t].tolist() == [0, 1, 2]
        else:                # expert 5 leads, then the tied ones by index
            assert idx[t].tolist() == [5, 0, 1]
    mask = np.ones(8, np.uint8)
    mask[[0, 2]] = 0
    prob.mask = mask
    _, idx, _, _ = oracle.Oracle(prob, nthreads=1).forward()
    for t in range(prob.T):
        assert idx[t].tolist() == ([1, 3, 4] if logits[t] > 0 else [5, 1, 3])


# ------------------------------------------------------------ shared expert + residual

@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("wfmt,xfmt", [("f32", "f32"), ("bf16", "bf16"), ("int8", "bf16"), ("int4", "bf16")])
def test_block_single_expert_equals_textbook(wfmt, xfmt, act):
    """k = E = 1 with a shared expert and a residual: y = residual + scale * FFN_0(x)
    + FFN_shared(x), against torch's activations and linear on independently decoded
    weights (shared I differs from the routed I)."""
    prob = synth.make_problem(1, T=4, H=64, I=64, E=1, k=1, wfmt=wfmt, xfmt=xfmt, seed=91, w_std=0.05,
                              bias=None, act=act, shared=96, residual=True)
    orc = oracle.Oracle(prob)
    idx, w, _ = orc.route()
    y = orc.block(range(prob.T), idx, w)
    x = dense_x(prob)
    ref = dense_x(prob, prob.residual) + prob.scale * textbook_swiglu(
        x, dense_weights(prob, "gate")[0], dense_weights(prob, "up")[0], dense_weights(prob, "down")[0], act)
    ref += textbook_swiglu(x, dense_weights(prob, "gate", True)[0], dense_weights(prob, "up", True)[0],
                           dense_weights(prob, "down", True)[0], act)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_block_without_shared_or_residual_is_the_routed_sum():
    prob = synth.make_problem(1, T=6, seed=92)
    orc = oracle.Oracle(prob, nthreads=1)
    idx, w, _ = orc.route()
    np.testing.assert_array_equal(orc.block(range(6), idx, w), orc.combine(range(6), idx, w))


def test_block_zero_shared_weights_add_only_the_residual():
    import dataclasses
    prob = synth.make_problem(1, T=6, seed=93, shared=64, residual=True)
    z = dataclasses.replace(prob, Ws_gate=np.zeros_like(prob.Ws_gate))
    orc = oracle.Oracle(z, nthreads=1)
    idx, w, _ = orc.route()
    np.testing.assert_array_equal(orc.block(range(6), idx, w),
                                  orc.combine(range(6), idx, w) + prob.residual.astype(np.float64))


def test_shared_expert_is_an_expert_with_weight_one():
    """A shared expert with the weights of routed expert e contributes exactly
    oracle_expert(e, x) (routing weights set to zero, no residual)."""
    import dataclasses
    prob = synth.make_problem(3, T=3, H=64, I=64, E=5, k=2, seed=94, shared=64)
    e = 3
    same = dataclasses.replace(prob, Ws_gate=prob.W_gate[e:e + 1].copy(), Ws_up=prob.W_up[e:e + 1].copy(),
                               Ws_down=prob.W_down[e:e + 1].copy(), ss_gate=prob.s_gate[e:e + 1].copy(),
                               ss_up=prob.s_up[e:e + 1].copy(), ss_down=prob.s_down[e:e + 1].copy())
    orc = oracle.Oracle(same, nthreads=1)
    idx, w, _ = orc.route()
    y = orc.block(range(3), idx, np.zeros_like(w))
    x = dense_x(same)
    for t in range(3):
        np.testing.assert_array_equal(y[t], orc.expert(e, x[t]))
