"""GPU parity of the MoE block entry point: routed experts + shared expert +
residual (Kimi-Linear APEX page: 256 routed + 1 shared expert FFN; Qwen3 card,
moe_fusion_guard bullet: the residual add sits outside the moe op and is fused
here into the combine)."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import synth
from gpu_util import (chunk_tokens, dense_cover_tokens, gpu_logits, judge, judge_block, layer_from_problem,
                      unit_cover_tokens, x_to_device)

pytestmark = pytest.mark.gpu

CASES = {
    # name: (config, overrides)
    "bf16-tc": (2, dict(T=37, H=256, E=32, I=256, shared=256, residual=True)),
    "bf16-tc-sharedI-192": (2, dict(T=45, H=256, E=32, I=128, shared=192, residual=True)),
    "int8-tc-gelu": (3, dict(T=203, H=384, E=24, I=256, shared=512, residual=True, act="gelu_tanh")),
    "int4-tc": (4, dict(T=150, H=256, E=16, I=128, shared=256, residual=True)),
    "int4b128-tc": (4, dict(T=70, H=256, E=16, I=256, shared=128, residual=True, wfmt="int4b128")),
    "fp32-gemv": (1, dict(shared=64, residual=True)),
    "bf16-gemv-oddH": (2, dict(T=29, H=320, E=16, I=128, shared=128, residual=True)),
    "shared-only": (3, dict(T=64, H=256, E=16, I=128, shared=128)),
    "residual-only": (2, dict(T=33, H=256, E=16, I=128, residual=True)),
    "large-T-chunks": (3, dict(T=1500, H=256, E=16, I=128, shared=256, residual=True)),
    "bf16-yp": (3, dict(T=2100, H=256, E=16, I=128, shared=256, residual=True)),  # routed rows in bf16
}


@pytest.fixture(autouse=True)
def _clear_flags():
    moe.moe_device_flags(clear=True)
    yield
    assert moe.moe_device_flags(clear=True) == 0


def _run_block(prob):
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    idx, w = layer.route(x)
    res = None if prob.residual is None else x_to_device(prob, prob.residual)
    y = layer.block(x, idx, w, residual=res)
    torch.cuda.synchronize()
    return layer, x, idx, w, res, y


@pytest.mark.parametrize("name", list(CASES))
def test_block_small(name):
    cid, over = CASES[name]
    prob = synth.make_problem(cid, **over)
    layer, x, idx, w, res, y = _run_block(prob)
    judge(prob, layer.forward(x, idx, w), idx, w, logits=gpu_logits(layer, x))  # the routing itself
    judge_block(prob, y, idx, w)


def test_block_decode_full_size():
    """The Kimi decode shape with a shared expert of the routed experts' size and a
    residual stream."""
    prob = synth.make_problem(2, shared=2048, residual=True)
    _, _, idx, w, _, y = _run_block(prob)
    judge_block(prob, y, idx, w)


def test_block_prefill_every_unit():
    """The int8 prefill widths with a shared expert of the routed size and a
    residual: the checked tokens reach every routed (expert, token chunk) unit and
    every unit of the shared expert, which runs as a dense problem (every token in
    order) inside the same grouped-GEMM launches."""
    prob = synth.make_problem(3, T=2048, shared=2048, residual=True)
    _, _, idx, w, _, y = _run_block(prob)
    routed, _ = unit_cover_tokens(idx.cpu().numpy(), prob.E, prob.T, prob.k)
    dense = dense_cover_tokens(prob.T, chunk_tokens(prob.T, 1, 1))
    judge_block(prob, y, idx, w, tokens=np.unique(np.concatenate([routed, dense])))


@pytest.mark.parametrize("T", [300, 2100])
def test_block_without_extras_equals_forward_bit_for_bit(T):
    prob = synth.make_problem(3, T=T, H=256, E=16, I=128)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    idx, w = layer.route(x)
    y1 = layer.forward(x, idx, w)
    y2 = layer.block(x, idx, w)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_block_in_place_residual():
    """y may be the residual buffer itself (an in-place residual update)."""
    prob = synth.make_problem(2, T=40, H=256, E=16, I=128, shared=128, residual=True)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    idx, w = layer.route(x)
    res = x_to_device(prob, prob.residual)
    y_sep = layer.block(x, idx, w, residual=res.clone())
    layer.block(x, idx, w, residual=res, y=res)
    torch.cuda.synchronize()
    assert torch.equal(y_sep.view(torch.int16), res.view(torch.int16))


def test_block_rejects_bad_shared_expert():
    prob = synth.make_problem(2, T=8, H=256, E=16, I=128, shared=128)
    layer = layer_from_problem(prob)
    layer.shared.I = 100
    x = x_to_device(prob)
    idx, w = layer.route(x)
    with pytest.raises(moe.MoeError) as ei:
        layer.block(x, idx, w)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
