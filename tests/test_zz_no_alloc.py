"""moe_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a plugin host that owns all device buffers, or a loop that must not
call cudaMalloc once running).  Its scratch is the library's static device
array; it runs the same kernels as moe_forward on the same data, so it must give
moe_forward's result bit for bit -- on consecutive calls too, since the array
keeps the previous call's contents.  This file is named to be collected last."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import synth
from gpu_util import layer_from_problem, x_to_device

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _noalloc(layer, x, idx, w, like):
    stream = torch.cuda.current_stream().cuda_stream
    y = torch.full_like(like, float("nan"))
    moe.moe_forward_noalloc(layer.desc, x.data_ptr(), x.shape[0], idx.data_ptr(), w.data_ptr(), y.data_ptr(), stream)
    torch.cuda.synchronize()
    return y


def _bits(y):
    return y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32)


@pytest.mark.parametrize("cases", [
    # two different problems in a row: the second call runs on scratch the first one filled
    ((2, dict(T=24, H=512, E=32, I=256, seed=11)), (2, dict(T=7, H=512, E=32, I=256, seed=12))),
    # int8 experts (dequantising path), then the fp32 layer (weight-streaming path)
    ((3, dict(T=40, H=256, E=16, I=128, seed=13)), (1, dict(seed=14))),
])
def test_noalloc_matches_workspace_forward_on_consecutive_calls(cases):
    for cid, over in cases:
        prob = synth.make_problem(cid, **over)
        layer = layer_from_problem(prob)
        x = x_to_device(prob)
        idx, w = layer.route(x)
        y_ws = layer.forward(x, idx, w)
        torch.cuda.synchronize()
        for _ in range(2):
            y = _noalloc(layer, x, idx, w, y_ws)
            assert torch.equal(_bits(y), _bits(y_ws))
    assert moe.moe_device_flags(clear=True) == 0


def test_noalloc_takes_batches_that_fit_the_forward_pass_alone():
    """115 tokens at the Kimi widths (H = 2304, I = 2048, k = 8) need more than the
    array under moe_workspace_size's layout, which also holds moe_route's logits and
    split router weights, but fit as a forward pass alone -- and give moe_forward's
    bits, twice in a row."""
    prob = synth.make_problem(2, T=115, E=32, seed=15)
    layer = layer_from_problem(prob)
    assert moe.moe_workspace_size(layer.desc, prob.T) > moe.MOE_NOALLOC_SCRATCH_BYTES
    x = x_to_device(prob)
    idx, w = layer.route(x)
    y_ws = layer.forward(x, idx, w)
    torch.cuda.synchronize()
    for _ in range(2):
        assert torch.equal(_bits(_noalloc(layer, x, idx, w, y_ws)), _bits(y_ws))
    assert moe.moe_device_flags(clear=True) == 0


def test_noalloc_rejects_problems_larger_than_its_scratch():
    prob = synth.make_problem(2, T=2, H=512, E=32, I=256)
    layer = layer_from_problem(prob)
    T_big = 4096  # needs far more than the static scratch holds
    assert moe.moe_workspace_size(layer.desc, T_big) > moe.MOE_NOALLOC_SCRATCH_BYTES
    n = moe.moe_launch_count()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward_noalloc(layer.desc, 1 << 20, T_big, 1 << 20, 1 << 20, 1 << 20, 0)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    assert "static scratch" in str(ei.value)
    assert moe.moe_launch_count() == n
