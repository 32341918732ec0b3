"""moe_forward_noalloc: the forward pass for callers that cannot allocate device
memory (a plugin host that owns all device buffers, or a loop that must not
call cudaMalloc once running).  Its scratch is the library's static device
array, so it must give what moe_forward gives with a caller workspace -- on
consecutive calls too, since the array keeps the previous call's contents.
This file is named to be collected last."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import synth
from gpu_util import TOL_BF16, layer_from_problem, x_to_device

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_noalloc_matches_workspace_forward_on_consecutive_calls():
    stream = torch.cuda.current_stream().cuda_stream
    # two different problems in a row: the second call runs on scratch the first one filled
    for T, seed in ((24, 11), (7, 12)):
        prob = synth.make_problem(2, T=T, H=512, E=32, I=256, seed=seed)
        layer = layer_from_problem(prob)
        x = x_to_device(prob)
        idx, w = layer.route(x)
        y_ws = layer.forward(x, idx, w)
        assert moe.moe_workspace_size(layer.desc, T) <= moe.MOE_NOALLOC_SCRATCH_BYTES
        for _ in range(2):
            y = torch.full_like(y_ws, float("nan"))
            moe.moe_forward_noalloc(layer.desc, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), y.data_ptr(), stream)
            torch.cuda.synchronize()
            assert torch.isfinite(y.float()).all()
            assert _rel(y, y_ws) <= TOL_BF16
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
