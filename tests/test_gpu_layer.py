"""GPU parity of moe_layer_forward: route and forward in one call, with the
router logits, top-k and expert sort fused into two launches for decode-sized
batches (T <= 32, E <= 256), and the separate steps otherwise."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import synth
from gpu_util import gpu_logits, judge, layer_from_problem, x_to_device

pytestmark = pytest.mark.gpu

CASES = {
    "kimi-bf16-decode": (2, dict(T=32, H=256, E=64, I=256)),
    "kimi-bf16-T1": (2, dict(T=1, H=256, E=64, I=128)),
    "kimi-bf16-T7-ragged": (2, dict(T=7, H=320, E=40, I=192)),
    "kimi-int8-decode": (3, dict(T=24, H=384, E=48, I=256)),
    "qwen3-int4-softmax": (4, dict(T=32, H=256, E=128, I=128)),
    "tiny-fp32": (1, {}),
    "skew-masked": (5, dict(T=30, H=256, E=64, I=128, n_active=20, bias=("skew", 0.2))),
    "wide-E-fallback": (2, dict(T=16, H=256, E=320, I=128)),
    "T33-fallback": (3, dict(T=33, H=256, E=32, I=128)),
    "gelu-int4b128": (4, dict(T=20, H=256, E=32, I=256, wfmt="int4b128", act="gelu_tanh")),
}


@pytest.fixture(autouse=True)
def _clear_flags():
    moe.moe_device_flags(clear=True)
    yield
    assert moe.moe_device_flags(clear=True) == 0


@pytest.mark.parametrize("name", list(CASES))
def test_layer_forward_matches_oracle_and_the_separate_steps(name):
    cid, over = CASES[name]
    prob = synth.make_problem(cid, **over)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    y, idx, w = layer.layer(x)
    torch.cuda.synchronize()
    judge(prob, y, idx, w, logits=gpu_logits(layer, x))
    # the separate entry points on the same input: same routing, same output, bit for bit
    i2, w2 = layer.route(x)
    y2 = layer.forward(x, i2, w2)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(w, w2)
    assert torch.equal(y.view(torch.int16) if y.dtype == torch.bfloat16 else y,
                       y2.view(torch.int16) if y2.dtype == torch.bfloat16 else y2)


def test_layer_forward_full_decode_shape():
    prob = synth.make_problem(2)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    y, idx, w = layer.layer(x)
    torch.cuda.synchronize()
    judge(prob, y, idx, w, logits=gpu_logits(layer, x))


def test_decode_router_mask_equals_slice():
    """The decode logits kernel keeps masking experts equal to slicing them, bit for bit."""
    prob = synth.make_problem(5, T=32, H=256, E=48, I=128, n_active=29, bias=("skew", 0.2))
    act = np.nonzero(prob.mask)[0]
    sl = synth.Problem(cfg=prob.cfg, T=prob.T, H=prob.H, I=prob.I, E=len(act), k=prob.k, router=prob.router,
                       scale=prob.scale, wfmt=prob.wfmt, xfmt=prob.xfmt, x=prob.x,
                       W_r=np.ascontiguousarray(prob.W_r[act]), b=np.ascontiguousarray(prob.b[act]), mask=None,
                       W_gate=np.ascontiguousarray(prob.W_gate[act]), W_up=np.ascontiguousarray(prob.W_up[act]),
                       W_down=np.ascontiguousarray(prob.W_down[act]), s_gate=np.ascontiguousarray(prob.s_gate[act]),
                       s_up=np.ascontiguousarray(prob.s_up[act]), s_down=np.ascontiguousarray(prob.s_down[act]))
    y1, i1, w1 = layer_from_problem(prob).layer(x_to_device(prob))
    y2, i2, w2 = layer_from_problem(sl).layer(x_to_device(sl))
    torch.cuda.synchronize()
    assert np.array_equal(act[i2.cpu().numpy()], i1.cpu().numpy())
    assert torch.equal(w1, w2)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_layer_forward_launches_fewer_kernels_at_decode():
    prob = synth.make_problem(2, T=32, H=256, E=64, I=128)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    layer.layer(x)
    n0 = moe.moe_launch_count()
    layer.layer(x)
    fused = moe.moe_launch_count() - n0
    n0 = moe.moe_launch_count()
    layer(x)
    separate = moe.moe_launch_count() - n0
    assert fused == separate - 1  # top-k and sort share one launch


EDGE = {
    "max-H-decode": (2, dict(T=32, H=8192, E=16, I=64)),       # decode logits split 8 ways (213 KB of smem)
    "max-E-decode": (2, dict(T=24, H=256, E=1024, I=64)),      # E > 256: route and forward, not the fused router
    "max-k-decode": (2, dict(T=32, H=256, E=64, I=64, k=32)),  # 1024 pairs through the fused router's sort
    "max-I-decode": (2, dict(T=8, H=256, E=8, I=8192)),
    "k1-decode": (3, dict(T=17, H=256, E=24, I=128, k=1)),
    "k-equals-active": (5, dict(T=12, H=256, E=32, I=128, n_active=8, bias=("skew", 0.1))),
    "fp32-H64": (1, dict(T=5, H=64, E=8, k=2, I=64)),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_layer_forward_edge_shapes(name):
    cid, over = EDGE[name]
    prob = synth.make_problem(cid, **over)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    y, idx, w = layer.layer(x)
    torch.cuda.synchronize()
    judge(prob, y, idx, w, logits=gpu_logits(layer, x))
    if prob.mask is not None:
        assert prob.mask[idx.cpu().numpy()].all()


def test_zero_tokens_is_a_no_op_on_every_entry_point():
    prob = synth.make_problem(2, T=4, H=256, E=16, I=128, shared=128, residual=True)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)[:0]
    idx = torch.empty((0, prob.k), dtype=torch.int32, device="cuda")
    w = torch.empty((0, prob.k), dtype=torch.float32, device="cuda")
    y = torch.empty((0, prob.H), dtype=torch.bfloat16, device="cuda")
    n0 = moe.moe_launch_count()
    ws = layer.workspace(1)
    moe.moe_layer_forward(layer.desc, x.data_ptr() or 256, 0, idx.data_ptr() or 256, w.data_ptr() or 256,
                          y.data_ptr() or 256, ws.data_ptr(), ws.numel())
    moe.moe_forward_block(layer.desc, layer.shared, x.data_ptr() or 256, 0, idx.data_ptr() or 256,
                          w.data_ptr() or 256, None, y.data_ptr() or 256, ws.data_ptr(), ws.numel())
    counts = torch.zeros(prob.E, dtype=torch.uint64, device="cuda")
    moe.moe_expert_counts(layer.desc, idx.data_ptr() or 256, 0, counts.data_ptr())
    torch.cuda.synchronize()
    assert moe.moe_launch_count() == n0
    assert int(counts.sum()) == 0


@pytest.mark.parametrize("cid,over", [(2, {}), (3, dict(T=600, H=256, E=32, I=256))])
def test_layer_replays_from_a_cuda_graph(cid, over):
    """One moe_layer_forward call captured into a CUDA graph (no allocation, no
    host synchronisation inside the call) replays to the same bits as a direct
    call, and stays correct for new inputs written into the captured buffer."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    prob = synth.make_problem(cid, **over)
    layer = layer_from_problem(prob)
    x = x_to_device(prob)
    y_ref, i_ref, w_ref = layer.layer(x)  # warm-up: device state, workspace, tensor maps
    torch.cuda.synchronize()
    xs = x.clone()
    y = torch.empty_like(y_ref)
    idx = torch.empty_like(i_ref)
    w = torch.empty_like(w_ref)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.layer(xs, out=(y, idx, w))
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx, i_ref) and torch.equal(w, w_ref)
    assert torch.equal(y.view(torch.int16) if y.dtype == torch.bfloat16 else y,
                       y_ref.view(torch.int16) if y_ref.dtype == torch.bfloat16 else y_ref)
    # new tokens in the captured input buffer: the replay routes and computes them
    x2 = torch.roll(x, shifts=1, dims=0)
    xs.copy_(x2)
    g.replay()
    y2, i2, w2 = layer.layer(x2)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(w, w2)
    assert torch.equal(y.view(torch.int16) if y.dtype == torch.bfloat16 else y,
                       y2.view(torch.int16) if y2.dtype == torch.bfloat16 else y2)
    assert moe.moe_device_flags(clear=True) == 0


def test_programmatic_launch_does_not_change_results(tmp_path):
    """The same layer calls with programmatic dependent launch (opt-in, MOE_PDL=1,
    read once per process, so in a child process) and with plain stream ordering
    (the default) give the same bits."""
    import os
    import subprocess
    import sys
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    here = os.path.dirname(os.path.abspath(__file__))
    script = tmp_path / "run_layer.py"
    script.write_text(
        "import sys, numpy as np, torch\n"
        f"sys.path[:0] = [{os.path.dirname(here)!r}, {here!r}]\n"
        "import synth\n"
        "from gpu_util import layer_from_problem, x_to_device\n"
        "out = {}\n"
        "for cid, over in ((2, {}), (3, dict(T=300, H=256, E=16, I=128)), (4, dict(T=150, H=256, E=16, I=128))):\n"
        "    prob = synth.make_problem(cid, **over)\n"
        "    layer = layer_from_problem(prob)\n"
        "    y, idx, w = layer.layer(x_to_device(prob))\n"
        "    torch.cuda.synchronize()\n"
        "    out[f'y{cid}'] = y.view(torch.int16).cpu().numpy() if y.dtype == torch.bfloat16 else y.cpu().numpy()\n"
        "    out[f'i{cid}'] = idx.cpu().numpy()\n"
        "    out[f'w{cid}'] = w.cpu().numpy()\n"
        "np.savez(sys.argv[1], **out)\n")
    runs = {}
    for pdl in ("1", "0"):
        dst = tmp_path / f"out_{pdl}.npz"
        env = dict(os.environ, MOE_PDL=pdl)
        subprocess.run([sys.executable, str(script), str(dst)], check=True, env=env, timeout=600)
        runs[pdl] = np.load(dst)
    for key in runs["1"].files:
        assert np.array_equal(runs["1"][key], runs["0"][key]), key
