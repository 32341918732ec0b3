"""GPU tests of the routing statistics: per-expert counts accumulated across
calls, and the Calibrate -> Defrag flow of the CMF code specialist page (How it
was made): record routing frequencies, keep the smallest expert set covering
95% of the mass, and run the layer masked (equal, bit for bit, to the sliced
layer)."""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import oracle
import synth
from gpu_util import run, x_to_device, layer_from_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    moe.moe_device_flags(clear=True)
    yield
    assert moe.moe_device_flags(clear=True) == 0


def test_counts_accumulate_and_match_oracle():
    prob = synth.make_problem(5, T=700, H=256, E=48, I=128, n_active=30, bias=("skew", 0.2))
    layer = layer_from_problem(prob)
    counts = torch.zeros(prob.E, dtype=torch.uint64, device="cuda")
    ref = np.zeros(prob.E, np.uint64)
    for rep in range(3):
        p = synth.make_problem(5, replica=rep, T=700, H=256, E=48, I=128, n_active=30, bias=("skew", 0.2))
        idx, _ = layer.route(x_to_device(p))
        layer.expert_counts(idx, counts)
        oracle.expert_counts(idx.cpu().numpy(), prob.E, counts=ref)
    got = counts.cpu().numpy().astype(np.uint64)
    np.testing.assert_array_equal(got, ref)
    assert got.sum() == 3 * 700 * prob.k
    assert got[prob.mask == 0].sum() == 0


def test_counts_skip_out_of_range_entries_and_ragged_sizes():
    E = 40
    layer = layer_from_problem(synth.make_problem(2, T=4, H=256, E=E, I=128))
    rng = np.random.default_rng(3)
    for T in (1, 3, 257, 5003):  # ragged: T*k not a multiple of the vector width
        idx_np = rng.integers(-2, E + 2, size=(T, 8)).astype(np.int32)
        counts = torch.zeros(E, dtype=torch.uint64, device="cuda")
        layer.expert_counts(torch.from_numpy(idx_np).cuda(), counts)
        np.testing.assert_array_equal(counts.cpu().numpy().astype(np.uint64), oracle.expert_counts(idx_np, E))


def test_counts_full_skewed_workload():
    prob = synth.make_problem(5)
    layer = layer_from_problem(prob)
    idx, _ = layer.route(x_to_device(prob))
    counts = layer.expert_counts(idx)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.uint64),
                                  oracle.expert_counts(idx.cpu().numpy(), prob.E))


def test_calibrate_then_defrag_flow():
    """Counts over calibration batches -> 95% cover set -> mask; the masked layer
    selects only kept experts and equals the sliced (renumbered) layer bit for bit."""
    base = dict(T=600, H=256, E=64, I=128, bias=("skew", 0.3), n_active=None)
    full = synth.make_problem(5, **base)
    layer = layer_from_problem(full)
    counts = torch.zeros(full.E, dtype=torch.uint64, device="cuda")
    for rep in range(2):
        idx, _ = layer.route(x_to_device(synth.make_problem(5, replica=rep, **base)))
        layer.expert_counts(idx, counts)
    keep, new_index, n = moe.moe_cover_set(counts.cpu().numpy(), 0.95)
    ref = oracle.cover_set(counts.cpu().numpy().astype(np.uint64), 0.95)
    assert n == ref[2] and np.array_equal(keep, ref[0]) and np.array_equal(new_index, ref[1])
    assert full.k <= n < full.E
    kept = np.nonzero(keep)[0]
    assert np.array_equal(new_index[kept], np.arange(n))
    test = synth.make_problem(5, replica=7, **base)
    masked = dataclasses.replace(test, mask=keep.astype(np.uint8))
    sl = dataclasses.replace(test, E=n, mask=None, W_r=np.ascontiguousarray(test.W_r[kept]),
                             b=np.ascontiguousarray(test.b[kept]),
                             W_gate=np.ascontiguousarray(test.W_gate[kept]),
                             W_up=np.ascontiguousarray(test.W_up[kept]),
                             W_down=np.ascontiguousarray(test.W_down[kept]),
                             s_gate=np.ascontiguousarray(test.s_gate[kept]),
                             s_up=np.ascontiguousarray(test.s_up[kept]),
                             s_down=np.ascontiguousarray(test.s_down[kept]))
    _, _, y1, i1, w1 = run(masked)
    _, _, y2, i2, w2 = run(sl)
    assert keep[i1.cpu().numpy()].all()
    assert np.array_equal(kept[i2.cpu().numpy()], i1.cpu().numpy())
    assert torch.equal(w1, w2)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
