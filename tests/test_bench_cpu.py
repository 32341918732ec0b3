"""CPU checks of bench.py's host-side accounting: the algorithmic bytes and flops
behind every roofline fraction, and the guard on committed DRAM-traffic figures.

The expected values are recomputed here from the problem's own arrays (weight and
scale bytes per expert, tokens, pairs), not from bench.py's helpers."""
import hashlib
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _routing(prob, seed=0):
    """A valid routing: k distinct experts per token, some experts left untouched."""
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(prob.E // 2, prob.k, replace=False) for _ in range(prob.T)]).astype(np.int32)
    return idx


def _nbytes(*arrays):
    return sum(0 if a is None else int(a.nbytes) for a in arrays)


@pytest.mark.parametrize("cid,over", [
    (2, dict(T=24, H=256, E=16, I=128)),                      # bf16 weights
    (3, dict(T=40, H=256, E=16, I=128)),                      # int8 rows with row scales
    (4, dict(T=33, H=256, E=16, I=128)),                      # int4 block 32 with block scales
])
def test_algorithmic_bytes_and_flops(cid, over):
    prob = synth.make_problem(cid, **over)
    idx = _routing(prob)
    acc = bench.algorithmic(prob, idx, "gemm")
    T, H, I, E, k = prob.T, prob.H, prob.I, prob.E, prob.k
    P = T * k
    touched = len(set(idx.ravel().tolist()))
    assert acc["touched"] == touched == bench.touched_experts(idx, E)
    xb = 2 if prob.xfmt == "bf16" else 4
    gate_up = (_nbytes(prob.W_gate, prob.s_gate) + _nbytes(prob.W_up, prob.s_up)) // E
    down = _nbytes(prob.W_down, prob.s_down) // E
    # the method's own bytes: touched experts' weights and scales, x once (gate/up), y once (down)
    assert acc["bytes"]["gemm_gateup"] == touched * gate_up + T * H * xb
    assert acc["bytes"]["gemm_down"] == touched * down + T * H * xb
    assert acc["flops"]["gemm_gateup"] == 4.0 * P * H * I
    assert acc["flops"]["gemm_down"] == 2.0 * P * H * I
    assert acc["layer_flops"] == 6.0 * P * H * I + 2.0 * T * H * E
    assert acc["layer_bytes"] == touched * (gate_up + down) + prob.W_r.nbytes + 2 * T * H * xb
    # the design's intermediates are kept apart: on the tensor-core path the token rows
    # gathered in expert order (written, then read) and h; the GEMV path reads x itself
    h = P * I * 2
    assert acc["overhead"]["gemm_gateup"] == 2 * P * H * 2 + h
    assert bench.algorithmic(prob, idx, "gemv")["overhead"]["gemv_gateup"] == h


def test_untouched_and_invalid_indices_do_not_count():
    prob = synth.make_problem(3, T=8, H=256, E=16, I=128)
    idx = np.full((prob.T, prob.k), 3, np.int32)
    idx[0, :] = np.arange(prob.k)
    idx[1, 0] = -1            # an empty slot
    idx[2, 0] = prob.E + 5    # out of range: flagged by the library, not counted here
    assert bench.touched_experts(idx, prob.E) == len(set(range(prob.k)) | {3})


def _fake_root(tmp_path, src_text, entry_sha):
    """A copy of the repository layout that known_traffic reads: the kernel source and
    profiles/ncu_traffic.json pointing at a given sha."""
    src_rel = "mixture_experts_layer_31_b200/csrc/gemm_tc.cu"
    (tmp_path / "mixture_experts_layer_31_b200" / "csrc").mkdir(parents=True)
    (tmp_path / src_rel).write_text(src_text)
    (tmp_path / "profiles").mkdir()
    entry = {"dram_bytes_per_launch": 123456789, "source": src_rel, "source_sha256": entry_sha, "how": "test"}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"gemm_gateup": {"wl": entry}}))
    return str(tmp_path)


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    text = "// kernel source as captured\n"
    sha = hashlib.sha256(text.encode()).hexdigest()
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path, text, sha))
    assert bench.known_traffic("gemm_gateup", "wl") == 123456789
    assert bench.known_traffic("gemm_gateup", "other-workload") is None
    assert bench.known_traffic("gemm_down", "wl") is None
    # any change to the source since the capture voids the figure
    (tmp_path / "mixture_experts_layer_31_b200" / "csrc" / "gemm_tc.cu").write_text(text + "// edited\n")
    assert bench.known_traffic("gemm_gateup", "wl") is None


def test_committed_traffic_entries_match_the_current_kernel_source():
    """The committed figures are live (not null in the bench line) only while the
    kernel source is the captured one; every entry names the same file and sha."""
    d = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    src = os.path.join(ROOT, "mixture_experts_layer_31_b200", "csrc", "gemm_tc.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    for kernel, per in d.items():
        for workload, ent in per.items():
            assert ent["source_sha256"] == sha, (kernel, workload)
            assert ent["dram_bytes_per_launch"] > 0
            assert bench.known_traffic(kernel, workload) == ent["dram_bytes_per_launch"]
