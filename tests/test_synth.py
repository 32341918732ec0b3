"""The seeded input generator: determinism, distributions, encoders, and the
skewed workload's realised routing share (measured with the oracle router)."""
import json
import os

import numpy as np
import pytest

import oracle
import synth


def test_counter_streams_independent_of_thread_count():
    a = synth.normal_f32((1001, 37), 9, 4, 0.0, 1.0, nthreads=1)
    b = synth.normal_f32((1001, 37), 9, 4, 0.0, 1.0, nthreads=7)
    assert np.array_equal(a, b)
    q1, s1 = synth.int8_rows(300, 64, 9, 5, 0.02, nthreads=1)
    q2, s2 = synth.int8_rows(300, 64, 9, 5, 0.02, nthreads=5)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)
    assert not np.array_equal(a, synth.normal_f32((1001, 37), 9, 5, 0.0, 1.0))
    assert not np.array_equal(a, synth.normal_f32((1001, 37), 10, 4, 0.0, 1.0))


def test_splitmix64_output_function():
    """The stream is SplitMix64's output function over a Weyl sequence: check the
    published reference outputs for seed state 0 (Vigna's splitmix64.c)."""
    def mix(z):
        M = (1 << 64) - 1
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)
    M, G = (1 << 64) - 1, 0x9E3779B97F4A7C15
    assert mix(G) == 0xE220A8397B1DCDAF
    assert mix((2 * G) & M) == 0x6E789E6AA1B965F4
    # the C stream is that function over key + (i + 1) * gamma
    lib = synth._load()
    key = mix(mix((123 + G) & M) ^ ((7 * 0xD1B54A32D192ED03) & M))
    for i in (0, 1, 2, 1000, 2**40):
        assert lib.synth_draw_u64(123, 7, i) == mix((key + (i + 1) * G) & M)


def test_normal_moments_and_bf16_rounding():
    z = synth.normal_f32((400000,), 3, 1)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    bits = synth.normal_bf16((4096,), 3, 1)
    f = synth.bf16_bits_to_f32(bits)
    ref = synth.normal_f32((4096,), 3, 1)
    assert np.all(np.abs(f - ref) <= np.abs(ref) * 2.0 ** -8)


def test_int4_encoder_range_and_clamp():
    q, s = synth.int4_blocks(64, 128, 1, 2, 1e-7)  # tiny weights: every scale clamps
    assert np.all(s == np.float32(2.0 ** -14))
    q, s = synth.int4_blocks(64, 128, 1, 2, 0.02)
    nib = np.concatenate([(q & 0xF), (q >> 4)]).astype(int)
    v = np.where(nib >= 8, nib - 16, nib)
    assert v.min() >= -8 and v.max() <= 7 and (s >= 2.0 ** -14).all()


def test_workload_shapes():
    for cid, c in synth.CONFIGS.items():
        assert c["k"] == 8 or cid == 1
    p = synth.make_problem(4, T=8, H=64, I=64, E=8)
    assert p.W_gate.shape == (8, 64, 32) and p.s_gate.shape == (8, 64, 2)
    assert p.W_down.shape == (8, 64, 32) and p.s_down.shape == (8, 64, 2)
    assert p.b is None and p.router == "softmax"
    m = synth.active_mask(synth.config(5))
    assert m.sum() == 160 and m.size == 256


def test_skewed_workload_share_on_token_sample():
    """The 64 highest-bias active experts take ~73% of selections (CMF page,
    Calibrate step); re-measured with the oracle router on 512 sampled tokens."""
    cal = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "skew_calibration.json")))
    assert cal["c"] == synth.SKEW_C and abs(cal["realised_top64_share"] - 0.73) <= 0.01
    cfg = synth.config(5)
    H, E, T = cfg["H"], cfg["E"], cfg["T"]
    prob = synth.make_problem(5, I=64)   # router inputs identical to the full workload
    rng = np.random.default_rng(0)
    toks = np.sort(rng.choice(T, 512, replace=False))
    idx, _, _ = oracle.Oracle(prob).route(toks)
    ranks = synth.skew_ranks(prob.cfg, prob.mask)
    top = np.nonzero((ranks >= 0) & (ranks < 64))[0]
    share = np.isin(idx, top).mean()
    assert abs(share - 0.73) < 0.03
    assert prob.mask[idx].all()
