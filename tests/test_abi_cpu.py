"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe.h declares, and rejects bad arguments with the
documented status before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import mixture_experts_layer_31_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt)
    return names


def test_library_exports_every_declared_symbol():
    names = declared_entry_points()
    assert set(moe.EXPORTS) <= set(names)
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def _desc(**kw):
    d = moe.moe_desc()
    d.H, d.I, d.E, d.k = 256, 128, 16, 4
    d.router, d.act, d.wfmt, d.xfmt, d.path, d.scale = 0, 0, moe.MOE_W_BF16, moe.MOE_X_BF16, 0, 2.446
    fake = 1 << 20  # never dereferenced: validation and sizing only
    d.W_r = d.W_gate = d.W_up = d.W_down = fake
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_grows_with_tokens():
    a = moe.moe_workspace_size(_desc(), 16)
    b = moe.moe_workspace_size(_desc(), 1024)
    assert 0 < a < b and a % 256 == 0


@pytest.mark.parametrize("field,value,status", [
    ("H", 100, moe.MOE_ERR_INVALID_ARG),
    ("I", 0, moe.MOE_ERR_INVALID_ARG),
    ("k", 17, moe.MOE_ERR_INVALID_ARG),
    ("k", 33, moe.MOE_ERR_INVALID_ARG),
    ("E", 2048, moe.MOE_ERR_UNSUPPORTED),
    ("act", 7, moe.MOE_ERR_INVALID_ARG),
    ("router", 5, moe.MOE_ERR_INVALID_ARG),
    ("wfmt", 9, moe.MOE_ERR_INVALID_ARG),
    ("W_r", None, moe.MOE_ERR_INVALID_ARG),
    ("W_gate", (1 << 20) + 4, moe.MOE_ERR_INVALID_ARG),
    ("wfmt", moe.MOE_W_INT8_ROW, moe.MOE_ERR_INVALID_ARG),  # int8 without scales
    ("wfmt", moe.MOE_W_INT4_B128, moe.MOE_ERR_INVALID_ARG),  # block 128 needs I % 128 (I = 192 below)
])
def test_invalid_descriptors_are_rejected(field, value, status):
    extra = dict(I=192, s_gate=1 << 20, s_up=1 << 20, s_down=1 << 20) if value == moe.MOE_W_INT4_B128 else {}
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_workspace_size(_desc(**{field: value}, **extra), 16)
    assert ei.value.status == status
    assert moe.moe_last_error()


def test_both_activations_and_int4_formats_are_accepted():
    for act in (moe.MOE_ACT_SILU, moe.MOE_ACT_GELU_TANH):
        assert moe.moe_workspace_size(_desc(act=act), 16) > 0
    sc = dict(s_gate=1 << 20, s_up=1 << 20, s_down=1 << 20)
    for wfmt in (moe.MOE_W_INT4_B32, moe.MOE_W_INT4_B128):
        assert moe.moe_workspace_size(_desc(wfmt=wfmt, **sc), 16) > 0


def test_route_and_forward_validate_before_launch():
    d = _desc()
    with pytest.raises(moe.MoeError) as ei:  # NULL x
        moe.moe_route(d, None, 16, 1 << 20, 1 << 20, 1 << 20, 1 << 30)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # workspace too small
        moe.moe_route(d, 1 << 20, 16, 1 << 20, 1 << 20, 1 << 20, 256)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoeError) as ei:  # misaligned workspace
        moe.moe_forward(d, 1 << 20, 16, 1 << 20, 1 << 20, 1 << 20, (1 << 20) + 64, 1 << 30)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoeError) as ei:  # negative T
        moe.moe_forward(d, 1 << 20, -1, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 30)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # NULL logits
        moe.moe_route_logits(d, 1 << 20, 16, None, 1 << 20, 1 << 30)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # workspace too small for the router's partial logits
        moe.moe_route_logits(d, 1 << 20, 16, 1 << 20, 1 << 20, 256)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    # T = 0 is a valid no-op that launches nothing
    n = moe.moe_launch_count()
    moe.moe_route_logits(d, 1 << 20, 0, None, None, 0)
    moe.moe_route(d, 1 << 20, 0, 1 << 20, 1 << 20, None, 0)
    moe.moe_forward(d, 1 << 20, 0, 1 << 20, 1 << 20, 1 << 20, None, 0)
    assert moe.moe_launch_count() == n


def test_header_declares_citations_and_ownership():
    txt = open(os.path.join(ROOT, "include", "moe.h")).read()
    for needle in ("Conversion notes", "Defrag", "owned by the caller", "MOE_ERR_UNSUPPORTED"):
        assert needle in txt


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("cover", [0.3, 0.95, 1.0])
def test_cover_set_matches_oracle(seed, cover):
    """The library's host cover-set utility against the oracle's, bit for bit
    (host-only: no device work)."""
    import oracle
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 300))
    counts = rng.integers(0, 50, size=E).astype(np.uint64)
    counts[rng.random(E) < 0.3] = 0
    counts[: E // 4] = counts[0]  # ties
    got = moe.moe_cover_set(counts, cover)
    ref = oracle.cover_set(counts, cover)
    assert got[2] == ref[2]
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[1], ref[1])


def test_cover_set_rejects_bad_arguments():
    for cover in (0.0, -1.0, 1.01, float("nan")):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_cover_set(np.ones(4, np.uint64), cover)
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG


def test_expert_counts_validates_before_launch():
    with pytest.raises(moe.MoeError) as ei:  # NULL counts
        moe.moe_expert_counts(_desc(), 1 << 20, 16, None)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    moe.moe_expert_counts(_desc(), 1 << 20, 0, 1 << 20)  # T = 0: nothing to count, nothing launched


def test_block_workspace_covers_the_shared_expert():
    d = _desc()
    sh = moe.moe_shared_expert()
    sh.I, sh.wfmt = 256, moe.MOE_W_BF16
    sh.W_gate = sh.W_up = sh.W_down = 1 << 20
    plain = moe.moe_workspace_size(d, 64)
    assert moe.moe_block_workspace_size(d, None, 64) == plain
    assert moe.moe_block_workspace_size(d, sh, 64) > plain
    sh.I = 96
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_block_workspace_size(d, sh, 64)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    sh.I, sh.wfmt = 256, moe.MOE_W_INT8_ROW  # int8 without scales
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_block_workspace_size(d, sh, 64)
    assert "shared expert" in str(ei.value)


def test_stage_timing_filter_validates_the_name():
    """Restricting the per-kernel timing to one kernel name needs no device;
    names longer than the stage-name field are rejected."""
    moe.moe_stage_timing_only("gemm_gateup")
    moe.moe_stage_timing_only(None)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_stage_timing_only("x" * 40)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
