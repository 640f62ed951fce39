"""The fused GEMM's work plans, checked on the host (no GPU): the plan a
launch would run is rebuilt from the shapes alone and decoded back.

Every tile's K range must be covered exactly once, by pieces in order; the
pairs' loads must be balanced; launches with fewer tiles than CTA pairs
(a decoder's lone o projection, its q/k/v group) take the stream-K plan,
layer-grouped launches the longest-first one.
"""
import pytest

from host_streamed_nf4_b200 import hsnf4, synth


def _proj(family):
    return {name: (n, k) for name, n, k in synth.FAMILIES[family].projections()}


def _groups(family):
    p = _proj(family)
    return {
        "layer": [p[x] for x in synth.PROJ_NAMES],
        "qkv": [p["q"], p["k"], p["v"]],
        "o": [p["o"]],
        "gate_up": [p["gate"], p["up"]],
        "down": [p["down"]],
    }


@pytest.mark.parametrize("family", ["qwen2.5-7b", "qwen2.5-72b", "llama-3.1-8b"])
@pytest.mark.parametrize("mode", ["fwd", "dx"])
@pytest.mark.parametrize("T", [512, 256, 100, 2048])
def test_plans_cover_every_tile_once_and_balance(family, mode, T):
    for name, shapes in _groups(family).items():
        info = hsnf4.gemm_plan(mode, shapes, T, 16)
        assert info["covered"] == 1, (family, mode, T, name, info)
        contraction = [(k if mode == "fwd" else n) // 64 for n, k in shapes]
        rows = [(n if mode == "fwd" else k) for n, k in shapes]
        t_tiles = -(-T // (512 if T > 256 else -(-T // 16) * 16))
        steps = sum(-(-m // 256) * t_tiles * c for m, c in zip(rows, contraction))
        assert info["total_steps"] == steps
        mean = steps / info["pairs"]
        if info["stream_k"]:  # equal shares, give or take the shortest piece
            assert info["max_pair_steps"] <= 1.35 * mean + 16, (name, info)


def test_plan_kinds_on_the_benchmarked_shapes():
    g = _groups("qwen2.5-72b")
    assert hsnf4.gemm_plan("fwd", g["layer"], 512, 16)["stream_k"] == 0
    assert hsnf4.gemm_plan("dx", g["layer"], 512, 16)["stream_k"] == 0
    assert hsnf4.gemm_plan("fwd", g["qkv"], 512, 16)["stream_k"] == 1
    assert hsnf4.gemm_plan("fwd", g["gate_up"], 512, 16)["stream_k"] == 1
    g7 = _groups("qwen2.5-7b")
    info = hsnf4.gemm_plan("fwd", g7["o"], 512, 16)  # 14 tiles for 74 pairs
    assert info["stream_k"] == 1 and info["split_tiles"] == 14 and info["pairs"] == 74


@pytest.mark.parametrize("family", ["qwen2.5-7b", "qwen2.5-72b", "llama-3.1-8b"])
@pytest.mark.parametrize("mode", ["fwd", "dx"])
def test_split_tiles_are_added_in_kernel_only_with_cover(family, mode):
    """A split tile's pieces are added by its last piece inside the kernel
    only where every piece has later work (or idle time) in its pair: all
    of them in the layer-grouped launches, whose pieces are the longest
    units and run first; none in launches with no more units than pairs,
    where every piece ends its pair's work."""
    g = _groups(family)
    for name, shapes in g.items():
        for T in (512, 100):
            info = hsnf4.gemm_plan(mode, shapes, T, 16)
            assert 0 <= info["fixup_tiles"] <= info["split_tiles"], (name, T, info)
            if info["units"] <= info["pairs"]:
                assert info["fixup_tiles"] == 0, (name, T, info)
    info = hsnf4.gemm_plan(mode, g["layer"], 512, 16)
    assert info["fixup_tiles"] == info["split_tiles"], info


def test_plan_rejects_bad_shapes():
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.gemm_plan("fwd", [(100, 512)], 512, 16)
    with pytest.raises(hsnf4.HsNf4Error):
        hsnf4.gemm_plan("fwd", [(512, 512)], 512, 0)


def _check_plan(mode, shapes, T, r):
    """Every plan the launch would run covers each tile's K range once, in
    order; its step count is the problem's; split tiles added in the kernel
    are a subset of the split tiles.  (A launch with fewer tiles than CTA
    pairs leaves some pairs without work; they exit at once.)"""
    info = hsnf4.gemm_plan(mode, shapes, T, r)
    assert info["covered"] == 1, (mode, shapes, T, r, info)
    contraction = [(k if mode == "fwd" else n) // 64 for n, k in shapes]
    rows = [(n if mode == "fwd" else k) for n, k in shapes]
    t_tiles = -(-T // (512 if T > 256 else -(-T // 16) * 16))
    steps = sum(-(-m // 256) * t_tiles * c for m, c in zip(rows, contraction))
    assert info["total_steps"] == steps, (mode, shapes, T, info)
    assert info["units"] >= 1 and info["max_pair_steps"] >= -(-steps // info["pairs"]), info
    assert 0 <= info["fixup_tiles"] <= info["split_tiles"], info
    return info


def test_plans_hold_on_random_groups():
    """Random groups of 1-8 problems (dimensions multiples of 64 up to
    32768), random T and ranks: every plan is valid, or the launch refuses
    it with an error (never a wrong plan)."""
    hypothesis = pytest.importorskip("hypothesis")
    st = hypothesis.strategies
    dim = st.integers(1, 512).map(lambda x: 64 * x)

    @hypothesis.settings(max_examples=400, deadline=None, derandomize=True)
    @hypothesis.given(mode=st.sampled_from(["fwd", "dx"]),
                      shapes=st.lists(st.tuples(dim, dim), min_size=1, max_size=8),
                      T=st.integers(1, 4096), r=st.sampled_from([8, 16, 32, 64]))
    def run(mode, shapes, T, r):
        try:
            _check_plan(mode, shapes, T, r)
        except hsnf4.HsNf4Error as e:  # refused: too many units or tiles for one launch
            assert e.status == 1, e

    run()
