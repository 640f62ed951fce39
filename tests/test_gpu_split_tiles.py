"""The fused GEMM's K-split tiles that are added inside the kernel.

In a longest-first plan every piece of a split tile writes its fp32 rows
to the workspace and counts itself on the tile's arrival word; the piece
that completes the count adds the pieces in split order and writes the
output.  The result must not depend on which piece finishes last, on what
the workspace held before the call (each launch tags its arrival words
with a fresh token; a word holding anything else counts as empty), or on
earlier calls (a completed launch leaves its words 0).  The grouped
forward and dX launches of a Qwen2.5-7B layer (T = 512, and a ragged 100)
and of a Llama-3.1-8B layer (T = 256) are such plans: every split tile of
both is added in the kernel.
"""
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.stack import LayerStack

pytestmark = pytest.mark.gpu


def _outputs(stack):
    stack.step()
    torch.cuda.synchronize()
    return [t.clone() for t in list(stack.Y) + list(stack.dX) + list(stack.t[0]) +
            list(stack.dA[0]) + list(stack.dB[0])]


@pytest.mark.parametrize("family,T", [("qwen2.5-7b", 512), ("qwen2.5-7b", 100),
                                      ("llama-3.1-8b", 256)])
def test_in_kernel_split_adds_are_repeatable_whatever_the_workspace_held(family, T):
    fam = synth.FAMILIES[family]
    shapes = [(n, k) for _, n, k in fam.projections()]
    for mode in ("fwd", "dx"):
        info = hsnf4.gemm_plan(mode, shapes, T, 16)
        assert info["split_tiles"] > 0 and info["fixup_tiles"] == info["split_tiles"], info
    s = LayerStack(fam, 1, T, block_size=1, streamed=False)
    try:
        ref = _outputs(s)
        for fill in ("as left", "random", "ones", "zeros", "as left"):
            if fill == "random":
                s.ws_f.random_(0, 256)
                s.ws_b.random_(0, 256)
            elif fill == "ones":
                s.ws_f.fill_(255)
                s.ws_b.fill_(255)
            elif fill == "zeros":
                s.ws_f.zero_()
                s.ws_b.zero_()
            got = _outputs(s)
            for a, b in zip(ref, got):
                assert torch.equal(a, b), fill
        assert hsnf4.device_status() == 0
    finally:
        s.close()
