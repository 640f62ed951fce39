"""lora_linear_fwd_noalloc: the LoRA forward for callers that cannot
allocate device memory (a runtime that reserves its whole device-memory
budget up front and forbids later allocations, a plugin or callback that may
not call the allocator).  It runs the same kernels and the same plan as
lora_linear_fwd on the library's built-in scratch instead of a caller
workspace, so its results must equal lora_linear_fwd's bit for bit, call
after call, although every call reuses (and leaves behind) the same scratch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from gpu_util import assert_lora_close, bf16_to_f64, oracle_nf4_weight, to_dev_bf16

SHAPES = [  # T, N, K: the single-linear case, a ragged case, a K-split case
    (64, 512, 512),
    (300, 192, 320),
    (512, 3584, 3584),
]
ROWS = np.array([0, 1, 63, 64, 255, 256, 299, 300, 511])


def _inputs(orc, T, N, K):
    case = synth.linear_case(9100 + T + N, T, N, K)
    W = oracle_nf4_weight(orc, case.W)
    X, A, B = (to_dev_bf16(a) for a in (case.X, case.A, case.B))
    return case, W, X, A, B


@pytest.mark.gpu
@pytest.mark.parametrize("T,N,K", SHAPES)
def test_noalloc_forward_equals_workspace_forward_twice(orc, T, N, K):
    case, W, X, A, B = _inputs(orc, T, N, K)
    Y_ref, t_ref = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
    torch.cuda.synchronize()
    for _ in range(2):  # the second call starts from the first call's leftovers
        Y, t = hsnf4.lora_linear_fwd_noalloc(W, X, A, B, case.alpha)
        torch.cuda.synchronize()
        assert hsnf4.device_status() == 0
        assert torch.equal(Y, Y_ref), f"noalloc Y {T}x{N}x{K}"
        assert torch.equal(t, t_ref), f"noalloc t {T}x{N}x{K}"
    # and once against the oracle, within the LoRA bar
    rows = ROWS[ROWS < T]
    Yr, tr = orc.lora_fwd(W.codes.cpu().numpy(), W.absmax.cpu().numpy(), N, K, case.X, case.A,
                          case.B, case.alpha, rows=rows)
    assert_lora_close(bf16_to_f64(Y)[rows], Yr, f"noalloc Y vs oracle {T}x{N}x{K}")
    assert_lora_close(t.cpu().numpy(), tr, f"noalloc t vs oracle {T}x{N}x{K}")


@pytest.mark.gpu
def test_noalloc_after_a_larger_call_with_another_plan(orc):
    """A call on scratch left behind by a larger shape with a K-split plan
    (partial tiles everywhere) still equals the workspace forward bitwise."""
    big = _inputs(orc, 512, 3584, 3584)
    small = _inputs(orc, 300, 192, 320)
    Y_ref, t_ref = hsnf4.lora_linear_fwd(*small[1:], small[0].alpha)
    hsnf4.lora_linear_fwd_noalloc(*big[1:], big[0].alpha)
    Y, t = hsnf4.lora_linear_fwd_noalloc(*small[1:], small[0].alpha)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    assert torch.equal(Y, Y_ref) and torch.equal(t, t_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked from the shapes alone: the call fails before touching memory."""
    L = hsnf4.lib()
    fake = 0x10000
    # a 128 x 131072 weight at 32768 tokens: few, very long tiles, so the GEMM
    # splits the contraction and its fp32 partial tiles need ~259 MiB
    assert L.lora_linear_fwd_workspace(32768, 128, 131072, 16) > 64 << 20
    W = hsnf4.Nf4WeightC(fake, fake, 128, 131072)
    rc = L.lora_linear_fwd_noalloc(ctypes.byref(W), fake, 32768, fake, fake, 16, 32.0, fake,
                                   fake, None)
    assert rc == hsnf4.ERR_INVALID
    msg = hsnf4.last_error()
    assert "scratch" in msg and "maximum" in msg
