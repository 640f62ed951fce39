"""lora_linear_fwd_noalloc: the LoRA forward for callers that cannot
allocate device memory (a runtime that reserves its whole device-memory
budget up front and forbids later allocations, a plugin or callback that may
not call the allocator).  It uses the library's built-in scratch instead of
a caller workspace; its results must match lora_linear_fwd's, call after
call, even though every call reuses (and leaves behind) the same scratch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from gpu_util import assert_lora_close, bf16_to_f64, to_dev_bf16

SHAPES = [  # T, N, K: the single-linear case, a ragged case, a K-split case
    (64, 512, 512),
    (300, 192, 320),
    (512, 3584, 3584),
]


@pytest.mark.gpu
@pytest.mark.parametrize("T,N,K", SHAPES)
def test_noalloc_forward_matches_workspace_forward_twice(T, N, K):
    case = synth.linear_case(9100 + T + N, T, N, K)
    W = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    X, A, B = (to_dev_bf16(a) for a in (case.X, case.A, case.B))
    Y_ref, t_ref = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
    torch.cuda.synchronize()
    for _ in range(2):  # the second call starts from the first call's leftovers
        Y, t = hsnf4.lora_linear_fwd_noalloc(W, X, A, B, case.alpha)
        torch.cuda.synchronize()
        assert hsnf4.device_status() == 0
        assert_lora_close(bf16_to_f64(Y), bf16_to_f64(Y_ref), f"noalloc Y {T}x{N}x{K}")
        assert_lora_close(t.cpu().numpy(), t_ref.cpu().numpy(), f"noalloc t {T}x{N}x{K}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked from the shapes alone: the call fails before touching memory."""
    L = hsnf4.lib()
    fake = 0x10000
    # r = 64 over a 32768-wide contraction at 16384 tokens: the rank-r
    # projection's partial sums alone need 128 MiB
    W = hsnf4.Nf4WeightC(fake, fake, 4096, 32768)
    rc = L.lora_linear_fwd_noalloc(ctypes.byref(W), fake, 16384, fake, fake, 64, 128.0, fake,
                                   fake, None)
    assert rc == hsnf4.ERR_INVALID
    msg = hsnf4.last_error()
    assert "scratch" in msg and "maximum" in msg
