"""LoRA linear forward/backward on the GPU (fused NF4 dequant + tcgen05 GEMM)
vs the fp32/double oracle, within the stated tolerance."""
import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from gpu_util import assert_lora_close, bf16_to_f64, oracle_nf4_weight, to_dev_bf16

pytestmark = pytest.mark.gpu


def _run(orc, case):
    """The GPU forward and backward on the oracle's NF4 codes of case.W."""
    T, N, K, r = case.shape
    W = oracle_nf4_weight(orc, case.W)
    X, A, B, dY = (to_dev_bf16(a) for a in (case.X, case.A, case.B, case.dY))
    Y, t = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
    dX, dA, dB = hsnf4.lora_linear_bwd(W, X, t, A, B, dY, case.alpha)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    return W, Y, t, dX, dA, dB


def _check(orc, case, got, rows=None, what=""):
    T, N, K, r = case.shape
    W, Y, t, dX, dA, dB = got
    codes, absmax = W.codes.cpu().numpy(), W.absmax.cpu().numpy()
    Yr, tr = orc.lora_fwd(codes, absmax, N, K, case.X, case.A, case.B, case.alpha, rows=rows)
    dXr, dAr, dBr = orc.lora_bwd(codes, absmax, N, K, case.X, case.A, case.B, case.dY,
                                 case.alpha, rows=rows)
    Yg, dXg = bf16_to_f64(Y), bf16_to_f64(dX)
    if rows is not None:
        Yg, dXg = Yg[rows], dXg[rows]
    assert_lora_close(Yg, Yr, what + " Y")
    assert_lora_close(t.cpu().numpy(), tr, what + " t")
    assert_lora_close(dXg, dXr, what + " dX")
    assert_lora_close(dA.cpu().numpy(), dAr, what + " dA")
    assert_lora_close(dB.cpu().numpy(), dBr, what + " dB")


CASES = [
    # T, N, K, r, alpha
    (64, 512, 512, 16, 32.0),     # the single-linear case
    (1, 128, 128, 16, 32.0),      # one token
    (37, 64, 64, 16, 32.0),       # smallest weight, ragged T
    (100, 192, 320, 8, 16.0),     # N, K not multiples of 128; r = 8
    (300, 256, 384, 32, 64.0),    # two token tiles, the second ragged
    (256, 128, 2048, 24, 48.0),   # r = 24 (padded rank slice), long K
    (512, 640, 1152, 64, 128.0),  # r = 64
    (129, 384, 192, 16, 7.0),     # alpha/r not a power of two
]


@pytest.mark.parametrize("T,N,K,r,alpha", CASES)
def test_lora_fwd_bwd_vs_oracle(orc, T, N, K, r, alpha):
    case = synth.linear_case(1000 + T + N + K + r, T, N, K, r=r, alpha=alpha)
    _check(orc, case, _run(orc, case), what=f"T{T} N{N} K{K} r{r}")


def test_deterministic_bitwise(orc):
    case = synth.linear_case(5, 300, 384, 640, r=16)
    a = _run(orc, case)
    b = _run(orc, case)
    for x, y in zip(a[1:], b[1:]):
        assert torch.equal(x, y)


def test_zero_adapter_B_gives_base_only(orc):
    """B = 0: Y is the plain NF4 matmul; dA = 0 exactly."""
    case = synth.linear_case(6, 128, 256, 512)
    case.B[:] = 0
    got = _run(orc, case)
    _check(orc, case, got, what="B=0")
    assert torch.count_nonzero(got[4]) == 0


@pytest.mark.parametrize("name", ["q", "k", "o", "gate", "down"])
def test_full_size_qwen7b_projection_sampled(orc, name):
    """Full Qwen2.5-7B shapes at T = 512 (the benchmarked launch
    configuration); Y and dX on 8 sampled token rows, t, dA, dB in full."""
    fam = synth.FAMILIES["qwen2.5-7b"]
    idx = synth.PROJ_NAMES.index(name)
    _, N, K = fam.projections()[idx]
    case = synth.linear_case(synth.sub_seed(42, 0, idx) % (2**31), 512, N, K)
    rows = np.array([0, 1, 127, 128, 255, 256, 400, 511])
    _check(orc, case, _run(orc, case), rows=rows, what=name)


# ---------------------------------------------------------------- grouped launches

GROUP = [  # (N, K): mixed shapes, one long-K problem (split along K), ragged N
    (512, 512), (192, 320), (128, 4096), (640, 256),
]


def _group_run(orc, cases, T, r, alpha, share_x=False):
    """One grouped forward + backward.  share_x: problems whose X is the same
    host array get the same device tensor (one pointer, as in a layer)."""
    Ws, ins, outs = [], [], []
    fa, ba = [], []
    dev_x = {}
    for c in cases:
        W = oracle_nf4_weight(orc, c.W)
        A, B, dY = (to_dev_bf16(a) for a in (c.A, c.B, c.dY))
        if share_x:
            X = dev_x.setdefault(id(c.X), to_dev_bf16(c.X))
        else:
            X = to_dev_bf16(c.X)
        N, K = c.W.shape
        Y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
        t = torch.empty(T, r, dtype=torch.float32, device="cuda")
        dX = torch.empty(T, K, dtype=torch.bfloat16, device="cuda")
        dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
        dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
        Ws.append(W)
        ins.append((X, A, B, dY))
        outs.append((Y, t, dX, dA, dB))
        fa.append(hsnf4.fwd_args(W, X, A, B, Y, t))
        ba.append(hsnf4.bwd_args(W, X, t, A, B, dY, dX, dA, dB))
    wf = torch.empty(hsnf4.group_fwd_workspace_bytes(fa, T, r), dtype=torch.uint8, device="cuda")
    wb = torch.empty(hsnf4.group_bwd_workspace_bytes(ba, T, r), dtype=torch.uint8, device="cuda")
    hsnf4.lora_group_fwd(fa, T, r, alpha, wf)
    hsnf4.lora_group_bwd(ba, T, r, alpha, wb)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    return Ws, outs


@pytest.mark.parametrize("T", [64, 300, 512])
def test_group_fwd_bwd_vs_oracle(orc, T):
    r, alpha = 16, 32.0
    cases = [synth.linear_case(7000 + i + T, T, N, K, r=r, alpha=alpha)
             for i, (N, K) in enumerate(GROUP)]
    Ws, outs = _group_run(orc, cases, T, r, alpha)
    for c, W, (Y, t, dX, dA, dB) in zip(cases, Ws, outs):
        _check(orc, c, (W, Y, t, dX, dA, dB), what=f"group T{T} {c.W.shape}")


@pytest.mark.parametrize("T,r", [(512, 16), (300, 8), (129, 64), (64, 24)])
def test_group_sharing_one_input_vs_oracle(orc, T, r):
    """Problems that read the same X (as q, k, v, gate and up do) are stacked
    on one read of X by the rank-r kernels; each must still match the
    oracle.  Their upstream gradients differ, and one problem reads another X."""
    alpha = 2.0 * r
    K = 640
    shared = synth.linear_case(9500 + T + r, T, 64, K, r=r, alpha=alpha)
    cases = []
    for i, N in enumerate([384, 128, 128, 1152, 1152]):
        c = synth.linear_case(9600 + 17 * i + T + r, T, N, K, r=r, alpha=alpha)
        c.X = shared.X  # the same input tensor for all five
        cases.append(c)
    cases.append(synth.linear_case(9700 + T + r, T, 512, 1152, r=r, alpha=alpha))
    Ws, outs = _group_run(orc, cases, T, r, alpha, share_x=True)
    for c, W, (Y, t, dX, dA, dB) in zip(cases, Ws, outs):
        _check(orc, c, (W, Y, t, dX, dA, dB), what=f"shared-X group T{T} r{r} {c.W.shape}")


def test_group_deterministic_bitwise(orc):
    T, r = 512, 16
    cases = [synth.linear_case(8000 + i, T, N, K, r=r) for i, (N, K) in enumerate(GROUP)]
    _, a = _group_run(orc, cases, T, r, 32.0)
    _, b = _group_run(orc, cases, T, r, 32.0)
    for xa, xb in zip(a, b):
        for u, v in zip(xa, xb):
            assert torch.equal(u, v)


def test_groupings_agree_within_tolerance(orc):
    """The same layer through grouped (decoder / layer) and per-projection
    launches: equal within the parity bar (K splits may differ)."""
    from host_streamed_nf4_b200.stack import LayerStack
    fam = synth.Family("tiny", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=1)
    res = {}
    for g in ("decoder", "layer", "none"):
        s = LayerStack(fam, 1, 192, streamed=False, grouping=g)
        rec = {}
        s.step(lambda l, p, n, t: rec.__setitem__((l, p, n), t.clone()))
        torch.cuda.synchronize()
        res[g] = rec
        s.close()
    for k in res["none"]:
        for g in ("decoder", "layer"):
            assert_lora_close(bf16_to_f64(res[g][k]), bf16_to_f64(res["none"][k]), f"{g} {k}")
