"""LoRA dropout on the GPU (Poros API reference: lora_dropout) against the
oracle: the mask and X_d bit-exact, the LoRA forward/backward with dropout
within the parity bar, streamed == resident bitwise with dropout on, and the
backward re-drawing the forward's mask from (seed, offset)."""
import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.stack import LayerStack
from gpu_util import assert_lora_close, bf16_bits, bf16_to_f64, oracle_nf4_weight, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,K,p,seed,offset", [
    (1, 64, 0.05, 1, 0),
    (37, 192, 0.05, 42, (3 << 32) | 17),
    (513, 3584, 0.5, 0xFFFF_FFFF_FFFF_FFFF, 0xFFFF_FFFF_0000_0001),
    (64, 18944, 0.9, 7, 1 << 40),
])
def test_dropout_apply_bitwise(orc, T, K, p, seed, offset):
    rng = np.random.default_rng(T + K)
    X = synth.normal_bf16(rng, (T, K), 1.0)
    got = bf16_bits(hsnf4.lora_dropout_apply(to_dev_bf16(X), p, seed, offset))
    ref = orc.dropout_apply(X, seed, offset, p)
    torch.cuda.synchronize()
    assert np.array_equal(got, ref)


def _group(orc, cases, T, r, alpha, drops):
    """One grouped forward + backward on the oracle's NF4 codes;
    drops[i] = (p, seed, offset) or None."""
    Ws, outs, fa, ba = [], [], [], []
    for c, d in zip(cases, drops):
        W = oracle_nf4_weight(orc, c.W)
        X, A, B, dY = (to_dev_bf16(a) for a in (c.X, c.A, c.B, c.dY))
        N, K = c.W.shape
        Y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
        t = torch.empty(T, r, dtype=torch.float32, device="cuda")
        dX = torch.empty(T, K, dtype=torch.bfloat16, device="cuda")
        dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
        dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
        Ws.append((W, X, A, B, dY))
        outs.append((Y, t, dX, dA, dB))
        fa.append(hsnf4.fwd_args(W, X, A, B, Y, t, d))
        ba.append(hsnf4.bwd_args(W, X, t, A, B, dY, dX, dA, dB, d))
    wf = torch.empty(hsnf4.group_fwd_workspace_bytes(fa, T, r), dtype=torch.uint8, device="cuda")
    wb = torch.empty(hsnf4.group_bwd_workspace_bytes(ba, T, r), dtype=torch.uint8, device="cuda")
    hsnf4.lora_group_fwd(fa, T, r, alpha, wf)
    hsnf4.lora_group_bwd(ba, T, r, alpha, wb)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    return Ws, outs


@pytest.mark.parametrize("T,p", [(64, 0.05), (300, 0.5), (512, 0.05)])
def test_group_with_dropout_vs_oracle(orc, T, p):
    r, alpha = 16, 32.0
    shapes = [(512, 512), (192, 320), (128, 4096), (640, 256)]
    cases = [synth.linear_case(9000 + i + T, T, N, K, r=r, alpha=alpha, b_std=0.05)
             for i, (N, K) in enumerate(shapes)]
    # one problem without dropout in the same group
    drops = [(p, 1234, (5 << 32) | i) if i != 1 else None for i in range(len(cases))]
    Ws, outs = _group(orc, cases, T, r, alpha, drops)
    for c, d, (W, *_), (Y, t, dX, dA, dB) in zip(cases, drops, Ws, outs):
        N, K = c.W.shape
        codes, absmax = W.codes.cpu().numpy(), W.absmax.cpu().numpy()
        pp, seed, off = d or (0.0, 0, 0)
        Yr, tr = orc.lora_fwd_drop(codes, absmax, N, K, c.X, c.A, c.B, alpha, pp, seed, off)
        dXr, dAr, dBr = orc.lora_bwd_drop(codes, absmax, N, K, c.X, c.A, c.B, c.dY, alpha, pp,
                                          seed, off)
        what = f"T{T} p{pp} {N}x{K}"
        assert_lora_close(bf16_to_f64(Y), Yr, what + " Y")
        assert_lora_close(t.cpu().numpy(), tr, what + " t")
        assert_lora_close(bf16_to_f64(dX), dXr, what + " dX")
        assert_lora_close(dA.cpu().numpy(), dAr, what + " dA")
        assert_lora_close(dB.cpu().numpy(), dBr, what + " dB")


def test_dropout_changes_the_adapter_path_and_is_reproducible(orc):
    T, r = 128, 16
    c = [synth.linear_case(9100, T, 256, 512, r=r, b_std=0.05)]
    _, a = _group(orc, c, T, r, 32.0, [(0.5, 9, 1)])
    _, b = _group(orc, c, T, r, 32.0, [(0.5, 9, 1)])
    _, o = _group(orc, c, T, r, 32.0, [(0.5, 9, 2)])
    for x, y in zip(a[0], b[0]):
        assert torch.equal(x, y)                    # same (seed, offset): same bits
    assert not torch.equal(a[0][1], o[0][1])        # another offset: another t


TINY = synth.Family("tiny", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=4)


def _stack_run(stack):
    rec = {}
    for _ in range(2):
        rec.clear()
        stack.step(lambda l, p, n, t: rec.__setitem__((l, p, n), t.clone()))
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    for l in range(stack.L):
        for p in range(stack.P):
            rec[(l, p, "t")] = stack.t[l][p].clone()
            rec[(l, p, "dA")] = stack.dA[l][p].clone()
            rec[(l, p, "dB")] = stack.dB[l][p].clone()
    return rec


def test_dropout_stack_streamed_equals_resident_bitwise():
    res = LayerStack(TINY, 4, 96, streamed=False, dropout=0.05)
    ref = _stack_run(res)
    res.close()
    for bs in (1, 2, 4):
        s = LayerStack(TINY, 4, 96, block_size=bs, streamed=True, dropout=0.05)
        got = _stack_run(s)
        s.close()
        for k in ref:
            assert torch.equal(got[k], ref[k]), (bs, k)
