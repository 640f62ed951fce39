"""The dense bf16 base (the quantization="bf16_bitwise" base of the Poros API
reference: streamed like NF4, never dequantized) and merge_and_unload
(PorosModel.merge_and_unload) on the GPU, against the oracle.

Parity bars: LoRA outputs as for NF4 (max|d| <= 2e-2 max|ref|, Frobenius
<= 5e-3); streamed == resident bitwise.  The merged weight is one bf16
rounding of a sum the GPU forms in fp32 and the oracle exactly: an element
may differ where the exact value sits within the fp32 error of a bf16
rounding boundary, by at most one bf16 unit in the last place plus that
fp32 error (which matters only where the sum nearly cancels); the test
checks that bound on every element and that at most 1e-3 of the elements
differ at all (expected about 2^-14).
"""
import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.stack import LayerStack
from gpu_util import assert_lora_close, bf16_bits, bf16_to_f64, oracle_nf4_weight, to_dev_bf16

pytestmark = pytest.mark.gpu

CASES = [
    # T, N, K, r, alpha
    (64, 512, 512, 16, 32.0),
    (1, 128, 128, 16, 32.0),
    (100, 192, 320, 8, 16.0),     # N, K not multiples of 128
    (300, 256, 384, 32, 64.0),    # ragged second token tile
    (256, 128, 2048, 24, 48.0),   # long K (split along K), padded rank
    (512, 640, 1152, 64, 128.0),
]


def _run_dense(case):
    W = hsnf4.Bf16Weight(to_dev_bf16(case.W))
    X, A, B, dY = (to_dev_bf16(a) for a in (case.X, case.A, case.B, case.dY))
    Y, t = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
    dX, dA, dB = hsnf4.lora_linear_bwd(W, X, t, A, B, dY, case.alpha)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    return Y, t, dX, dA, dB


@pytest.mark.parametrize("T,N,K,r,alpha", CASES)
def test_dense_base_fwd_bwd_vs_oracle(orc, T, N, K, r, alpha):
    case = synth.linear_case(3000 + T + N + K + r, T, N, K, r=r, alpha=alpha)
    Y, t, dX, dA, dB = _run_dense(case)
    Yr, tr = orc.lora_fwd_bf16w(case.W, case.X, case.A, case.B, alpha)
    dXr, dAr, dBr = orc.lora_bwd_bf16w(case.W, case.X, case.A, case.B, case.dY, alpha)
    what = f"dense T{T} N{N} K{K} r{r}"
    assert_lora_close(bf16_to_f64(Y), Yr, what + " Y")
    assert_lora_close(t.cpu().numpy(), tr, what + " t")
    assert_lora_close(bf16_to_f64(dX), dXr, what + " dX")
    assert_lora_close(dA.cpu().numpy(), dAr, what + " dA")
    assert_lora_close(dB.cpu().numpy(), dBr, what + " dB")


def test_dense_base_full_size_gate_sampled(orc):
    """Qwen2.5-7B gate shape at T = 512 with a dense base; Y and dX on sampled rows."""
    fam = synth.FAMILIES["qwen2.5-7b"]
    _, N, K = fam.projections()[synth.PROJ_NAMES.index("gate")]
    case = synth.linear_case(77, 512, N, K)
    Y, t, dX, dA, dB = _run_dense(case)
    rows = np.array([0, 255, 256, 511])
    Yr, tr = orc.lora_fwd_bf16w(case.W, case.X, case.A, case.B, case.alpha, rows=rows)
    dXr, dAr, dBr = orc.lora_bwd_bf16w(case.W, case.X, case.A, case.B, case.dY, case.alpha,
                                       rows=rows)
    assert_lora_close(bf16_to_f64(Y)[rows], Yr, "gate Y")
    assert_lora_close(bf16_to_f64(dX)[rows], dXr, "gate dX")
    assert_lora_close(dA.cpu().numpy(), dAr, "gate dA")
    assert_lora_close(dB.cpu().numpy(), dBr, "gate dB")


def test_dense_base_of_dequantized_weight_equals_nf4_path():
    """The dense kernels on W = deq(codes) and the fused-dequant kernels on
    the codes run the same tensor-core accumulation on the same bf16
    operand: the results are bitwise equal."""
    case = synth.linear_case(31, 300, 384, 640, r=16)
    Wq = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    Wd = hsnf4.Bf16Weight(hsnf4.nf4_dequant(Wq))
    X, A, B, dY = (to_dev_bf16(a) for a in (case.X, case.A, case.B, case.dY))
    outs = []
    for W in (Wq, Wd):
        Y, t = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
        dX, dA, dB = hsnf4.lora_linear_bwd(W, X, t, A, B, dY, case.alpha)
        outs.append((Y, t, dX, dA, dB))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_group_rejects_mixed_formats():
    case = synth.linear_case(32, 64, 128, 128)
    Wq = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    Wd = hsnf4.Bf16Weight(to_dev_bf16(case.W))
    X, A, B = (to_dev_bf16(a) for a in (case.X, case.A, case.B))
    Y1 = torch.empty(64, 128, dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty_like(Y1)
    fa = [hsnf4.fwd_args(Wq, X, A, B, Y1), hsnf4.fwd_args(Wd, X, A, B, Y2)]
    ws = torch.empty(hsnf4.group_fwd_workspace_bytes(fa, 64, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(hsnf4.HsNf4Error) as e:
        hsnf4.lora_group_fwd(fa, 64, 16, 32.0, ws)
    assert e.value.status == hsnf4.ERR_INVALID and "format" in e.value.detail


# ---------------------------------------------------------------- merge_and_unload

def _next_up(bits):
    """bf16 bits of the next value away from zero (magnitude + 1 ulp)."""
    return (bits.astype(np.uint32) + 1).astype(np.uint16)


def _ulp_diff(a_bits, b_bits):
    """|a - b| in bf16 units in the last place (same-sign finite values)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordered(a_bits) - ordered(b_bits))


@pytest.mark.parametrize("N,K,r,alpha", [(64, 64, 8, 16.0), (192, 320, 16, 32.0),
                                         (512, 1152, 64, 128.0), (128, 640, 24, 7.0),
                                         # more 128 x 128 tiles than the persistent
                                         # grid has CTAs: each CTA takes several
                                         (4096, 4160, 16, 32.0)])
@pytest.mark.parametrize("base", ["nf4", "bf16"])
def test_merge_vs_oracle(orc, N, K, r, alpha, base):
    case = synth.linear_case(4000 + N + K + r, 1, N, K, r=r, alpha=alpha, b_std=0.05)
    A, B = to_dev_bf16(case.A), to_dev_bf16(case.B)
    if base == "nf4":
        W = oracle_nf4_weight(orc, case.W)
        ref = orc.lora_merge(case.A, case.B, alpha, codes=W.codes.cpu().numpy(),
                             absmax=W.absmax.cpu().numpy(), N=N, K=K)
    else:
        W = hsnf4.Bf16Weight(to_dev_bf16(case.W))
        ref = orc.lora_merge(case.A, case.B, alpha, W=case.W)
    got = bf16_bits(hsnf4.lora_merge(W, A, B, alpha))
    torch.cuda.synchronize()
    # bound: one bf16 rounding of the exact value, plus what the GPU's fp32
    # arithmetic can move that value before it is rounded -- an r-term fp32
    # sum of exact products, a scale and an add: (r + 2) 2^-24 of the sum of
    # magnitudes.  The bf16 rounding doubles an fp32 error at worst.
    deq = synth.bits_to_f32(case.W if base == "bf16" else
                            orc.dequant(W.codes.cpu().numpy(), W.absmax.cpu().numpy(), N, K))
    mag = (alpha / r) * (np.abs(synth.bits_to_f32(case.B)).astype(np.float64) @
                         np.abs(synth.bits_to_f32(case.A)).astype(np.float64))
    mag += np.abs(deq.astype(np.float64))
    fp32_err = 2 * (r + 2) * 2.0 ** -24 * mag
    g64, r64 = synth.bits_to_f32(got).astype(np.float64), synth.bits_to_f32(ref).astype(np.float64)
    ulp = np.abs(synth.bits_to_f32(_next_up(ref)).astype(np.float64) - r64)
    bad = np.abs(g64 - r64) > ulp + fp32_err
    assert not bad.any(), f"{bad.sum()} elements beyond one bf16 ulp + the fp32 bound"
    d = _ulp_diff(got, ref)
    assert (d > 0).mean() <= 1e-3, f"{(d > 0).mean():.2e} of the elements differ from the oracle"


def test_merge_repeatable_on_a_full_size_gate(orc):
    """The Qwen2.5-72B gate projection (29568 x 8192, r 16): about 50 tiles
    per CTA, so every stage and accumulator buffer is reused many times while
    the producer runs ahead.  Every launch gives the same bits (a stage
    released before its reads completed showed up here as a few hundred wrong
    elements in most launches), and sampled rows, first and last tiles among
    them, agree with the oracle within the merge bound."""
    N, K, r, alpha = 29568, 8192, 16, 32.0
    case = synth.linear_case(4343, 1, N, K, r=r, alpha=alpha, b_std=0.05)
    W = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    A, B = to_dev_bf16(case.A), to_dev_bf16(case.B)
    first = hsnf4.lora_merge(W, A, B, alpha)
    out = torch.empty_like(first)
    for _ in range(5):
        hsnf4.lora_merge(W, A, B, alpha, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out, first)
    assert hsnf4.device_status() == 0
    rows = np.array([0, 1, 127, 128, 8191, 14783, 29439, 29567])
    codes, absmax = orc.quantize(case.W[rows])
    # the GPU quantizer's codes of these rows are the oracle's (codec parity)
    kb = K // 64
    gpu_codes = W.codes.view(N, K // 2)[torch.from_numpy(rows).cuda()].cpu().numpy()
    gpu_absmax = W.absmax.view(N, kb)[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(gpu_codes.reshape(-1), codes)
    assert np.array_equal(gpu_absmax.reshape(-1), absmax)
    ref = orc.lora_merge(case.A, case.B[rows], alpha, codes=codes, absmax=absmax, N=len(rows),
                         K=K)
    got = bf16_bits(first[torch.from_numpy(rows).cuda()])
    deq = synth.bits_to_f32(orc.dequant(codes, absmax, len(rows), K))
    mag = (alpha / r) * (np.abs(synth.bits_to_f32(case.B[rows])).astype(np.float64) @
                         np.abs(synth.bits_to_f32(case.A)).astype(np.float64))
    mag += np.abs(deq.astype(np.float64))
    fp32_err = 2 * (r + 2) * 2.0 ** -24 * mag
    g64, r64 = synth.bits_to_f32(got).astype(np.float64), synth.bits_to_f32(ref).astype(np.float64)
    ulp = np.abs(synth.bits_to_f32(_next_up(ref)).astype(np.float64) - r64)
    assert not (np.abs(g64 - r64) > ulp + fp32_err).any()
    assert (_ulp_diff(got, ref) > 0).mean() <= 1e-3


def test_merge_zero_adapter_is_dequant_bitwise():
    case = synth.linear_case(41, 1, 384, 512)
    W = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    A = to_dev_bf16(case.A)
    B = torch.zeros(384, 16, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(hsnf4.lora_merge(W, A, B, 32.0), hsnf4.nf4_dequant(W))


def test_merged_weight_reproduces_the_adapter_forward(orc):
    """Y from the merged dense weight with the adapter removed vs the NF4 +
    adapter forward: equal within the parity bar (the merge rounds W' to
    bf16 once; the adapter path rounds s t to bf16 once)."""
    case = synth.linear_case(42, 256, 384, 512, r=16, b_std=0.05)
    W = hsnf4.nf4_quantize_pack(to_dev_bf16(case.W))
    X, A, B = (to_dev_bf16(a) for a in (case.X, case.A, case.B))
    Y_adapter, _ = hsnf4.lora_linear_fwd(W, X, A, B, case.alpha)
    Wm = hsnf4.Bf16Weight(hsnf4.lora_merge(W, A, B, case.alpha))
    Y_merged, _ = hsnf4.lora_linear_fwd(Wm, X, A, torch.zeros_like(B), case.alpha)
    torch.cuda.synchronize()
    assert_lora_close(bf16_to_f64(Y_merged), bf16_to_f64(Y_adapter), "merged vs adapter")


# ---------------------------------------------------------------- streamed dense stack

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
            rec[(l, p, "dA")] = stack.dA[l][p].clone()
            rec[(l, p, "dB")] = stack.dB[l][p].clone()
    return rec


def test_dense_stack_streamed_equals_resident_bitwise():
    res = LayerStack(TINY, 4, 96, streamed=False, base="bf16")
    ref = _stack_run(res)
    res.close()
    for bs in (1, 2):
        s = LayerStack(TINY, 4, 96, block_size=bs, streamed=True, base="bf16")
        got = _stack_run(s)
        assert s.layer_bytes >= 3.5 * LayerStack(TINY, 1, 8, streamed=False).layer_bytes
        s.close()
        assert got.keys() == ref.keys()
        for k in ref:
            assert torch.equal(got[k], ref[k]), (bs, k)
