"""NF4 quantize+pack and dequantize on the GPU vs the oracle: bit-exact."""
import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from gpu_util import bf16_bits, to_dev_bf16

pytestmark = pytest.mark.gpu

SHAPES = [
    (1, 64),        # one block
    (3, 64),        # odd block count (a lone block in the last pair)
    (5, 192),       # odd block count, several per row
    (64, 64),
    (192, 320),
    (512, 512),     # the single-linear case
    (128, 4160),
]


def _quant_both(orc, w_bits):
    n, k = w_bits.shape
    codes_ref, absmax_ref = orc.quantize(w_bits)
    W = hsnf4.nf4_quantize_pack(to_dev_bf16(w_bits))
    torch.cuda.synchronize()
    return W, codes_ref, absmax_ref


@pytest.mark.parametrize("n,k", SHAPES)
def test_quantize_bit_exact(orc, n, k):
    rng = np.random.default_rng(n * 1000 + k)
    w = synth.normal_bf16(rng, (n, k), 0.02)
    W, codes_ref, absmax_ref = _quant_both(orc, w)
    assert np.array_equal(W.codes.cpu().numpy(), codes_ref)
    assert np.array_equal(W.absmax.cpu().numpy().view(np.uint32), absmax_ref.view(np.uint32))


@pytest.mark.parametrize("n,k", SHAPES)
def test_dequant_bit_exact(orc, n, k):
    rng = np.random.default_rng(7 + n + k)
    w = synth.normal_bf16(rng, (n, k), 0.02)
    codes, absmax = orc.quantize(w)
    ref = orc.dequant(codes, absmax, n, k)
    W = hsnf4.Nf4Weight(torch.from_numpy(codes).cuda(), torch.from_numpy(absmax).cuda(), n, k)
    out = hsnf4.nf4_dequant(W)
    assert np.array_equal(bf16_bits(out), ref)


def test_dequant_every_code_and_scale(orc):
    """All 16 codes at many absmax values (incl. 0, tiny, huge, powers of 2)."""
    rng = np.random.default_rng(11)
    n, k = 64, 256
    codes = rng.integers(0, 256, size=n * k // 2, dtype=np.uint8)
    scales = np.concatenate([[0.0, 1.0, 2.0**-20, 2.0**20, 3.0e-5, 65504.0],
                             rng.uniform(1e-4, 1e2, n * k // 64 - 6)]).astype(np.float32)
    ref = orc.dequant(codes, scales, n, k)
    W = hsnf4.Nf4Weight(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), n, k)
    assert np.array_equal(bf16_bits(hsnf4.nf4_dequant(W)), ref)


def test_quantize_special_blocks(orc):
    """All-zero, signed-zero, +-absmax and codebook-exact blocks."""
    cb = orc.codebook()
    w = np.zeros((4, 128), np.float32)
    w[1, :64] = -0.0
    w[2, 0], w[2, 1] = 3.0, -3.0
    w[3] = cb[np.arange(128) % 16] * np.float32(0.25)
    bits = synth.to_bf16_bits(w)
    W, codes_ref, absmax_ref = _quant_both(orc, bits)
    assert np.array_equal(W.codes.cpu().numpy(), codes_ref)
    assert np.array_equal(W.absmax.cpu().numpy(), absmax_ref)


@pytest.mark.parametrize("name", ["q", "k", "gate", "down"])
def test_quantize_dequant_full_size_qwen7b(orc, name):
    """Full Qwen2.5-7B-shaped projection weights (up to 18944 x 3584)."""
    fam = synth.FAMILIES["qwen2.5-7b"]
    idx = synth.PROJ_NAMES.index(name)
    _, n, k = fam.projections()[idx]
    rng = np.random.default_rng(synth.sub_seed(42, 0, idx))
    w = synth.normal_bf16(rng, (n, k), 0.02)
    W, codes_ref, absmax_ref = _quant_both(orc, w)
    assert np.array_equal(W.codes.cpu().numpy(), codes_ref)
    assert np.array_equal(W.absmax.cpu().numpy(), absmax_ref)
    out = hsnf4.nf4_dequant(W)
    assert np.array_equal(bf16_bits(out), orc.dequant(codes_ref, absmax_ref, n, k))


def test_device_codebook_equals_oracle(orc):
    assert np.array_equal(np.array(hsnf4.codebook(), np.float32), orc.codebook())
