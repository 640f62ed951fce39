"""Helpers shared by the GPU tests: moving bf16 bit patterns between numpy
and torch, and the floating-point parity bar."""
import numpy as np
import torch

# LoRA outputs vs the fp32 oracle: max|d| <= 2e-2 max|ref| and
# ||d||_F <= 5e-3 ||ref||_F.  (bf16 outputs carry a relative rounding error
# <= 2^-9 per element; the rank-r factor is rounded to bf16 once before the
# tensor-core slice, another <= 2^-9 on a term that is a fraction of the
# output; fp32 accumulation over <= 30k terms adds ~1e-6.  The Frobenius
# bound therefore has ~3x headroom and the max bound ~10x.)
MAX_REL = 2e-2
FRO_REL = 5e-3


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_nf4_weight(orc, w_bits: np.ndarray):
    """Quantize a bf16 weight (uint16 bits [N, K]) with the oracle and upload
    its codes and absmax, so that a LoRA check does not depend on the GPU
    quantizer (which the codec tests check separately)."""
    from host_streamed_nf4_b200 import hsnf4
    n, k = w_bits.shape
    codes, absmax = orc.quantize(w_bits)
    return hsnf4.Nf4Weight(torch.from_numpy(codes).cuda(), torch.from_numpy(absmax).cuda(), n, k)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_lora_close(got, ref, what="", max_rel=MAX_REL, fro_rel=FRO_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    d = np.abs(got - ref)
    scale = np.abs(ref).max()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert d.max() <= max_rel * scale, f"{what}: max|d| {d.max():.3e} > {max_rel} * {scale:.3e}"
    assert fro <= fro_rel, f"{what}: rel Frobenius {fro:.3e} > {fro_rel}"
    return (d.max() / scale if scale > 0 else 0.0), fro
