"""Streamed == resident, bitwise, at the full sizes of the benchmarked stacks.

The pages' bar for streaming is exact identity with a resident run at any
block size ("Poros on consumer GPUs": NF4 is the precision with 0.00e+00
parity to a fully resident run in "Quick start on a consumer card", and
lowering block_size never affects parity in the "OOM playbook"; Poros API
reference, block_size).  The small-family tests in test_gpu_stream.py check
the ring's logic; these run the real shapes, which reach what the small ones
cannot: 512-token tensor-memory units, the K-split plans the 8B and 72B
projections select, ring slots of several GB and slab offsets beyond 32 GiB
(the 72B slab is 39.5 GB).  Every Y and dX of every layer and projection,
every saved t and every dA and dB is compared with torch.equal, over two
steps (the second starts from the blocks the first left resident).

The last layer of the 72B stack -- the slab's last 494 MB -- is also checked
against the oracle: its seven projections' codes and absmax must be the
oracle's own quantization of the seeded weights, and Y and dX on sampled
token rows, t, dA and dB in full must meet the LoRA bar.
"""
import gc

import numpy as np
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.stack import INPUT_OF, LayerStack
from gpu_util import assert_lora_close, bf16_bits, bf16_to_f64

pytestmark = pytest.mark.gpu

ROWS = np.array([0, 1, 127, 128, 255, 256, 400, 511])


def _record_run(stack, steps=2):
    rec = {}

    def record(l, p, name, t):
        rec[(l, p, name)] = t.clone()

    for _ in range(steps):
        rec.clear()
        stack.step(record)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    for l in range(stack.L):
        for p in range(stack.P):
            rec[(l, p, "t")] = stack.t[l][p].clone()
            rec[(l, p, "dA")] = stack.dA[l][p].clone()
            rec[(l, p, "dB")] = stack.dB[l][p].clone()
    return rec


def _assert_bitwise(got, ref, what):
    assert got.keys() == ref.keys(), what
    bad = [k for k in ref if not torch.equal(got[k], ref[k])]
    assert not bad, f"{what}: {len(bad)} of {len(ref)} tensors differ, first {bad[:4]}"


def _reclaim():
    """Return the device memory of stacks already closed and dropped."""
    gc.collect()
    torch.cuda.empty_cache()


def _resident_record(fam, L, T, slab):
    res = LayerStack(fam, L, T, streamed=False, slab=slab)
    rec = _record_run(res)
    res.close()
    del res
    _reclaim()
    return rec


# ---------------------------------------------------------------- Llama-3.1-8B, 32 layers

@pytest.fixture(scope="module")
def llama8b():
    fam = synth.FAMILIES["llama-3.1-8b"]
    res = LayerStack(fam, 32, 512, streamed=False)
    rec = _record_run(res)
    slab = res.slab
    res.close()
    del res
    _reclaim()
    yield fam, slab, rec


@pytest.mark.parametrize("bs", [1, 2, 4])
def test_llama8b_stack_streamed_equals_resident(llama8b, bs):
    fam, slab, ref = llama8b
    s = LayerStack(fam, 32, 512, block_size=bs, streamed=True, slab=slab)
    got = _record_run(s)
    moved = s.streamer.stats()["h2d_bytes"]
    s.close()
    del s
    _reclaim()
    _assert_bitwise(got, ref, f"llama-3.1-8b stack, block_size {bs}")
    assert moved > 0


# ---------------------------------------------------------------- Qwen2.5-72B, 80 layers

@pytest.fixture(scope="module")
def qwen72b_slab():
    """The 72B stack's pinned NF4 slab (39.5 GB), drawn and quantized once."""
    fam = synth.FAMILIES["qwen2.5-72b"]
    s = LayerStack(fam, 80, 512, block_size=4, streamed=True)
    slab = s.slab
    s.close()
    del s
    _reclaim()
    yield fam, slab


def _check_last_layer_vs_oracle(orc, stack, rec):
    l = stack.L - 1
    slab = stack.slab.numpy()
    base = l * stack.layer_bytes
    assert base + stack.layer_bytes > 32 << 30  # the layer lies past 32 GiB in the slab
    for p, (name, n, k) in enumerate(stack.projs):
        co, ao = stack.offs[p]
        codes, absmax = orc.quantize(bf16_bits(stack.base_weight_bf16(l, p)))
        assert np.array_equal(slab[base + co: base + co + n * k // 2], codes), name
        assert np.array_equal(slab[base + ao: base + ao + n * k // 16].view(np.float32),
                              absmax), name
        X = bf16_bits(stack.X[INPUT_OF[name]])
        A, B, dY = bf16_bits(stack.A[l][p]), bf16_bits(stack.B[l][p]), bf16_bits(stack.dY[p])
        Yr, tr = orc.lora_fwd(codes, absmax, n, k, X, A, B, stack.alpha, rows=ROWS)
        dXr, dAr, dBr = orc.lora_bwd(codes, absmax, n, k, X, A, B, dY, stack.alpha, rows=ROWS)
        what = f"72b layer {l} {name}"
        assert_lora_close(bf16_to_f64(rec[(l, p, "Y")])[ROWS], Yr, what + " Y")
        assert_lora_close(rec[(l, p, "t")].cpu().numpy(), tr, what + " t")
        assert_lora_close(bf16_to_f64(rec[(l, p, "dX")])[ROWS], dXr, what + " dX")
        assert_lora_close(rec[(l, p, "dA")].cpu().numpy(), dAr, what + " dA")
        assert_lora_close(rec[(l, p, "dB")].cpu().numpy(), dBr, what + " dB")


@pytest.mark.parametrize("T,bs", [(512, 4), (512, 1), (256, 4)])
def test_qwen72b_stack_streamed_equals_resident(orc, qwen72b_slab, T, bs):
    fam, slab = qwen72b_slab
    ref = _resident_record(fam, 80, T, slab)
    s = LayerStack(fam, 80, T, block_size=bs, streamed=True, slab=slab)
    got = _record_run(s)
    try:
        _assert_bitwise(got, ref, f"qwen2.5-72b stack, T {T}, block_size {bs}")
        del ref
        if (T, bs) == (512, 4):
            _check_last_layer_vs_oracle(orc, s, got)
    finally:
        s.close()
        del s, got
        _reclaim()
