"""Decoder-layer glue and the rematerialized decoder stack on the GPU vs the
oracle (oracle/decoder.py and the module oracles), and the stack's bitwise
properties: streamed == resident, and the backward's recomputed forward ==
the forward."""
import numpy as np
import pytest
import torch

import oracle
from oracle import decoder as odec
from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.decoder import EPS, DecoderStack
from gpu_util import assert_lora_close, bf16_bits, bf16_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _rand_bf16(rng, shape, std=1.0):
    return synth.normal_bf16(rng, shape, std)


def _close_bf16(got, ref, what, rel=2.0 ** -7):
    """bf16 module outputs from fp32 arithmetic vs the double oracle rounded
    to bf16: within two bf16 units in the last place of the value (plus a
    floor at the output's scale for values near zero)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = rel * np.abs(ref) + 1e-3 * rel * np.abs(ref).max()
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {np.abs(got - ref).max():.3e}"


# ---------------------------------------------------------------- modules

@pytest.mark.parametrize("T,n", [(1, 256), (37, 3584), (64, 8192)])
def test_rmsnorm_fwd_bwd_vs_oracle(T, n):
    rng = np.random.default_rng(T + n)
    xa, xb, dy1, dy2, dy3, dres = (_rand_bf16(rng, (T, n)) for _ in range(6))
    g = _rand_bf16(rng, (n,), 0.1)
    g = synth.to_bf16_bits(1.0 + synth.bits_to_f32(g))
    f = lambda a: synth.bits_to_f32(a).astype(np.float64)
    # plain norm
    y = hsnf4.rmsnorm_fwd(to_dev_bf16(xa), to_dev_bf16(g), EPS)
    _close_bf16(bf16_to_f64(y), odec.rnd_bf16(oracle.rmsnorm_fwd(f(xa), f(g), EPS)), "rmsnorm")
    # fused residual add: h = bf16(xa + xb), y = rmsnorm(h)
    y2, h = hsnf4.rmsnorm_fwd(to_dev_bf16(xa), to_dev_bf16(g), EPS, res=to_dev_bf16(xb))
    h_ref = odec.rnd_bf16(f(xa) + f(xb))
    assert np.array_equal(bf16_to_f64(h), h_ref)  # one fp32 add of bf16 values: exact rounding
    _close_bf16(bf16_to_f64(y2), odec.rnd_bf16(oracle.rmsnorm_fwd(h_ref, f(g), EPS)), "add+norm")
    # backward with three branches and a residual gradient
    dx = hsnf4.rmsnorm_bwd(to_dev_bf16(xa), to_dev_bf16(g),
                           [to_dev_bf16(a) for a in (dy1, dy2, dy3)], EPS, dres=to_dev_bf16(dres))
    ref = odec.rnd_bf16(f(dres) + oracle.rmsnorm_bwd(f(xa), f(g), f(dy1) + f(dy2) + f(dy3), EPS))
    torch.cuda.synchronize()
    assert_lora_close(bf16_to_f64(dx), ref, "rmsnorm bwd")


def test_swiglu_vs_oracle():
    rng = np.random.default_rng(60)
    a, b, dm = (_rand_bf16(rng, (64, 18944), 2.0) for _ in range(3))
    f = lambda x: synth.bits_to_f32(x).astype(np.float64)
    m = hsnf4.swiglu_fwd(to_dev_bf16(a), to_dev_bf16(b))
    _close_bf16(bf16_to_f64(m), odec.rnd_bf16(oracle.silu_mul_fwd(f(a), f(b))), "swiglu")
    da, db = hsnf4.swiglu_bwd(to_dev_bf16(a), to_dev_bf16(b), to_dev_bf16(dm))
    rda, rdb = oracle.silu_mul_bwd(f(a), f(b), f(dm))
    torch.cuda.synchronize()
    _close_bf16(bf16_to_f64(da), odec.rnd_bf16(rda), "swiglu da", rel=2.0 ** -6)
    _close_bf16(bf16_to_f64(db), odec.rnd_bf16(rdb), "swiglu db")


@pytest.mark.parametrize("T,H,KV", [(1, 2, 1), (64, 2, 1), (100, 4, 2), (300, 4, 1),
                                    (128, 28, 4)])
def test_attention_vs_oracle(T, H, KV):
    rng = np.random.default_rng(T * 7 + H)
    d = 128
    q, k, v = (_rand_bf16(rng, (T, n * d)) for n in (H, KV, KV))
    do = _rand_bf16(rng, (T, H * d))
    f = lambda x: synth.bits_to_f32(x).astype(np.float64)
    sc = 1.0 / np.sqrt(128.0)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    o, lse = hsnf4.attention_fwd(qd, kd, vd, H, KV)
    ro, rlse = oracle.attention_fwd(f(q), f(k), f(v), H, KV, d, sc)
    assert_lora_close(bf16_to_f64(o), ro, f"attn o T{T}")
    assert np.abs(lse.cpu().numpy() - rlse).max() < 1e-3
    dq, dk, dv = hsnf4.attention_bwd(qd, kd, vd, o, lse, to_dev_bf16(do), H, KV)
    torch.cuda.synchronize()
    rdq, rdk, rdv = oracle.attention_bwd(f(q), f(k), f(v), f(do), H, KV, d, sc)
    if T == 1:  # one key: softmax is constant, dq = dk = 0 exactly (GPU: rounding of dP - D)
        for got, ref in ((dq, rdq), (dk, rdk)):
            assert np.abs(ref).max() == 0 and np.abs(bf16_to_f64(got)).max() < 1e-4
    else:
        assert_lora_close(bf16_to_f64(dq), rdq, f"attn dq T{T}")
        assert_lora_close(bf16_to_f64(dk), rdk, f"attn dk T{T}")
    assert_lora_close(bf16_to_f64(dv), rdv, f"attn dv T{T}")
    assert hsnf4.device_status() == 0


def test_attention_deterministic():
    rng = np.random.default_rng(61)
    T, H, KV = 200, 4, 2
    q, k, v, do = (to_dev_bf16(_rand_bf16(rng, (T, n * 128))) for n in (H, KV, KV, H))
    outs = []
    for _ in range(2):
        o, lse = hsnf4.attention_fwd(q, k, v, H, KV)
        outs.append((o, lse) + hsnf4.attention_bwd(q, k, v, o, lse, do, H, KV))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


# ---------------------------------------------------------------- decoder stack

TINY = synth.Family("tiny", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=2)


def _oracle_layers(orc, st, dropout=None, step=0):
    """The stack's weights as oracle layers: the oracle quantizes the seeded
    bf16 weights itself, and the slab the GPU filled must hold those exact
    codes and absmax values."""
    layers = []
    slab = st.slab.numpy()
    for l in range(st.L):
        lin = {}
        base = l * st.layer_bytes
        for p, (name, n, k) in enumerate(st.projs):
            co, ao = st.offs[p]
            codes, absmax = orc.quantize(bf16_bits(st.base_weight_bf16(l, p)))
            assert np.array_equal(slab[base + co: base + co + n * k // 2], codes), (l, name)
            assert np.array_equal(slab[base + ao: base + ao + n * k // 16].view(np.float32),
                                  absmax), (l, name)
            drop = (dropout, st.seed, (step << 32) | (l << 4) | p) if dropout else None
            lin[name] = odec.Linear(n, k, A=bf16_bits(st.A[l][p]), B=bf16_bits(st.B[l][p]),
                                    codes=codes, absmax=absmax, dropout=drop)
        layers.append(odec.Layer(H=st.H, KV=st.KV, d=128, g1=bf16_to_f64(st.g1[l]),
                                 g2=bf16_to_f64(st.g2[l]), lin=lin, alpha=st.alpha))
    return layers


# The composed layer chains about ten bf16 roundings (every module output,
# the gradient sums, and with dropout the second rounding of dX) plus the
# attention kernels' bf16 probabilities, each ~2^-9 / sqrt(3) ~ 1.1e-3
# relative in Frobenius norm, against the oracle's exact modules: sqrt(10)
# x 1.1e-3 ~ 3.5e-3, and the attention backward's bf16 P and dS add about as
# much again.  So the stack's outputs are held to max|d| <= 2e-2 max|ref|
# (as the linear) and a relative Frobenius error of 1e-2.
STACK_FRO = 1e-2


def _stack_close(got, ref, what):
    return assert_lora_close(got, ref, what, fro_rel=STACK_FRO)


@pytest.mark.parametrize("T,dropout", [(96, 0.0), (64, 0.1)])
def test_decoder_stack_vs_oracle(orc, T, dropout):
    st = DecoderStack(TINY, 2, T, streamed=False, block_size=2, dropout=dropout)
    st.step()
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    layers = _oracle_layers(orc, st, dropout or None, step=0)
    h = bf16_to_f64(st.h_in)
    acts = []
    for L in layers:
        s = odec.layer_forward(L, h)
        acts.append(s)
        h = s["h2"]
    _stack_close(bf16_to_f64(st.h_cur), h, "stack output")
    dh = bf16_to_f64(st.dh_top)
    for l in reversed(range(len(layers))):
        dh, grads = odec.layer_backward(layers[l], acts[l], dh)
        for p, name in enumerate(odec.PROJ):
            dA, dB = grads[name]
            _stack_close(st.dA[l][p].cpu().numpy(), dA, f"layer {l} {name} dA")
            _stack_close(st.dB[l][p].cpu().numpy(), dB, f"layer {l} {name} dB")
    _stack_close(bf16_to_f64(st.dh_cur), dh, "stack input gradient")
    st.close()


def _run_stack(st, steps=2):
    rec = {}
    for _ in range(steps):
        rec.clear()
        st.step(lambda l, p, n, t: rec.__setitem__((l, p, n), t.clone()))
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    out = dict(rec)
    out["h_out"] = st.h_cur.clone()
    out["dh_in"] = st.dh_cur.clone()
    for l in range(st.L):
        for p in range(st.P):
            out[(l, p, "dA")] = st.dA[l][p].clone()
            out[(l, p, "dB")] = st.dB[l][p].clone()
    return out


FAM4 = synth.Family("tiny4", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=4)


@pytest.mark.parametrize("dropout", [0.0, 0.05])
def test_decoder_streamed_equals_resident_bitwise(dropout):
    res = DecoderStack(FAM4, 4, 64, streamed=False, block_size=2, dropout=dropout)
    ref = _run_stack(res)
    res.close()
    for bs in (1, 2, 4):
        s = DecoderStack(FAM4, 4, 64, streamed=True, block_size=bs, dropout=dropout)
        got = _run_stack(s)
        s.close()
        for key in ("h_out", "dh_in") + tuple(k for k in ref if isinstance(k, tuple) and
                                             k[2] in ("dA", "dB")):
            assert torch.equal(got[key], ref[key]), (bs, key)


def test_recomputed_forward_equals_forward():
    """The backward's rematerialized layer outputs are the forward's, bit for
    bit; the last block, whose backward follows its forward at once, keeps
    its activations and is not recomputed."""
    s = DecoderStack(FAM4, 4, 64, streamed=True, block_size=2, dropout=0.05)
    rec = {}
    s.step(lambda l, p, n, t: rec.__setitem__((l, n), t.clone()))
    torch.cuda.synchronize()
    for l in range(2):  # block 0
        assert torch.equal(rec[(l, "h_out")], rec[(l, "h_out_recomputed")]), l
    for l in range(2, 4):  # block 1, the last
        assert (l, "h_out_recomputed") not in rec, l
    s.close()
