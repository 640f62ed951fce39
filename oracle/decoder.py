"""Oracle of one decoder layer around the seven LoRA projections.

TEST INFRASTRUCTURE ONLY: imported by tests/ and bench.py's CPU legs, never
by the product path.

The pages train rank-16 LoRA on Qwen2.5 / Llama-3.1 decoder layers and
recompute each block's forward inside the backward (Poros on consumer GPUs,
"OOM playbook": activation memory at the rematerialization boundary; Poros
API reference, patch_hf_model: forward/backward routed through per-block
autograd functions).  The layer is the standard pre-norm decoder layer of
those families, with causal grouped-query attention and no rotary embedding
(an attention stand-in that keeps SDPA's arithmetic):

    a  = rmsnorm(h0; g1)
    q, k, v = lora_q(a), lora_k(a), lora_v(a)
    att = sdpa_causal(q, k, v)              (KV heads shared by H/KV query heads)
    h1 = h0 + lora_o(att)
    b  = rmsnorm(h1; g2)
    m  = silu(lora_gate(b)) * lora_up(b)
    h2 = h1 + lora_down(m)

Backward from dh2 through every module, in the reverse order.  The compute
dtype is bf16 (the workloads' dtype): every module's output, and every sum
of gradient branches, is rounded once to bf16 (`rnd`); inside a module the
arithmetic is the oracle's double.  With `rnd` = identity and dense double
projections the same code is the exact layer, which the tests check against
central finite differences -- pinning the wiring (which tensor feeds which
module, the residual paths, the gradient sums).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import (attention_bwd, attention_fwd, lora_bwd, lora_bwd_drop, lora_fwd, lora_fwd_drop,
               rmsnorm_bwd, rmsnorm_fwd, silu_mul_bwd, silu_mul_fwd, lora_bwd_f64, lora_fwd_f64)

PROJ = ("q", "k", "v", "o", "gate", "up", "down")
EPS = 1e-6


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits: rounded to fp32, then to bf16 (nearest, ties to even)."""
    f = np.ascontiguousarray(np.asarray(x, np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def bits_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rnd_bf16(x: np.ndarray) -> np.ndarray:
    return bits_f64(bf16_bits(x))


@dataclass
class Linear:
    """One LoRA projection: NF4 base (codes, absmax) or a dense double base W;
    adapters A [r, k_in], B [n_out, r] as bf16 bits (NF4) or doubles (dense)."""
    n_out: int
    k_in: int
    A: np.ndarray
    B: np.ndarray
    codes: np.ndarray | None = None
    absmax: np.ndarray | None = None
    W: np.ndarray | None = None
    dropout: tuple | None = None  # (p, seed, offset)


@dataclass
class Layer:
    H: int
    KV: int
    d: int
    g1: np.ndarray  # norm weights (double values of bf16)
    g2: np.ndarray
    lin: dict = field(default_factory=dict)  # name -> Linear
    alpha: float = 32.0


def _fwd(L: Linear, X: np.ndarray, alpha: float):
    """Y (double) and t of one projection on input X (double values)."""
    if L.W is not None:  # exact double layer
        Y, t = lora_fwd_f64(L.W, X, L.A, L.B, alpha / L.A.shape[0])
        return Y, t
    xb = bf16_bits(X)
    if L.dropout:
        p, seed, off = L.dropout
        Y, t = lora_fwd_drop(L.codes, L.absmax, L.n_out, L.k_in, xb, L.A, L.B, alpha, p, seed, off)
    else:
        Y, t = lora_fwd(L.codes, L.absmax, L.n_out, L.k_in, xb, L.A, L.B, alpha)
    return Y.astype(np.float64), t


def _bwd(L: Linear, X: np.ndarray, dY: np.ndarray, alpha: float):
    """dX (double), dA, dB of one projection."""
    if L.W is not None:
        return lora_bwd_f64(L.W, X, L.A, L.B, dY, alpha / L.A.shape[0])
    xb, gb = bf16_bits(X), bf16_bits(dY)
    if L.dropout:
        p, seed, off = L.dropout
        dX, dA, dB = lora_bwd_drop(L.codes, L.absmax, L.n_out, L.k_in, xb, L.A, L.B, gb, alpha, p,
                                   seed, off)
    else:
        dX, dA, dB = lora_bwd(L.codes, L.absmax, L.n_out, L.k_in, xb, L.A, L.B, gb, alpha)
    return dX.astype(np.float64), dA, dB


def layer_forward(layer: Layer, h0: np.ndarray, rnd=rnd_bf16) -> dict:
    """All activations of one layer (doubles holding bf16 values unless
    rnd is the identity).  h0 [T, hidden]."""
    H, KV, d = layer.H, layer.KV, layer.d
    s = {}
    s["h0"] = h0
    s["a"] = rnd(rmsnorm_fwd(h0, layer.g1, EPS))
    for n in ("q", "k", "v"):
        s[n] = rnd(_fwd(layer.lin[n], s["a"], layer.alpha)[0])
    att, _ = attention_fwd(s["q"], s["k"], s["v"], H, KV, d, 1.0 / np.sqrt(d))
    s["att"] = rnd(att)
    s["o"] = rnd(_fwd(layer.lin["o"], s["att"], layer.alpha)[0])
    s["h1"] = rnd(h0 + s["o"])
    s["b"] = rnd(rmsnorm_fwd(s["h1"], layer.g2, EPS))
    s["gate"] = rnd(_fwd(layer.lin["gate"], s["b"], layer.alpha)[0])
    s["up"] = rnd(_fwd(layer.lin["up"], s["b"], layer.alpha)[0])
    s["m"] = rnd(silu_mul_fwd(s["gate"], s["up"]))
    s["dn"] = rnd(_fwd(layer.lin["down"], s["m"], layer.alpha)[0])
    s["h2"] = rnd(s["h1"] + s["dn"])
    return s


def layer_backward(layer: Layer, s: dict, dh2: np.ndarray, rnd=rnd_bf16):
    """(dh0, {name: (dA, dB)}) from the forward's activations s and dh2."""
    H, KV, d = layer.H, layer.KV, layer.d
    al = layer.alpha
    g = {}
    dm, *g["down"] = _bwd(layer.lin["down"], s["m"], dh2, al)
    dm = rnd(dm)
    dgate, dup = silu_mul_bwd(s["gate"], s["up"], dm)
    dgate, dup = rnd(dgate), rnd(dup)
    db_g, *g["gate"] = _bwd(layer.lin["gate"], s["b"], dgate, al)
    db_u, *g["up"] = _bwd(layer.lin["up"], s["b"], dup, al)
    db = rnd(db_g) + rnd(db_u)
    dh1 = rnd(dh2 + rmsnorm_bwd(s["h1"], layer.g2, db, EPS))
    datt, *g["o"] = _bwd(layer.lin["o"], s["att"], dh1, al)
    datt = rnd(datt)
    dq, dk, dv = attention_bwd(s["q"], s["k"], s["v"], datt, H, KV, d, 1.0 / np.sqrt(d))
    da = 0.0
    for n, dy in (("q", rnd(dq)), ("k", rnd(dk)), ("v", rnd(dv))):
        dx, *g[n] = _bwd(layer.lin[n], s["a"], dy, al)
        da = da + rnd(dx)
    dh0 = rnd(dh1 + rmsnorm_bwd(s["h0"], layer.g1, da, EPS))
    return dh0, {n: tuple(v) for n, v in g.items()}
