"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

None of these tests re-types an oracle formula: each one checks a closed
form, an exact round trip, an independent algorithm, a brute-force search
or a finite-difference derivative, chosen so that a plausible mistake in the
oracle (a dropped term, a wrong sign or scale, a transposed operand, a
swapped nibble, a wrong tie-break) fails at least one of them.
"""
import json
import os
import statistics

import numpy as np
import pytest

from host_streamed_nf4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- codebook

def test_codebook_structure(orc):
    cb = orc.codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert np.all(np.diff(cb) > 0), "strictly ascending"
    assert cb[0] == -1.0 and cb[7] == 0.0 and cb[15] == 1.0
    assert (cb < 0).sum() == 7 and (cb > 0).sum() == 8


def _published_codebook():
    """The NF4 values QLoRA prints (Appendix E), from the golden fixture,
    as float32; the decimal strings and the bit patterns must agree."""
    g = json.load(open(os.path.join(GOLDEN, "nf4_codebook.json")))
    vals = np.array([float(v) for v in g["values"]], np.float64)
    f32 = vals.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), vals), "every printed value is a float32"
    bits = np.array([int(b, 16) for b in g["f32_bits"]], np.uint32)
    assert np.array_equal(f32.view(np.uint32), bits)
    return f32


def _construction_codebook():
    """The NormalFloat construction in exact arithmetic, with Python's own
    inverse normal CDF (statistics.NormalDist, a rational-approximation
    algorithm unrelated to the oracle's bisection on erfc)."""
    nd = statistics.NormalDist()
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    top = nd.inv_cdf(delta)
    pos = [nd.inv_cdf(delta + j * (0.5 - delta) / 8.0) / top for j in range(8)]
    neg = [-nd.inv_cdf(delta + j * (0.5 - delta) / 7.0) / top for j in range(7)]
    return np.array(sorted(neg + [0.0] + pos), np.float64)


def test_codebook_is_the_published_table(orc):
    """Bitwise the 16 float32 values of the NF4 data type as published."""
    assert np.array_equal(orc.codebook().view(np.uint32), _published_codebook().view(np.uint32))


def test_published_codebook_follows_the_construction():
    """The published values are the NormalFloat construction carried with the
    probabilities and the last division in single precision: within a few
    float32 ulps (at most 9 here) of the same construction in exact
    arithmetic.  A wrong probability grid, a missing normalisation or a
    swapped side would be off by far more."""
    pub = _published_codebook().astype(np.float64)
    ref = _construction_codebook()
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    ulp[7] = np.spacing(np.float32(0))
    assert np.all(np.abs(pub - ref) <= 10 * ulp), (pub - ref) / ulp
    assert np.max(np.abs(pub - ref)) < 5e-7


def test_oracle_quantile_reproduces_the_construction(orc):
    """The oracle's own quantile routine gives the same construction."""
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    top = orc.normal_quantile(delta)
    pos = [orc.normal_quantile(delta + j * (0.5 - delta) / 8.0) / top for j in range(8)]
    neg = [-orc.normal_quantile(delta + j * (0.5 - delta) / 7.0) / top for j in range(7)]
    got = np.array(sorted(neg + [0.0] + pos), np.float64)
    assert np.allclose(got, _construction_codebook(), rtol=0, atol=1e-13)


def test_normal_quantile_against_stdlib(orc):
    nd = statistics.NormalDist()
    for p in (0.5, 0.55, 0.6, 0.75, 0.9, 0.9677083333333334, 0.99, 1e-6, 0.025):
        assert abs(orc.normal_quantile(p) - nd.inv_cdf(p)) < 1e-12


# ---------------------------------------------------------------- nearest code

def test_nearest_exact_codebook_values(orc):
    cb = orc.codebook()
    for i, c in enumerate(cb):
        assert orc.nearest(c) == i


def test_nearest_tie_goes_to_lower_index(orc):
    cb = orc.codebook()
    # c8/2 is exactly halfway between 0 (code 7) and c8 (both distances are
    # the same fp32 number by Sterbenz), likewise c6/2 between c6 and 0.
    assert orc.nearest(np.float32(cb[8] / 2)) == 7
    assert orc.nearest(np.float32(cb[6] / 2)) == 6


def test_nearest_bruteforce_all_bf16_in_range(orc):
    """Every bf16 value in [-1, 1] maps to a code at minimum distance
    (distances in exact double arithmetic, allowing fp32-rounding ties)."""
    cb = orc.codebook().astype(np.float64)
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    xf = synth.bits_to_f32(bits)
    keep = np.isfinite(xf) & (np.abs(xf) <= 1.0)
    bits, x = bits[keep], xf[keep].astype(np.float64)
    # sample to keep the ctypes loop short, plus the extremes
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([rng.choice(x.size, 6000, replace=False),
                                    np.argsort(np.abs(x))[:50]]))
    d = np.abs(x[idx, None] - cb[None, :])
    dmin = d.min(axis=1)
    for j, i in enumerate(idx):
        code = orc.nearest(np.float32(x[i]))
        # nearest in exact arithmetic, or tied after fp32 rounding
        got = np.float32(d[j, code])
        assert got <= np.float32(dmin[j]) or d[j, code] <= dmin[j] * (1 + 2**-23), (x[i], code)
        # among exact-distance ties the lowest index wins
        ties = np.flatnonzero(np.float32(d[j]) == np.float32(dmin[j]))
        assert code == ties[0]


# ---------------------------------------------------------------- quantize / dequant

def _block_from_codes(rng, cb, a_bits, n_blocks):
    """Blocks whose values are exactly dequant's outputs for random codes at a
    bf16 scale `a`, with one element at +-a so that a is the block absmax."""
    a = synth.bits_to_f32(np.array([a_bits], np.uint16))[0]
    codes = rng.integers(0, 16, size=(n_blocks, 64))
    codes[:, rng.integers(0, 64)] = rng.choice([0, 15])
    vals = cb[codes].astype(np.float32) * np.float32(a)
    return codes, synth.to_bf16_bits(vals), a


def test_roundtrip_codebook_exact_blocks(orc):
    cb = orc.codebook()
    rng = np.random.default_rng(1)
    # power-of-two scales and general bf16 scales, normal range only
    for a in [2.0**m for m in (-12, -6, -1, 0, 3)] + [0.02, 0.3721, 5.5, 117.0]:
        a_bits = synth.to_bf16_bits(np.array([a], np.float32))[0]
        codes, w, a_f = _block_from_codes(rng, cb, a_bits, 8)
        w = w.reshape(8, 64)
        qc, qa = orc.quantize(w)
        assert np.all(qa == np.float32(a_f))
        hi, lo = qc >> 4, qc & 15
        got = np.empty(8 * 64, np.int64)
        got[0::2], got[1::2] = hi, lo
        assert np.array_equal(got, codes.reshape(-1))
        back = orc.dequant(qc, qa, 8, 64)
        assert np.array_equal(back, w)


def test_dequant_code_sweep_is_bf16_of_codebook(orc):
    """codes 0..15 at absmax 1 dequantize to bf16 of the published codebook,
    in order (pins the lookup and the nibble order)."""
    ref = _published_codebook()
    seq = np.tile(np.arange(16), 4)                  # 64 elements
    packed = ((seq[0::2] << 4) | seq[1::2]).astype(np.uint8)
    out = orc.dequant(packed, np.ones(1, np.float32), 1, 64)
    assert np.array_equal(out.reshape(-1), synth.to_bf16_bits(ref[seq]))


def test_all_zero_block(orc):
    w = np.zeros((2, 64), np.uint16)
    w[1] = 0x8000  # -0.0
    codes, absmax = orc.quantize(w)
    assert np.all(codes == 0x77) and np.all(absmax == 0.0)
    out = orc.dequant(codes, absmax, 2, 64)
    assert np.all(out == 0)  # +0.0 bit pattern


def test_nibble_order_even_element_high(orc):
    w = np.zeros((1, 64), np.float32)
    w[0, 0], w[0, 1], w[0, 3] = 1.0, -1.0, 1.0
    codes, absmax = orc.quantize(synth.to_bf16_bits(w))
    assert absmax[0] == 1.0
    assert codes[0] == 0xF0 and codes[1] == 0x7F and codes[2] == 0x77


def test_absmax_is_block_max_abs(orc):
    rng = np.random.default_rng(2)
    w = synth.normal_bf16(rng, (32, 256), 0.02)
    _, absmax = orc.quantize(w)
    ref = np.abs(synth.bits_to_f32(w)).reshape(-1, 64).max(axis=1)
    assert np.array_equal(absmax, ref)


def test_quantize_error_bounded_by_half_gap(orc):
    """|w - deq(w)| <= absmax * (largest half-gap) + bf16 rounding."""
    cb = orc.codebook().astype(np.float64)
    half_gap = np.max(np.diff(cb)) / 2
    rng = np.random.default_rng(3)
    w = synth.normal_bf16(rng, (64, 512), 0.02)
    codes, absmax = orc.quantize(w)
    back = synth.bits_to_f32(orc.dequant(codes, absmax, 64, 512)).astype(np.float64)
    wf = synth.bits_to_f32(w).astype(np.float64)
    a = np.repeat(absmax.astype(np.float64), 64).reshape(64, 512)
    assert np.all(np.abs(wf - back) <= a * half_gap * (1 + 1e-6) + a * 2**-8)


def test_rejects_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.quantize(np.zeros((2, 48), np.uint16))


# ---------------------------------------------------------------- storage format

def test_storage_footprint_matches_pages(orc):
    """0.5 byte/param of codes + one fp32 per 64 params reproduces the host
    footprints the consumer-GPU page prints for the NF4 base."""
    g = json.load(open(os.path.join(GOLDEN, "nf4_host_footprint.json")))
    for fam, quoted in g["quoted_gb"].items():
        f = synth.FAMILIES[fam]
        total = f.layers * sum(orc.storage_bytes(n, k) for _, n, k in f.projections())
        gb = total / 1e9
        assert abs(gb - quoted) / quoted <= g["relative_tolerance"], (fam, gb, quoted)


def test_storage_bytes_equals_buffer_sizes(orc):
    w = np.zeros((128, 192), np.uint16)
    codes, absmax = orc.quantize(w)
    assert codes.nbytes + absmax.nbytes == orc.storage_bytes(128, 192)


# ---------------------------------------------------------------- LoRA forward

def _nf4_from_dense_pm1(W):
    """NF4 codes/absmax for a matrix with entries in {-1, 0, +1}: absmax 1
    per block (0 for all-zero blocks), codes 0 / 7 / 15."""
    N, K = W.shape
    flat = W.reshape(-1)
    codes_full = np.where(flat > 0, 15, np.where(flat < 0, 0, 7))
    packed = ((codes_full[0::2] << 4) | codes_full[1::2]).astype(np.uint8)
    absmax = (np.abs(flat).reshape(-1, 64).max(axis=1)).astype(np.float32)
    return packed, absmax


def test_fwd_permutation_base_no_adapter(orc):
    """W = permutation-like selection, B = 0  =>  Y[t, n] = X[t, pi(n)]."""
    rng = np.random.default_rng(4)
    T, N, K, r = 5, 96, 128, 4
    pi = rng.permutation(K)[:N]
    W = np.zeros((N, K))
    W[np.arange(N), pi] = 1.0
    codes, absmax = _nf4_from_dense_pm1(W)
    X = synth.normal_bf16(rng, (T, K), 1.0)
    A = synth.normal_bf16(rng, (r, K), 0.1)
    B = np.zeros((N, r), np.uint16)
    Y, _ = orc.lora_fwd(codes, absmax, N, K, X, A, B, 32.0)
    assert np.array_equal(Y, synth.bits_to_f32(X)[:, pi])


@pytest.mark.parametrize("alpha,r", [(32.0, 16), (16.0, 16), (8.0, 4), (1.0, 4)])
def test_fwd_adapter_selection_closed_form(orc, alpha, r):
    """W = 0, A selects input columns sigma(j), B routes rank j to output
    tau(j) with weight b_j (powers of two): Y[:, tau(j)] = (alpha/r) b_j X[:, sigma(j)]."""
    rng = np.random.default_rng(5)
    T, N, K = 3, 64, 128
    sigma = rng.permutation(K)[:r]
    tau = rng.permutation(N)[:r]
    b = 2.0 ** rng.integers(-3, 3, size=r)
    A = np.zeros((r, K), np.float32)
    A[np.arange(r), sigma] = 1.0
    B = np.zeros((N, r), np.float32)
    B[tau, np.arange(r)] = b
    codes, absmax = _nf4_from_dense_pm1(np.zeros((N, K)))
    X = synth.normal_bf16(rng, (T, K), 1.0)
    Y, t = orc.lora_fwd(codes, absmax, N, K, X, synth.to_bf16_bits(A), synth.to_bf16_bits(B), alpha)
    Xf = synth.bits_to_f32(X).astype(np.float64)
    ref = np.zeros((T, N))
    ref[:, tau] = (alpha / r) * b[None, :] * Xf[:, sigma]
    assert np.array_equal(Y, ref.astype(np.float32))
    assert np.array_equal(t, Xf[:, sigma].astype(np.float32))


def test_fwd_additive_in_base_and_adapter(orc):
    rng = np.random.default_rng(6)
    c = synth.linear_case(7, 4, 64, 128, r=4)
    codes, absmax = orc.quantize(c.W)
    zero_codes, zero_abs = _nf4_from_dense_pm1(np.zeros((64, 128)))
    Yfull, _ = orc.lora_fwd(codes, absmax, 64, 128, c.X, c.A, c.B, 32.0)
    Ybase, _ = orc.lora_fwd(codes, absmax, 64, 128, c.X, c.A, np.zeros_like(c.B), 32.0)
    Ylora, _ = orc.lora_fwd(zero_codes, zero_abs, 64, 128, c.X, c.A, c.B, 32.0)
    assert np.allclose(Yfull, Ybase.astype(np.float64) + Ylora, rtol=1e-6, atol=1e-6)
    assert not np.allclose(Ylora, 0)


def test_fwd_rows_subset_and_threads_deterministic(orc):
    c = synth.linear_case(8, 16, 128, 192)
    codes, absmax = orc.quantize(c.W)
    Y1, t1 = orc.lora_fwd(codes, absmax, 128, 192, c.X, c.A, c.B, 32.0, n_threads=1)
    Y8, t8 = orc.lora_fwd(codes, absmax, 128, 192, c.X, c.A, c.B, 32.0, n_threads=8)
    rows = np.array([3, 0, 15])
    Ys, _ = orc.lora_fwd(codes, absmax, 128, 192, c.X, c.A, c.B, 32.0, rows=rows, n_threads=3)
    assert np.array_equal(Y1, Y8) and np.array_equal(t1, t8)
    assert np.array_equal(Ys, Y1[rows])


# ---------------------------------------------------------------- LoRA backward

def _fd_case(seed, T=4, N=64, K=64, r=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, K)), rng.standard_normal((T, K)),
            rng.standard_normal((r, K)), rng.standard_normal((N, r)),
            rng.standard_normal((T, N)))


def test_bwd_matches_central_finite_differences(orc):
    """loss = <G, Y(X, A, B)> is linear in X and in B and bilinear in (A, B),
    so central differences are exact up to rounding."""
    W, X, A, B, G = _fd_case(9)
    s = 2.0
    dX, dA, dB = orc.lora_bwd_f64(W, X, A, B, G, s)

    def loss(X_, A_, B_):
        Y, _ = orc.lora_fwd_f64(W, X_, A_, B_, s)
        return float(np.sum(G * Y))

    h = 0.5
    rng = np.random.default_rng(10)
    for name, M, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for _ in range(12):
            idx = tuple(rng.integers(0, d) for d in M.shape)
            P, Mm = M.copy(), M.copy()
            P[idx] += h
            Mm[idx] -= h
            args_p = {"X": (P, A, B), "A": (X, P, B), "B": (X, A, P)}[name]
            args_m = {"X": (Mm, A, B), "A": (X, Mm, B), "B": (X, A, Mm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-9 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_bwd_zero_adapters(orc):
    W, X, A, B, G = _fd_case(11)
    _, _, dB = orc.lora_bwd_f64(W, X, np.zeros_like(A), B, G, 2.0)
    assert np.all(dB == 0)
    dX0, dA, _ = orc.lora_bwd_f64(W, X, A, np.zeros_like(B), G, 2.0)
    assert np.all(dA == 0)
    assert np.allclose(dX0, G @ W, rtol=0, atol=1e-12)  # no adapter => plain dY W


def test_bwd_permutation_base_closed_form(orc):
    """W[n, pi(n)] = 1, B = 0  =>  dX[t, pi(n)] = dY[t, n], other columns 0."""
    rng = np.random.default_rng(12)
    T, N, K, r = 3, 64, 128, 4
    pi = rng.permutation(K)[:N]
    W = np.zeros((N, K))
    W[np.arange(N), pi] = 1.0
    codes, absmax = _nf4_from_dense_pm1(W)
    X = synth.normal_bf16(rng, (T, K), 1.0)
    A = synth.normal_bf16(rng, (r, K), 0.1)
    dY = synth.normal_bf16(rng, (T, N), 1.0)
    dX, dA, dB = orc.lora_bwd(codes, absmax, N, K, X, A, np.zeros((N, r), np.uint16), dY, 32.0)
    ref = np.zeros((T, K), np.float32)
    ref[:, pi] = synth.bits_to_f32(dY)
    assert np.array_equal(dX, ref)
    assert np.all(dA == 0)


def test_bf16_wrapper_equals_fp32_rounding_of_double_core(orc):
    """The NF4/bf16 entry points are the FD-pinned double core on widened
    inputs, rounded once to fp32."""
    c = synth.linear_case(13, 8, 64, 128, r=4)
    codes, absmax = orc.quantize(c.W)
    Wd = synth.bits_to_f32(orc.dequant(codes, absmax, 64, 128)).astype(np.float64)
    f = lambda a: synth.bits_to_f32(a).astype(np.float64)
    Y, t = orc.lora_fwd(codes, absmax, 64, 128, c.X, c.A, c.B, 32.0)
    s = 32.0 / 4
    Yd, td = orc.lora_fwd_f64(Wd, f(c.X), f(c.A), f(c.B), s)
    assert np.array_equal(Y, Yd.astype(np.float32)) and np.array_equal(t, td.astype(np.float32))
    dX, dA, dB = orc.lora_bwd(codes, absmax, 64, 128, c.X, c.A, c.B, c.dY, 32.0)
    dXd, dAd, dBd = orc.lora_bwd_f64(Wd, f(c.X), f(c.A), f(c.B), f(c.dY), s)
    assert np.array_equal(dX, dXd.astype(np.float32))
    assert np.array_equal(dA, dAd.astype(np.float32))
    assert np.array_equal(dB, dBd.astype(np.float32))


# ---------------------------------------------------------------- dense bf16 base

def test_dense_base_equals_nf4_path_on_its_dequantized_weight(orc):
    """The dense-bf16-base entry points on W = deq(codes) give exactly what the
    (FD- and closed-form-pinned) NF4 entry points give on the codes."""
    c = synth.linear_case(21, 6, 128, 192, r=8)
    codes, absmax = orc.quantize(c.W)
    Wd = orc.dequant(codes, absmax, 128, 192)
    Y, t = orc.lora_fwd(codes, absmax, 128, 192, c.X, c.A, c.B, 16.0)
    Yd, td = orc.lora_fwd_bf16w(Wd, c.X, c.A, c.B, 16.0)
    assert np.array_equal(Y, Yd) and np.array_equal(t, td)
    dX, dA, dB = orc.lora_bwd(codes, absmax, 128, 192, c.X, c.A, c.B, c.dY, 16.0)
    dXd, dAd, dBd = orc.lora_bwd_bf16w(Wd, c.X, c.A, c.B, c.dY, 16.0)
    assert np.array_equal(dX, dXd) and np.array_equal(dA, dAd) and np.array_equal(dB, dBd)


def test_dense_base_reads_the_weight_not_a_quantized_copy(orc):
    """A dense weight with values NF4 cannot hold (3/8, 5/8 of the absmax)
    must come through exactly: W = diag(w_i), B = 0  =>  Y[:, i] = w_i X[:, i]."""
    rng = np.random.default_rng(22)
    T, N = 4, 64
    w = np.where(np.arange(N) % 2 == 0, 0.375, 0.625).astype(np.float32)
    W = np.diag(w)
    X = synth.normal_bf16(rng, (T, N), 1.0)
    A = synth.normal_bf16(rng, (8, N), 0.1)
    Y, _ = orc.lora_fwd_bf16w(synth.to_bf16_bits(W), X, A, np.zeros((N, 8), np.uint16), 16.0)
    ref = synth.bits_to_f32(X).astype(np.float64) * w[None, :]
    assert np.array_equal(Y, ref.astype(np.float32))


# ---------------------------------------------------------------- merge_and_unload

def _bf16_of_fraction(q):
    """Exact round-to-nearest-even of a rational to bf16 bits (normal range),
    by integer arithmetic only -- independent of any float rounding."""
    from fractions import Fraction
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    a = abs(Fraction(q))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    m = a / Fraction(2) ** (e - 7)          # 128 <= m < 256
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    if fl == 256:
        fl, e = 128, e + 1
    return sign | ((e + 127) << 7) | (fl - 128)


def test_merge_zero_adapter_is_dequant(orc):
    c = synth.linear_case(23, 1, 128, 256, r=16)
    codes, absmax = orc.quantize(c.W)
    out = orc.lora_merge(c.A, np.zeros_like(c.B), 32.0, codes=codes, absmax=absmax, N=128, K=256)
    assert np.array_equal(out, orc.dequant(codes, absmax, 128, 256))
    Wd = orc.dequant(codes, absmax, 128, 256)
    assert np.array_equal(orc.lora_merge(c.A, np.zeros_like(c.B), 32.0, W=Wd), Wd)


def test_merge_exact_rational_bruteforce(orc):
    """Every element against exact rational arithmetic rounded once: catches a
    transposed operand, a wrong scale, a missing base term or a double
    rounding."""
    from fractions import Fraction
    rng = np.random.default_rng(24)
    N, K, r, alpha = 64, 64, 8, 16.0
    c = synth.linear_case(24, 1, N, K, r=r)
    codes, absmax = orc.quantize(c.W)
    deq = synth.bits_to_f32(orc.dequant(codes, absmax, N, K))
    A = synth.normal_bf16(rng, (r, K), 0.5)
    B = synth.normal_bf16(rng, (N, r), 0.5)
    Af, Bf = synth.bits_to_f32(A), synth.bits_to_f32(B)
    out = orc.lora_merge(A, B, alpha, codes=codes, absmax=absmax, N=N, K=K)
    s = Fraction(alpha) / r
    for n in range(N):
        for k in range(K):
            acc = sum(Fraction(float(Bf[n, j])) * Fraction(float(Af[j, k])) for j in range(r))
            assert out[n, k] == _bf16_of_fraction(Fraction(float(deq[n, k])) + s * acc), (n, k)


def test_merge_rounds_once_at_a_bf16_midpoint(orc):
    """1 + 2^-8 is exactly halfway between bf16 1.0 and 1 + 2^-7: ties go to
    even (1.0).  1 + 2^-8 + 2^-30 is above halfway: it must round up, which
    a float32 intermediate (2^-30 lost) would get wrong."""
    N, K, r = 64, 64, 8
    W = np.full((N, K), 1.0, np.float32)
    A = np.zeros((r, K), np.float32)
    B = np.zeros((N, r), np.float32)
    A[0, :] = 1.0
    A[1, :] = 2.0 ** -24
    B[:, 0] = 2.0 ** -8 / 2.0        # s = 16/8 = 2
    B[: N // 2, 1] = 2.0 ** -7        # rows 0..31: + 2 * 2^-7 * 2^-24 = 2^-30
    out = orc.lora_merge(synth.to_bf16_bits(A), synth.to_bf16_bits(B), 16.0,
                         W=synth.to_bf16_bits(W))
    assert np.all(out[N // 2:] == 0x3F80)   # tie -> even
    assert np.all(out[: N // 2] == 0x3F81)  # just above the tie -> up


# ---------------------------------------------------------------- LoRA dropout

def test_philox_known_answer_vectors(orc):
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        got = orc.philox4x32_10([int(x, 16) for x in v["ctr"]], [int(x, 16) for x in v["key"]])
        assert [f"{int(x):08x}" for x in got] == v["out"]


def test_dropout_mask_follows_its_definition(orc):
    """keep[t, k] from word (e % 4) of the Philox block of e // 4 (e = t K + k)
    and the 24-bit threshold floor(p 2^24); checked on scattered elements with
    the KAT-pinned generator."""
    seed, offset, p, T, K = 0x1234_5678_9ABC_DEF0, (7 << 32) | 3, 0.3, 37, 192
    keep = orc.dropout_keep(seed, offset, p, T, K)
    thr = int(np.float32(p) * np.float32(2.0 ** 24))
    rng = np.random.default_rng(30)
    for _ in range(200):
        t, k = int(rng.integers(T)), int(rng.integers(K))
        e = t * K + k
        q = e >> 2
        w = orc.philox4x32_10([q & 0xFFFFFFFF, q >> 32, offset & 0xFFFFFFFF, offset >> 32],
                              [seed & 0xFFFFFFFF, seed >> 32])[e & 3]
        assert keep[t, k] == int((int(w) >> 8) >= thr), (t, k)


@pytest.mark.parametrize("p", [0.0, 0.05, 0.5, 0.9])
def test_dropout_keep_rate(orc, p):
    T, K = 1024, 1024
    keep = orc.dropout_keep(11, 5, p, T, K)
    n = T * K
    rate = keep.mean()
    sigma = np.sqrt(p * (1 - p) / n)
    assert abs(rate - (1 - p)) <= 6 * sigma + 1e-12
    if p == 0.0:
        assert keep.all()


def test_dropout_masks_differ_across_offsets_and_seeds(orc):
    """Independent streams agree on about p^2 + (1-p)^2 of the elements."""
    p, T, K = 0.5, 512, 512
    a = orc.dropout_keep(1, 0, p, T, K)
    b = orc.dropout_keep(1, 1, p, T, K)
    c = orc.dropout_keep(2, 0, p, T, K)
    for x, y in ((a, b), (a, c), (b, c)):
        agree = (x == y).mean()
        assert abs(agree - 0.5) < 0.01
    assert np.array_equal(a, orc.dropout_keep(1, 0, p, T, K))  # reproducible


def test_dropout_apply_values(orc):
    """Dropped -> +0; kept -> bf16_rne(fp32(x * scale)) with scale =
    fp32(1 / fp32(1 - p)), rounded exactly (rational arithmetic); p = 0 ->
    the input unchanged."""
    from fractions import Fraction
    rng = np.random.default_rng(31)
    T, K, p = 16, 128, 0.05
    X = synth.normal_bf16(rng, (T, K), 1.0)
    assert np.array_equal(orc.dropout_apply(X, 3, 4, 0.0), X)
    out = orc.dropout_apply(X, 3, 4, p)
    keep = orc.dropout_keep(3, 4, p, T, K)
    scale = np.float32(1.0) / (np.float32(1.0) - np.float32(p))
    xf = synth.bits_to_f32(X)
    for t in range(T):
        for k in range(K):
            if not keep[t, k]:
                assert out[t, k] == 0
            else:
                prod = np.float32(xf[t, k]) * scale  # IEEE fp32 multiply (RN)
                assert out[t, k] == _bf16_of_fraction(Fraction(float(prod))), (t, k)


def test_dropout_zero_p_equals_plain_lora(orc):
    c = synth.linear_case(32, 8, 128, 192, r=8)
    codes, absmax = orc.quantize(c.W)
    Y, t = orc.lora_fwd(codes, absmax, 128, 192, c.X, c.A, c.B, 16.0)
    Yd, td = orc.lora_fwd_drop(codes, absmax, 128, 192, c.X, c.A, c.B, 16.0, 0.0, 9, 9)
    assert np.array_equal(Y, Yd) and np.array_equal(t, td)
    g = orc.lora_bwd(codes, absmax, 128, 192, c.X, c.A, c.B, c.dY, 16.0)
    gd = orc.lora_bwd_drop(codes, absmax, 128, 192, c.X, c.A, c.B, c.dY, 16.0, 0.0, 9, 9)
    for a, b in zip(g, gd):
        assert np.array_equal(a, b)


def test_dropout_gradient_matches_finite_differences(orc):
    """With the mask m fixed, Y(X) = X W^T + s ((X * m) A^T) B^T: the loss
    <G, Y> is linear in X, so central differences give dX exactly up to
    rounding -- pinning the masked dX term and dA = s u^T (X * m)."""
    W, X, A, B, G = _fd_case(33, T=4, N=64, K=64, r=2)
    rng = np.random.default_rng(34)
    m = np.where(rng.random(X.shape) < 0.3, 0.0, 1.0 / 0.7)
    s = 2.0
    dX, dA, dB = orc.lora_bwd_f64m(W, X * m, m, A, B, G, s)

    def loss(X_, A_, B_):
        Y, _ = orc.lora_fwd_f64m(W, X_, X_ * m, A_, B_, s)
        return float(np.sum(G * Y))

    h = 0.5
    for name, M, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, d)) for d in M.shape)
            P, Mm = M.copy(), M.copy()
            P[idx] += h
            Mm[idx] -= h
            ap = {"X": (P, A, B), "A": (X, P, B), "B": (X, A, P)}[name]
            am = {"X": (Mm, A, B), "A": (X, Mm, B), "B": (X, A, Mm)}[name]
            fd = (loss(*ap) - loss(*am)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-9 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_dropout_wrapper_is_the_masked_core(orc):
    """The bf16 entry points with dropout are the FD-pinned masked core on
    X_d = dropout_apply(X) and g = keep * scale, rounded once to fp32."""
    c = synth.linear_case(35, 8, 64, 128, r=4)
    p, seed, off = 0.25, 77, 12
    codes, absmax = orc.quantize(c.W)
    Wd = synth.bits_to_f32(orc.dequant(codes, absmax, 64, 128)).astype(np.float64)
    f = lambda a: synth.bits_to_f32(a).astype(np.float64)
    Xd = f(orc.dropout_apply(c.X, seed, off, p))
    g = orc.dropout_keep(seed, off, p, 8, 128) * float(np.float32(1) / (np.float32(1) - np.float32(p)))
    s = 32.0 / 4
    Y, t = orc.lora_fwd_drop(codes, absmax, 64, 128, c.X, c.A, c.B, 32.0, p, seed, off)
    Yc, tc = orc.lora_fwd_f64m(Wd, f(c.X), Xd, f(c.A), f(c.B), s)
    assert np.array_equal(Y, Yc.astype(np.float32)) and np.array_equal(t, tc.astype(np.float32))
    dX, dA, dB = orc.lora_bwd_drop(codes, absmax, 64, 128, c.X, c.A, c.B, c.dY, 32.0, p, seed, off)
    dXc, dAc, dBc = orc.lora_bwd_f64m(Wd, Xd, g, f(c.A), f(c.B), f(c.dY), s)
    assert np.array_equal(dX, dXc.astype(np.float32))
    assert np.array_equal(dA, dAc.astype(np.float32))
    assert np.array_equal(dB, dBc.astype(np.float32))


# ---------------------------------------------------------------- decoder glue

def _fd_check(f, x, grad, n=10, h=1e-4, seed=0, tol=1e-6):
    """Central differences of the scalar f at n random entries of x."""
    rng = np.random.default_rng(seed)
    for _ in range(n):
        idx = tuple(int(rng.integers(0, s)) for s in x.shape)
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (f(xp) - f(xm)) / (2 * h)
        assert abs(fd - grad[idx]) <= tol * max(1.0, abs(fd)), (idx, fd, grad[idx])


def test_rmsnorm_unit_rms_scale_invariance_and_gradient(orc):
    rng = np.random.default_rng(40)
    x = rng.standard_normal((5, 64))
    y = orc.rmsnorm_fwd(x, np.ones(64), 0.0)
    assert np.allclose(np.mean(y * y, axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.allclose(orc.rmsnorm_fwd(7.5 * x, np.ones(64), 0.0), y, rtol=0, atol=1e-12)
    g = rng.standard_normal(64)
    assert np.allclose(orc.rmsnorm_fwd(x, g, 0.0), y * g[None, :], rtol=0, atol=1e-12)
    G = rng.standard_normal((5, 64))
    dx = orc.rmsnorm_bwd(x, g, G, 1e-6)
    _fd_check(lambda x_: float(np.sum(G * orc.rmsnorm_fwd(x_, g, 1e-6))), x, dx, seed=41)


def test_silu_mul_closed_forms_and_gradient(orc):
    a = np.array([0.0, 30.0, -30.0, 1.0])
    b = np.array([2.0, 1.0, 1.0, 1.0])
    m = orc.silu_mul_fwd(a, b)
    assert m[0] == 0.0 and abs(m[1] - 30.0) < 1e-9 and abs(m[2]) < 1e-9
    assert abs(m[3] - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15
    da, db = orc.silu_mul_bwd(a, b, np.ones(4))
    assert da[0] == 0.5 * 2.0 and db[0] == 0.0  # silu'(0) = 1/2, silu(0) = 0
    rng = np.random.default_rng(42)
    A, B, G = (rng.standard_normal((6, 8)) for _ in range(3))
    dA, dB = orc.silu_mul_bwd(A, B, G)
    _fd_check(lambda a_: float(np.sum(G * orc.silu_mul_fwd(a_, B))), A, dA, seed=43)
    _fd_check(lambda b_: float(np.sum(G * orc.silu_mul_fwd(A, b_))), B, dB, seed=44)


def test_attention_special_cases(orc):
    rng = np.random.default_rng(45)
    T, H, KV, d = 6, 4, 2, 8
    q, k, v = (rng.standard_normal((T, n * d)) for n in (H, KV, KV))
    # one token: each head returns its KV head's value
    o1, lse1 = orc.attention_fwd(q[:1], k[:1], v[:1], H, KV, d, 0.3)
    for h in range(H):
        kh = h // (H // KV)
        assert np.allclose(o1[0, h * d:(h + 1) * d], v[0, kh * d:(kh + 1) * d], rtol=0, atol=1e-15)
    # zero queries: uniform weights over the causal prefix -> running mean of v
    o0, lse0 = orc.attention_fwd(np.zeros_like(q), k, v, H, KV, d, 0.3)
    for h in range(H):
        kh = h // (H // KV)
        vh = v[:, kh * d:(kh + 1) * d]
        ref = np.cumsum(vh, axis=0) / np.arange(1, T + 1)[:, None]
        assert np.allclose(o0[:, h * d:(h + 1) * d], ref, rtol=0, atol=1e-13)
        assert np.allclose(lse0[h], np.log(np.arange(1, T + 1)), rtol=0, atol=1e-13)
    # causality: the first i rows do not see tokens after i
    o, _ = orc.attention_fwd(q, k, v, H, KV, d, 0.3)
    k2, v2 = k.copy(), v.copy()
    k2[4:] += 5.0
    v2[4:] -= 3.0
    o2, _ = orc.attention_fwd(q, k2, v2, H, KV, d, 0.3)
    assert np.array_equal(o[:4], o2[:4]) and not np.allclose(o[4:], o2[4:])


def test_attention_gradient_matches_finite_differences(orc):
    rng = np.random.default_rng(46)
    T, H, KV, d, sc = 5, 4, 2, 8, 0.35
    q, k, v = (rng.standard_normal((T, n * d)) for n in (H, KV, KV))
    G = rng.standard_normal((T, H * d))
    dq, dk, dv = orc.attention_bwd(q, k, v, G, H, KV, d, sc)
    loss = lambda q_, k_, v_: float(np.sum(G * orc.attention_fwd(q_, k_, v_, H, KV, d, sc)[0]))
    _fd_check(lambda x: loss(x, k, v), q, dq, seed=47)
    _fd_check(lambda x: loss(q, x, v), k, dk, seed=48)
    _fd_check(lambda x: loss(q, k, x), v, dv, seed=49)


def test_decoder_layer_wiring_matches_finite_differences(orc):
    """The layer composition with exact arithmetic (no bf16 rounding, dense
    double projections) against central differences of <G, h2>: dh0 and
    the adapter gradients of every projection."""
    from oracle import decoder as dec
    rng = np.random.default_rng(50)
    T, hid, H, KV, d, inter, r = 5, 16, 4, 2, 4, 24, 2
    shapes = {"q": (H * d, hid), "k": (KV * d, hid), "v": (KV * d, hid), "o": (hid, H * d),
              "gate": (inter, hid), "up": (inter, hid), "down": (hid, inter)}
    lin = {n: dec.Linear(N, K, A=rng.standard_normal((r, K)) * 0.3,
                         B=rng.standard_normal((N, r)) * 0.3,
                         W=rng.standard_normal((N, K)) / np.sqrt(K))
           for n, (N, K) in shapes.items()}
    layer = dec.Layer(H=H, KV=KV, d=d, g1=1 + 0.1 * rng.standard_normal(hid),
                      g2=1 + 0.1 * rng.standard_normal(hid), lin=lin, alpha=4.0)
    ident = lambda x: x
    h0 = rng.standard_normal((T, hid))
    G = rng.standard_normal((T, hid))
    s = dec.layer_forward(layer, h0, rnd=ident)
    dh0, grads = dec.layer_backward(layer, s, G, rnd=ident)
    loss = lambda: float(np.sum(G * dec.layer_forward(layer, h0_[0], rnd=ident)["h2"]))
    h0_ = [h0]

    def f_h0(x):
        h0_[0] = x
        return loss()
    _fd_check(f_h0, h0, dh0, n=12, seed=51)
    h0_[0] = h0
    for name in dec.PROJ:
        dA, dB = grads[name]
        L = lin[name]
        for M, g in ((L.A, dA), (L.B, dB)):
            base = M.copy()

            def f(x, M=M, base=base):
                M[...] = x
                out = loss()
                M[...] = base
                return out
            _fd_check(f, base, g, n=4, seed=52)
