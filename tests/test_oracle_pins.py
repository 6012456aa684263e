"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test checks the oracle against something the pages or mathematics fix:
closed forms, invariants, special cases with a known exact answer, an
independent fp64 / int64 brute force on tiny inputs, and numbers printed on
the pages (tests/golden/paper_constants.json).  Sources are the MLSys 2026
talk notes on MixLLM (notes.yuuk.io) and the awesome-system-papers summary
page of MixLLM; sections are named per test.
"""
import json
import os

import numpy as np
import pytest

from mixed_precision_quantized_act_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_constants.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ------------------------------------------------------------ fp16 conversion

def test_f16_to_f32_all_patterns(oracle_mod):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle_mod.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_matches_ieee_rne(oracle_mod):
    rng = np.random.default_rng(0)
    parts = [
        rng.standard_normal(200000).astype(np.float32) * np.float32(1000.0),
        (rng.standard_normal(100000) * 1e-5).astype(np.float32),  # subnormal range
        (rng.standard_normal(100000) * 1e-8).astype(np.float32),  # underflow
    ]
    # exact ties between adjacent fp16 values, normal and subnormal
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    parts.append(((lo + hi) / 2).astype(np.float32))
    parts.append(np.array([65504, 65519.99, 65520, 65536, 1e9, -65520, 6e-8, 2.9802322e-08,
                           2.98023259e-08, 0.0, -0.0, np.inf, -np.inf], np.float32))
    x = np.concatenate(parts)
    got = oracle_mod.f32_to_f16(x).view(np.uint16)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ fast I2F

def test_i2f_bias_exhaustive_window(oracle_mod, golden):
    """NOTES §高速 I2F 変換: adding 0x4b400000 and subtracting the float bias
    equals the int->float conversion; the window is exactly [-2^22, 2^22]."""
    assert golden["i2f_bias_bits"]["value"] == "0x4b400000"
    bias_f = np.array([0x4B400000], np.uint32).view(np.float32)[0]
    assert float(bias_f) == 1.5 * 2 ** 23 == 12582912.0
    assert oracle_mod.i2f_mismatches(-(1 << 22), (1 << 22) + 1) == 0
    assert oracle_mod.i2f_mismatches((1 << 22) + 1, (1 << 22) + 2) == 1
    assert oracle_mod.i2f_mismatches(-(1 << 22) - 1, -(1 << 22)) == 1
    # closed form with numpy's own bit reinterpretation
    p = np.arange(-(1 << 22), (1 << 22) + 1, 977, dtype=np.int64)
    v = (p + 0x4B400000).astype(np.uint32).view(np.float32) - np.float32(12582912.0)
    assert np.array_equal(v, p.astype(np.float32))
    # the page's span: a k-element int8 dot product spans 2^16*k; k=128 fits
    k = golden["i2f_safe_group"]["value"]
    assert (1 << 16) * k == 1 << 23  # total span fits the +-2^22 window


# ------------------------------------------------------------ activation quant

def test_act_quant_invariants(oracle_mod):
    layer = wl.TINY
    X = wl.make_x(layer, seed=1)
    A, s = oracle_mod.quantize_act(X)
    x = X.astype(np.float32).reshape(layer.M, layer.G, 128)
    a = A.astype(np.float32).reshape(layer.M, layer.G, 128)
    assert A.min() >= -127 and A.max() <= 127
    assert np.all(np.abs(a).max(axis=2) == 127)  # amax maps to +-127
    err = np.abs(x - s[:, :, None].astype(np.float64) * a)
    assert np.all(err <= s[:, :, None] * 0.5 * (1 + 1e-5))  # + rounding of x/s
    # the scale carries amax at fp32 precision: 127 * s_a gives back amax to
    # within the rounding of the quotient and of the product (a scale rounded
    # to bf16 or fp16, or a divisor other than 127, misses by far more)
    amax = np.abs(x).max(axis=2).astype(np.float64)
    assert np.all(np.abs(127.0 * s.astype(np.float64) - amax) <= amax * 2.0 ** -23)


def test_act_quant_ties_half_even_and_zero_group(oracle_mod):
    x = np.zeros((2, 256), np.float16)
    x[0, 0] = 127.0        # amax = 127 -> s_a = 1 exactly
    x[0, 1:9] = [2.5, 3.5, -2.5, 0.5, 1.5, -1.5, 126.5, -0.5]
    A, s = oracle_mod.quantize_act(x)
    assert s[0, 0] == 1.0  # 127/127
    assert list(A[0, 1:9]) == [2, 4, -2, 0, 2, -2, 126, 0]
    assert s[0, 1] == 0.0 and np.all(A[0, 128:] == 0)   # all-zero group
    assert s[1, 0] == 0.0 and np.all(A[1] == 0)


def test_act_quant_scale_keeps_full_precision(oracle_mod):
    """amax = 100 gives s_a = 100/127 = 0.78740157..., which needs all 24 bits
    of an fp32 significand.  The codes of the values k * (100/127) (their fp16
    roundings) must come back as k for every k: the fp16 rounding moves each
    value by at most 2^-11 of itself, far less than half a step, so the
    quantizer must return k exactly whatever the precision of its arithmetic,
    and s_a itself must be the fp32 quotient to the bit (checked against a
    decimal expansion of 100/127 computed here)."""
    from fractions import Fraction
    ks = np.arange(-127, 128)
    vals = np.array([float(Fraction(100, 127) * int(k)) for k in ks])
    x = np.zeros((1, 256), np.float16)
    x[0, 0] = 100.0
    x[0, 1:1 + len(ks) - 1] = vals[np.arange(len(ks)) != 227].astype(np.float16)  # 227 -> k = 100: amax itself
    A, s = oracle_mod.quantize_act(x[:, :256].reshape(1, 256)[:, :256])
    s0 = s[0, 0]
    # the correctly rounded fp32 value of 100/127, from exact rationals
    exact = Fraction(100, 127)
    cand = [np.float32(float(exact)), np.nextafter(np.float32(float(exact)), np.float32(0)),
            np.nextafter(np.float32(float(exact)), np.float32(2))]
    best = min(cand, key=lambda c: abs(Fraction(float(c)) - exact))
    assert s0 == best
    assert A[0, 0] == 127
    got = A[0, 1:len(ks)].astype(np.int64)
    want = ks[np.arange(len(ks)) != 227]
    assert np.array_equal(got, want)


def _rn_f32(fr):
    """The fp32 value nearest to the rational fr (ties to even), by exact arithmetic."""
    from fractions import Fraction
    f = np.float32(float(fr))  # within one ulp of fr
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    errs = [abs(Fraction(float(c)) - fr) for c in cands]
    m = min(errs)
    best = [c for c, e in zip(cands, errs) if e == m]
    if len(best) > 1:  # a tie: the even significand
        best = [c for c in best if (np.array(c, np.float32).view(np.uint32) & 1) == 0]
    return best[0]


def test_act_quant_scale_is_correctly_rounded(oracle_mod):
    """s_a is amax/127 correctly rounded to fp32 for every group: checked
    against exact rational arithmetic over 3000 fp16 values of amax (random
    bit patterns plus the extremes of the fp16 range)."""
    from fractions import Fraction
    rng = np.random.default_rng(21)
    bits = rng.integers(0x0001, 0x7C00, size=3000).astype(np.uint16)
    bits[:4] = [0x0001, 0x03FF, 0x0400, 0x7BFF]  # smallest subnormal, largest subnormal, smallest normal, 65504
    amax = bits.view(np.float16)
    X = np.zeros((len(amax), 128), np.float16)
    X[:, 5] = amax
    X[:, 9] = -amax / np.float16(3)
    _, s = oracle_mod.quantize_act(X)
    want = np.array([_rn_f32(Fraction(float(a)) / 127) for a in amax], np.float32)
    assert np.array_equal(s[:, 0].view(np.uint32), want.view(np.uint32))


def test_act_quant_lossless_grid(oracle_mod):
    rng = np.random.default_rng(3)
    q = rng.integers(-127, 128, size=(4, 384))
    q[:, ::128] = 127
    q[:, 1::128] = -127
    x = (q * 2.0 ** -3).astype(np.float16)  # exactly representable
    A, s = oracle_mod.quantize_act(x)
    assert np.all(s == 2.0 ** -3)
    assert np.array_equal(A.astype(np.int64), q)


# ------------------------------------------------------------ weight quant

def test_w4_invariants(oracle_mod):
    W = wl.make_w(wl.TINY, seed=2)
    q, z, s = oracle_mod.quantize_w4(W)
    assert q.max() <= 15 and z.max() <= 15
    sf = s.astype(np.float32)
    d = (q.astype(np.float64).reshape(512, 4, 128) - z[:, :, None]) * sf[:, :, None]
    err = np.abs(W.reshape(512, 4, 128) - d)
    # s/2 from rounding, plus at most 15 units of the fp16 rounding of s for
    # codes clamped at the top of the grid
    assert np.all(err <= sf[:, :, None] * (0.5 + 15 * 2.0 ** -11) + 1e-12)
    inner = (q.reshape(512, 4, 128) > 0) & (q.reshape(512, 4, 128) < 15)
    assert np.all(err[inner] <= (sf[:, :, None] * 0.5 * (1 + 1e-5) + 1e-12).repeat(128, 2)[inner])
    qz = q.reshape(512, 4, 128).astype(np.int64) - z[:, :, None]
    assert np.abs(qz).max() <= 15


def test_w4_lossless_grid_and_special_groups(oracle_mod):
    rng = np.random.default_rng(4)
    N, K = 8, 256
    z = rng.integers(0, 16, size=(N, K // 128))
    q = rng.integers(0, 16, size=(N, K))
    q[:, ::128] = 0
    q[:, 1::128] = 15
    sc = 2.0 ** -6
    W = ((q - np.repeat(z, 128, axis=1)) * sc).astype(np.float32)
    # a group with z such that the lowest weight is not below 0 needs z = 0
    W[0, :128] = np.abs(W[0, :128])
    qq, zz, ss = oracle_mod.quantize_w4(W)
    assert np.all(ss.astype(np.float32)[1:] == sc)
    assert np.array_equal(qq[1:].astype(np.int64), q[1:])
    assert np.array_equal(zz[1:].astype(np.int64), z[1:])
    assert zz[0, 0] == 0  # all-positive group
    # all-zero group: scale 0, zero point 0, codes 0
    W2 = np.zeros((1, 128), np.float32)
    q2, z2, s2 = oracle_mod.quantize_w4(W2)
    assert s2[0, 0] == 0 and z2[0, 0] == 0 and not q2.any()


def test_w8_invariants_and_lossless(oracle_mod):
    W = wl.make_w(wl.TINY, seed=5)
    q, s = oracle_mod.quantize_w8(W)
    assert q.min() >= -127 and q.max() <= 127
    sf = s.astype(np.float32)[:, :, None]
    x = W.reshape(512, 4, 128)
    amax = np.abs(x).max(axis=2)[:, :, None]
    err = np.abs(x - sf * q.reshape(512, 4, 128))
    assert np.all(err <= sf * 0.5 + amax * 2.0 ** -10)
    rng = np.random.default_rng(6)
    qi = rng.integers(-127, 128, size=(3, 256))
    qi[:, 0] = 127
    qi[:, 128] = -127
    Wl = (qi * 2.0 ** -9).astype(np.float32)
    q2, s2 = oracle_mod.quantize_w8(Wl)
    assert np.all(s2.astype(np.float32) == 2.0 ** -9)
    assert np.array_equal(q2.astype(np.int64), qi)


# ------------------------------------------------------------ the GEMM

def _brute_force_y64(A, sa, Wq):
    """fp64 dequantize-then-matmul: sum_k (s_a*A_q)(s_w*(W_q - z))."""
    M, K = A.shape
    G = K // 128
    a = A.astype(np.float64) * np.repeat(sa.astype(np.float64), 128, axis=1)
    Y = np.zeros((M, Wq.N))
    if Wq.idx4.size:
        w4 = (Wq.q4.astype(np.float64) - np.repeat(Wq.z4.astype(np.float64), 128, axis=1)) \
            * np.repeat(Wq.s4.astype(np.float64), 128, axis=1)
        Y[:, Wq.idx4] = a @ w4.T
    if Wq.idx8.size:
        w8 = Wq.q8.astype(np.float64) * np.repeat(Wq.s8.astype(np.float64), 128, axis=1)
        Y[:, Wq.idx8] = a @ w8.T
    return Y


def _abs_terms(A, sa, Wq):
    """sum_k |s_a A| |s_w (W_q - z)| -- scale of the fp32 rounding error."""
    a = np.abs(A.astype(np.float64)) * np.repeat(sa.astype(np.float64), 128, axis=1)
    T = np.zeros((A.shape[0], Wq.N))
    if Wq.idx4.size:
        w4 = np.abs(Wq.q4.astype(np.float64) - np.repeat(Wq.z4, 128, axis=1)) \
            * np.repeat(Wq.s4.astype(np.float64), 128, axis=1)
        T[:, Wq.idx4] = a @ w4.T
    if Wq.idx8.size:
        w8 = np.abs(Wq.q8.astype(np.float64)) * np.repeat(Wq.s8.astype(np.float64), 128, axis=1)
        T[:, Wq.idx8] = a @ w8.T
    return T


CASES = [
    ("tiny", wl.TINY, None),
    ("tiny_p0", wl.Linear("t_p0", 16, 512, 512, ((0, 512, 0),), 4), None),
    ("tiny_p100", wl.Linear("t_p100", 16, 512, 512, ((0, 512, 512),), 4), None),
    ("odd", wl.Linear("odd", 3, 77, 384, ((0, 77, 9),), 3), None),
    ("m1", wl.Linear("m1", 1, 40, 256, ((0, 40, 5),), 2), None),
]


@pytest.mark.parametrize("name,layer,_", CASES)
def test_gemm_matches_fp64_brute_force(oracle_mod, name, layer, _):
    X = wl.make_x(layer, seed=0)
    W = wl.make_w(layer, seed=0)
    is8 = wl.make_bitmap(layer, seed=0)
    A, sa = oracle_mod.quantize_act(X)
    Wq = oracle_mod.Quantized(W, is8)
    Y = oracle_mod.gemm_w4w8a8(A, sa, Wq).astype(np.float64)
    Y64 = _brute_force_y64(A, sa, Wq)
    T = _abs_terms(A, sa, Wq)
    G = layer.G
    # fp16 output rounding + fp32 accumulation of G group terms
    bound = 2.0 ** -11 * np.abs(Y64) + (G + 2) * 2.0 ** -23 * T + 2.0 ** -24
    assert np.all(np.abs(Y - Y64) <= bound), np.max(np.abs(Y - Y64) - bound)
    # and the layer output approximates the unquantized product
    ref = X.astype(np.float64) @ W.T.astype(np.float64)
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert rel < 0.15


def test_group_partials_int64_brute_force(oracle_mod):
    layer = wl.Linear("odd2", 5, 70, 384, ((0, 70, 11),), 3)
    X, W, is8 = wl.make_x(layer, 1), wl.make_w(layer, 1), wl.make_bitmap(layer, 1)
    A, sa = oracle_mod.quantize_act(X)
    Wq = oracle_mod.Quantized(W, is8)
    P = oracle_mod.group_partials(A, Wq)
    G = layer.G
    a = A.astype(np.int64).reshape(layer.M, G, 128)
    ref = np.zeros((layer.M, layer.N, G), np.int64)
    w4 = Wq.q4.astype(np.int64).reshape(-1, G, 128) - Wq.z4.astype(np.int64)[:, :, None]
    ref[:, Wq.idx4, :] = np.einsum("mgk,ngk->mng", a, w4)
    w8 = Wq.q8.astype(np.int64).reshape(-1, G, 128)
    ref[:, Wq.idx8, :] = np.einsum("mgk,ngk->mng", a, w8)
    assert np.array_equal(P.astype(np.int64), ref)


def test_partial_bounds_fit_bias_window(oracle_mod):
    """|P| <= 15*127*128 (4-bit) and 127*127*128 (8-bit), both < 2^22, so the
    bias-trick conversion is exact for every reachable partial."""
    X = np.full((1, 128), 3.0, np.float16)
    A, sa = oracle_mod.quantize_act(X)
    assert np.all(A == 127)
    W = np.full((2, 128), 0.01, np.float32)
    W[1] = -0.01
    Wq = oracle_mod.Quantized(W, np.array([0, 0], np.uint8))
    P = oracle_mod.group_partials(A, Wq)
    assert P[0, 0, 0] == 15 * 127 * 128 == 243840
    assert P[0, 1, 0] == -243840
    Wq8 = oracle_mod.Quantized(W, np.array([1, 1], np.uint8))
    P8 = oracle_mod.group_partials(A, Wq8)
    assert P8[0, 0, 0] == 127 * 127 * 128 == 2064512 < 2 ** 22
    assert P8[0, 1, 0] == -2064512


def test_moving_a_channel_changes_only_its_column(oracle_mod):
    layer = wl.TINY
    X, W, is8 = wl.make_x(layer, 2), wl.make_w(layer, 2), wl.make_bitmap(layer, 2)
    A, sa = oracle_mod.quantize_act(X)
    Y0 = oracle_mod.gemm_w4w8a8(A, sa, oracle_mod.Quantized(W, is8))
    c = int(np.flatnonzero(is8 == 0)[7])
    is8b = is8.copy()
    is8b[c] = 1
    Y1 = oracle_mod.gemm_w4w8a8(A, sa, oracle_mod.Quantized(W, is8b))
    diff = np.flatnonzero(np.any(Y0.view(np.uint16) != Y1.view(np.uint16), axis=0))
    assert set(diff.tolist()) <= {c}


# ------------------------------------------------------------ packed layout

def test_packed_nibbles_round_trip(oracle_mod):
    rng = np.random.default_rng(7)
    N4, K = 133, 256  # two tiles of 128 channels, the second one ragged
    q = rng.integers(0, 16, size=(N4, K)).astype(np.uint8)
    P = oracle_mod.pack_w4(q)
    assert P.shape == (2, 2, 128, 64)
    # unpack by the layout's definition: tile t, group g is a [128 rows x 64 B]
    # block; in a run of 32 codes, byte i = (k_i low, k_{i+16} high)
    r = np.zeros((256, K), np.uint8)
    for t in range(2):
        for g in range(2):
            blk = P[t, g]
            lo, hi = blk & 0x0F, blk >> 4
            for run in range(4):
                k0 = g * 128 + run * 32
                r[t * 128:(t + 1) * 128, k0:k0 + 16] = lo[:, run * 16:(run + 1) * 16]
                r[t * 128:(t + 1) * 128, k0 + 16:k0 + 32] = hi[:, run * 16:(run + 1) * 16]
    assert np.array_equal(r[:N4], q)
    assert not r[N4:].any()  # rows past the set are zero
    z = rng.integers(0, 16, size=(5, 2)).astype(np.uint8)
    zp = oracle_mod.pack_zeros(z)
    assert zp.shape == (2, 128)
    assert zp[1, 2] & 0x0F == z[4, 1] and zp[0, 1] >> 4 == z[3, 0]


def test_footprint_matches_paper(oracle_mod, golden):
    """NOTES §ルーフラインモデルによる性能分析: 0.5 + 2.5/G bytes per 4-bit
    weight and 1 + 2/G per 8-bit weight, with the packed layout's arrays."""
    N, K = 512, 1024
    G = K // 128
    q4 = np.zeros((N, K), np.uint8)
    z = np.zeros((N, G), np.uint8)
    s = np.zeros((N, G), np.float16)
    b4 = oracle_mod.pack_w4(q4).nbytes + oracle_mod.pack_zeros(z).nbytes + oracle_mod.pack_scales(s).nbytes
    assert b4 / (N * K) == golden["footprint_w4_asym"]["bytes_per_weight_at_G128"] == 0.5 + 2.5 / 128
    b8 = N * K + oracle_mod.pack_scales(s).nbytes
    assert b8 / (N * K) == golden["footprint_w8_sym"]["bytes_per_weight_at_G128"] == 1 + 2 / 128


# ------------------------------------------------------------ paper numbers

def test_config_table_effective_bits(golden):
    """NOTES §量子化構成の選択: effective bits = 4 + 4 * (8-bit fraction)."""
    for row in golden["quant_configs"]["value"]:
        assert abs(4.0 * (1 - row["frac8"]) + 8.0 * row["frac8"] - row["bits"]) < 1e-9
    fr = {int(l.name.split("_p")[1].split("_")[0]): l.N8 / l.N for l in wl.BIT_MIX}
    assert fr == {0: 0.0, 10: 410 / 4096, 20: 819 / 4096, 50: 0.5, 100: 1.0}


def test_intensity_gains_match_paper(golden):
    """WIKI observation 3: at M=512, N=K=4096, activations 8->4 bit add about
    5.88% arithmetic intensity and weights 8->4 bit about 80%."""
    M, N, K = 512, 4096, 4096

    def ai(a_bits, w_bits):
        return 2 * M * N * K / (M * K * a_bits / 8 + N * K * w_bits / 8)

    g_act = ai(4, 8) / ai(8, 8) - 1
    g_w = ai(8, 4) / ai(8, 8) - 1
    assert round(g_act, 4) == golden["intensity_gain_act_8_to_4"]["value"]
    assert round(g_w, 2) == golden["intensity_gain_w_8_to_4"]["value"]


def test_a100_ridge_point(golden):
    r = golden["a100_roofline"]
    assert round(r["int8_tops"] * 1e12 / (r["hbm_gbs"] * 1e9)) == r["w8a8_ridge_ops_per_byte"]
    assert round(r["int8_tops"] / r["fp32_tflops"]) == r["tc_to_simt_ratio"]
