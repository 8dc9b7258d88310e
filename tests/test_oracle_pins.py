"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a closed form, an invariant, a brute
force computation or a worked example derived by hand (tests/golden/), so that
a plausible mistake in the oracle -- a dropped term, a wrong sign or index, a
transposed operand, a wrong nibble order or rounding mode -- fails here before
the oracle is trusted as the reference of the CUDA path.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int4_weight_quantized_block_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GROUPS = (16, 64, 256)


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(x):
    return inputs.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ---------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("g", GROUPS + (4, 1024))
def test_hadamard_orthonormal_exact(g):
    """H H^T = I exactly: entries are +-2^-k, so every product sum is exact."""
    H = oracle.hadamard(g)
    assert np.array_equal(H @ H.T, np.eye(g))
    assert np.array_equal(H, H.T)


@pytest.mark.parametrize("g", GROUPS + (1024,))
def test_hadamard_walsh_closed_form(g):
    """Sylvester order: H[i, j] = (-1)^popcount(i & j) / sqrt(g)."""
    H = oracle.hadamard(g)
    i = np.arange(g)[:, None]
    j = np.arange(g)[None, :]
    par = np.vectorize(lambda v: bin(v).count("1") & 1)(i & j)
    closed = np.where(par == 1, -1.0, 1.0) / math.sqrt(g)
    assert np.array_equal(H, closed)


@pytest.mark.parametrize("g", GROUPS)
def test_fwht_unit_vectors_are_hadamard_columns(g):
    """FWHT(e_j) is column j of H, exactly (sums of +-1 then a power-of-two scale)."""
    H = oracle.hadamard(g)
    for j in (0, 1, g // 2 - 1, g - 1):
        e = np.zeros(g, np.float32)
        e[j] = 1.0
        assert np.array_equal(oracle.fwht_f32(e).astype(np.float64), H[:, j])


@pytest.mark.parametrize("g", GROUPS + (1024,))
def test_fwht_matches_dense_fp64(g):
    """The fp32 FWHT equals the dense fp64 product H v up to fp32 rounding."""
    r = np.random.default_rng(1)
    H = oracle.hadamard(g)
    for _ in range(20):
        v = r.standard_normal(g).astype(np.float32) * np.float32(r.uniform(0.1, 100))
        ref = H @ v.astype(np.float64)
        got = oracle.fwht_f32(v).astype(np.float64)
        tol = 1e-6 * math.log2(g) * np.abs(v).max()
        assert np.abs(got - ref).max() <= tol


@pytest.mark.parametrize("g", GROUPS + (1024,))
def test_rotation_is_an_involution(g):
    """H is symmetric and orthogonal, so rotating twice gives back the input."""
    r = np.random.default_rng(2)
    x = r.standard_normal((3, 4 * g)).astype(np.float32)
    back = oracle.rotate_rows_f32(oracle.rotate_rows_f32(x, g), g)
    assert np.allclose(back, x, rtol=0, atol=1e-5 * np.abs(x).max())


@pytest.mark.parametrize("g", GROUPS + (1024,))
def test_rotation_leaves_product_unchanged(g):
    """(x R)(W R)^T = x W^T: rotating both operands by the same block rotation
    leaves the product unchanged (to 1e-5 relative in fp32)."""
    r = np.random.default_rng(3)
    K = 4 * g
    x = r.standard_normal((7, K)).astype(np.float32)
    x[:, 3] *= 50
    W = (r.standard_normal((9, K)) * 0.02).astype(np.float32)
    xr = oracle.rotate_rows_f32(x, g).astype(np.float64)
    Wr = oracle.rotate_rows_f32(W, g).astype(np.float64)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    got = xr @ Wr.T
    scale = np.abs(x).max() * np.abs(W).max() * math.sqrt(K)
    assert np.abs(got - ref).max() <= 1e-5 * scale


def test_rotation_acts_blockwise():
    """Each g-block is rotated on its own: a one-hot in block b touches only block b."""
    g, K = 16, 64
    x = np.zeros((1, K), np.float32)
    x[0, 2 * g + 5] = 3.0
    v = oracle.rotate_rows_f32(x, g)[0]
    H = oracle.hadamard(g)
    assert np.all(v[: 2 * g] == 0) and np.all(v[3 * g:] == 0)
    assert np.array_equal(v[2 * g: 3 * g].astype(np.float64), 3.0 * H[:, 5])


# ---------------------------------------------------------------- packing

def test_pack_order_golden():
    d = golden("pack_order.json")
    codes = np.array([d["codes"]], np.int8)
    assert oracle.pack_int4(codes).tolist() == [d["packed"]]
    assert oracle.unpack_int4(np.array([d["packed"]], np.uint8)).tolist() == [d["codes"]]


def test_pack_roundtrip_all_codes():
    allc = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)], np.int8).reshape(1, -1)
    p = oracle.pack_int4(allc)
    assert len(set(p[0].tolist())) == 256          # every byte value occurs once
    assert np.array_equal(oracle.unpack_int4(p), allc)


def test_unpack_pack_roundtrip_random_bytes():
    b = inputs.random_bytes(33, 48)
    assert np.array_equal(oracle.pack_int4(oracle.unpack_int4(b)), b)


# ---------------------------------------------------------------- quantization

def test_rounding_ties_golden():
    d = golden("rounding_ties.json")
    W = np.array([d["w_row"]], np.float32)
    packed, s, codes = oracle.pack_weights(W, 0)
    assert s[0] == np.float32(d["w_scale"])
    assert codes[0].tolist() == d["w_codes"]
    x = bits([d["x_row"]])
    c8, s8, _ = oracle.quantize_act(x, 0, 8)
    assert c8[0].tolist() == d["x_codes_int8"] and s8[0] == 1.0
    c4, s4, p4 = oracle.quantize_act(x, 0, 4)
    assert c4[0].tolist() == d["x_codes_int4"]
    assert np.array_equal(oracle.unpack_int4(p4), c4)


@pytest.mark.parametrize("bits_", (8, 4))
@pytest.mark.parametrize("g", GROUPS)
def test_act_quant_error_bound(g, bits_):
    """|v - q s| <= s/2 per element, where v = H x is computed independently in
    fp64; the largest |v| maps to +-Q; codes stay in [-Q, Q]."""
    Q = 127 if bits_ == 8 else 7
    x = inputs.activations(8, 2 * g, seed=11)
    codes, s, _ = oracle.quantize_act(x, g, bits_)
    H = oracle.hadamard(g)
    xf = oracle.bf16_bits_to_f32(x).astype(np.float64)
    v = (xf.reshape(8, -1, g) @ H.T).reshape(8, -1)
    for m in range(8):
        assert np.all(np.abs(codes[m]) <= Q)
        err = np.abs(v[m] - codes[m].astype(np.float64) * s[m])
        # s/2 from rounding, plus the fp32 rounding of v and s
        assert err.max() <= 0.5 * s[m] * (1 + 1e-5) + 1e-6 * np.abs(v[m]).max()
        assert abs(int(codes[m][np.argmax(np.abs(v[m]))])) == Q
        assert abs(s[m] - np.abs(v[m]).max() / Q) <= 1e-6 * s[m]


@pytest.mark.parametrize("g", GROUPS)
def test_weight_quant_error_bound(g):
    W = inputs.weights(6, 2 * g, seed=12)
    packed, s, codes = oracle.pack_weights(W, g)
    H = oracle.hadamard(g)
    v = (W.astype(np.float64).reshape(6, -1, g) @ H.T).reshape(6, -1)
    for n in range(6):
        err = np.abs(v[n] - codes[n] * np.float64(s[n]))
        assert err.max() <= 0.5 * s[n] * (1 + 1e-5) + 1e-6 * np.abs(v[n]).max()
        assert np.abs(codes[n]).max() == 7
    assert np.array_equal(oracle.unpack_int4(packed), codes)


def test_int8_weight_codes_golden():
    d = golden("w8a8_weight_codes.json")
    codes, s = oracle.quantize_weights_int8(np.array(d["W"], np.float32), d["group"])
    assert codes.tolist() == d["codes"]
    assert s.tolist() == d["row_scale"]


@pytest.mark.parametrize("g", (0,) + GROUPS)
def test_int8_weight_quant_error_bound(g):
    """Rotated rows (an independent fp64 rotation) within s/2 of q s, the
    largest entry of every row at +-127; a one-hot row under group 16 becomes
    16 equal values 1/4, all coded 127."""
    K = 2 * (g or 32)
    W = inputs.weights(6, K, seed=13)
    codes, s = oracle.quantize_weights_int8(W, g)
    if g:
        H = oracle.hadamard(g)
        v = (W.astype(np.float64).reshape(6, -1, g) @ H.T).reshape(6, -1)
    else:
        v = W.astype(np.float64)
    for n in range(6):
        err = np.abs(v[n] - codes[n] * np.float64(s[n]))
        assert err.max() <= 0.5 * s[n] * (1 + 1e-5) + 1e-6 * np.abs(v[n]).max()
        assert np.abs(codes[n]).max() == 127
        assert abs(int(codes[n][np.argmax(np.abs(v[n]))])) == 127
    e = np.zeros((1, 16), np.float32)
    e[0, 0] = 1.0
    c1, s1 = oracle.quantize_weights_int8(e, 16)
    assert np.all(c1 == 127) and s1[0] == np.float32(np.float32(0.25) / np.float32(127))


def test_zero_rows():
    """A zero row has scale 0 and codes 0 (no division by zero)."""
    x = np.zeros((2, 64), np.uint16)
    c, s, _ = oracle.quantize_act(x, 16, 8)
    assert np.all(c == 0) and np.all(s == 0)
    p, sw, cw = oracle.pack_weights(np.zeros((2, 64), np.float32), 64)
    assert np.all(p == 0) and np.all(sw == 0)


def test_onehot_worked_example():
    d = golden("onehot_g16.json")
    g = d["g"]
    x = bits([d["x"]])
    c8, s8, _ = oracle.quantize_act(x, g, 8)
    assert c8[0].tolist() == d["act_codes_int8"]
    c4, s4, _ = oracle.quantize_act(x, g, 4)
    assert c4[0].tolist() == d["act_codes_int4"]
    W = np.array(d["W"], np.float32)
    packed, sw, cw = oracle.pack_weights(W, g)
    assert cw.tolist() == d["w_codes"]
    assert packed.tolist() == d["w_packed"]
    assert np.allclose(sw, d["w_row_scale_exact"], rtol=1e-7)
    acc8 = oracle.gemm_i32(c8, cw)
    assert acc8[0].tolist() == d["acc_int8"]
    acc4 = oracle.gemm_i32(c4, cw)
    assert acc4[0].tolist() == d["acc_int4"]
    y = oracle.bf16_bits_to_f32(oracle.epilogue(acc8, s8, sw))
    assert y[0].tolist() == d["y"]
    y2 = oracle.bf16_bits_to_f32(oracle.convrot_linear(x, packed, sw, g, 8))
    assert y2[0].tolist() == d["y"]
    y3 = oracle.bf16_bits_to_f32(oracle.convrot_linear(x, packed, sw, g, 4))
    assert y3[0].tolist() == d["y"]


# ---------------------------------------------------------------- GEMM

@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 7), (17, 9, 64), (8, 33, 130)])
def test_gemm_brute_force(shape):
    """int32 GEMM == exact integer matmul (numpy int64) on tiny shapes."""
    M, N, K = shape
    a = inputs.random_codes(M, K, -127, 127, seed=5)
    w = inputs.random_codes(N, K, -8, 7, seed=6)
    ref = a.astype(np.int64) @ w.astype(np.int64).T
    assert np.array_equal(oracle.gemm_i32(a, w), ref)


def test_gemm_operand_orientation():
    """acc[m, n] pairs row m of a with row n of w (not a transposed operand)."""
    a = np.zeros((2, 4), np.int8)
    w = np.zeros((3, 4), np.int8)
    a[1, 2] = 5
    w[2, 2] = -3
    acc = oracle.gemm_i32(a, w)
    expect = np.zeros((2, 3), np.int64)
    expect[1, 2] = -15
    assert np.array_equal(acc, expect)


def test_gemm_sampled_matches_full():
    a = inputs.random_codes(20, 96, -127, 127, seed=7)
    w = inputs.random_codes(30, 96, -7, 7, seed=8)
    full = oracle.gemm_i32(a, w)
    pairs = np.array([[0, 0], [19, 29], [5, 17], [11, 3]], np.int64)
    assert np.array_equal(oracle.gemm_i32_sampled(a, w, pairs), full[pairs[:, 0], pairs[:, 1]])


def test_gemm_rejects_int32_overflow():
    a = np.full((1, 140000), 127, np.int8)
    w = np.full((1, 140000), 127, np.int8)
    with pytest.raises(ValueError):
        oracle.gemm_i32(a, w)


# ---------------------------------------------------------------- bf16 rounding / epilogue

def _bf16_nearest_even(v: float) -> float:
    """Brute force: the bf16 value nearest to v, ties to an even mantissa."""
    fv = Fraction(v)
    if v == 0:
        return 0.0
    best = None
    sign = 1 if v > 0 else -1
    e = math.frexp(abs(v))[1]
    cands = []
    for ee in (e - 1, e, e + 1):
        for m in range(128, 256):
            cands.append(Fraction(m) * Fraction(2) ** (ee - 8))
    for c in cands:
        c = c * sign
        d = abs(c - fv)
        key = (d, 0 if (int(abs(c) / Fraction(2) ** (math.frexp(float(abs(c)))[1] - 8)) % 2 == 0) else 1)
        if best is None or key < best[0]:
            best = (key, c)
    return float(best[1])


def test_double_to_bf16_brute_force():
    r = np.random.default_rng(4)
    vals = list(r.standard_normal(300) * 10.0 ** r.integers(-5, 6, 300))
    # exact ties between neighbouring bf16 values (odd mantissa + half ulp)
    vals += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7), 3.0 + 2.0 ** -7]
    for v in vals:
        b = oracle.double_to_bf16_bits(v)
        got = float(oracle.bf16_bits_to_f32(np.array([b], np.uint16))[0])
        assert got == _bf16_nearest_even(float(v)), v


def test_epilogue_closed_form():
    r = np.random.default_rng(5)
    acc = r.integers(-10 ** 6, 10 ** 6, size=(6, 5)).astype(np.int32)
    st = inputs.positive_scales(6, seed=3)
    sr = inputs.positive_scales(5, seed=4)
    bias = bits(r.standard_normal(5))
    y = oracle.bf16_bits_to_f32(oracle.epilogue(acc, st, sr, bias))
    ref = (acc.astype(np.float64) * st.astype(np.float64)[:, None] * sr.astype(np.float64)[None, :]
           + oracle.bf16_bits_to_f32(bias).astype(np.float64)[None, :])
    for m in range(6):
        for n in range(5):
            assert y[m, n] == _bf16_nearest_even(float(ref[m, n]))
    pairs = np.array([[0, 0], [5, 4], [2, 3]], np.int64)
    ys = oracle.epilogue_sampled(acc[pairs[:, 0], pairs[:, 1]], st, sr, pairs, bias)
    assert np.array_equal(ys, oracle.epilogue(acc, st, sr, bias)[pairs[:, 0], pairs[:, 1]])


# ---------------------------------------------------------------- whole layer

@pytest.mark.parametrize("act_bits,rel", [(8, 0.2), (4, 0.3)])
def test_linear_approximates_float_product(act_bits, rel):
    """The quantized layer approximates the plain float product x W^T: the
    error is the quantization noise, far below the signal (a transposed operand,
    a wrong scale or a wrong sign would give an O(1) relative error)."""
    g = 64
    x = inputs.activations(32, 256, seed=21)
    W = inputs.weights(48, 256, seed=22)
    packed, sr, _ = oracle.pack_weights(W, g)
    y = oracle.bf16_bits_to_f32(oracle.convrot_linear(x, packed, sr, g, act_bits)).astype(np.float64)
    ref = oracle.bf16_bits_to_f32(x).astype(np.float64) @ W.astype(np.float64).T
    err = np.sqrt(np.mean((y - ref) ** 2)) / np.sqrt(np.mean(ref ** 2))
    assert err < rel


def test_rotation_reduces_quant_error_with_outliers():
    """With outlier channels, rotating before quantization lowers the activation
    quantization error (the reason the pages rotate): rebuild x from its codes
    (inverse rotation = the same rotation) and compare with and without it."""
    x = inputs.activations(32, 256, seed=23)
    xf = oracle.bf16_bits_to_f32(x).astype(np.float64)
    for act_bits, gain in ((8, 4.0), (4, 1.8)):
        errs = {}
        for g in (0, 256):
            c, s, _ = oracle.quantize_act(x, g, act_bits)
            deq = c.astype(np.float64) * s[:, None].astype(np.float64)
            if g:
                deq = oracle.rotate_rows_f32(deq.astype(np.float32), g).astype(np.float64)
            errs[g] = np.sqrt(np.mean((deq - xf) ** 2))
        assert errs[0] > gain * errs[256]


def test_linear_is_composition():
    g = 16
    x = inputs.activations(5, 64, seed=25)
    W = inputs.weights(7, 64, seed=26)
    packed, sr, cw = oracle.pack_weights(W, g)
    c, st, _ = oracle.quantize_act(x, g, 8)
    y = oracle.epilogue(oracle.gemm_i32(c, oracle.unpack_int4(packed)), st, sr)
    assert np.array_equal(oracle.convrot_linear(x, packed, sr, g, 8), y)


# ---------------------------------------------------------------- W4A16

def test_w4a16_golden():
    d = golden("w4a16_groups.json")
    K, G = d["K"], d["group"]
    q = np.array([[b] * (K // 2) for b in d["row_byte"]], np.uint8)
    z = np.array(d["zero"], np.uint8)
    s = bits(d["scale"])
    x = bits(np.ones((1, K)))
    y = oracle.bf16_bits_to_f32(oracle.w4a16(x, q, s, z, G))
    assert y[0].tolist() == d["y"]


def test_w4a16_reduces_to_plain_matmul():
    """z = 8, s = 1: the layer is x . (q - 8)^T, exactly an integer-weight matmul."""
    M, N, K, G = 3, 10, 256, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=31)
    z = np.full((N, K // G), 8, np.uint8)
    s = bits(np.ones((N, K // G)))
    y = oracle.bf16_bits_to_f32(oracle.w4a16(op.x, op.q, s, z, G)).astype(np.float64)
    lo = (op.q & 0xF).astype(np.int64)
    hi = (op.q >> 4).astype(np.int64)
    qk = np.empty((N, K), np.int64)
    qk[:, 0::2] = lo
    qk[:, 1::2] = hi
    ref = oracle.bf16_bits_to_f32(op.x).astype(np.float64) @ (qk - 8).T.astype(np.float64)
    for m in range(M):
        for n in range(N):
            assert y[m, n] == _bf16_nearest_even(float(ref[m, n]))


def test_w4a16_general_dequant():
    M, N, K, G = 2, 12, 384, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=32)
    y = oracle.bf16_bits_to_f32(oracle.w4a16(op.x, op.q, op.scale, op.zero, G)).astype(np.float64)
    qk = np.empty((N, K), np.float64)
    qk[:, 0::2] = op.q & 0xF
    qk[:, 1::2] = op.q >> 4
    zk = np.repeat(op.zero.astype(np.float64), G, axis=1)
    sk = np.repeat(oracle.bf16_bits_to_f32(op.scale).astype(np.float64), G, axis=1)
    ref = oracle.bf16_bits_to_f32(op.x).astype(np.float64) @ ((qk - zk) * sk).T
    for m in range(M):
        for n in range(N):
            assert y[m, n] == _bf16_nearest_even(float(ref[m, n]))


def test_w4a16_dequant_golden():
    """Worked example of the 16-bit unpack form: each weight rounded to bf16
    (ties to even) before the products; the exact form on the same inputs."""
    d = golden("w4a16_dequant_rounding.json")
    K, G = d["K"], d["group"]
    q = np.array([[b] * (K // 2) for b in d["row_byte"]], np.uint8)
    z = np.array(d["zero"], np.uint8)
    s = bits(d["scale"])
    x = bits(np.ones((1, K)))
    assert oracle.w4a16_dequant_f64(x, q, s, z, G)[0].tolist() == d["y"]
    assert oracle.w4a16_f64(x, q, s, z, G)[0].tolist() == d["y_unrounded_weights"]


def test_w4a16_dequant_equals_exact_form_for_power_of_two_scales():
    """With every scale a power of two, (q - z) * s has at most 4 significant
    bits: the bf16 widening is exact and both forms give the same values."""
    M, N, K, G = 3, 9, 384, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=33)
    rng = np.random.default_rng(34)
    s = bits(np.ldexp(1.0, rng.integers(-12, 4, size=(N, K // G))))
    a = oracle.w4a16_dequant_f64(op.x, op.q, s, op.zero, G)
    b = oracle.w4a16_f64(op.x, op.q, s, op.zero, G)
    assert np.array_equal(a, b)


def test_w4a16_dequant_error_within_half_ulp_bound():
    """Rounding each weight to 8 significant bits moves it by at most 2^-8 of
    its size, so the two forms differ by at most sum_k |x_k| |w_k| 2^-8; on
    general scales they do differ."""
    M, N, K, G = 4, 16, 512, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=35)
    a = oracle.w4a16_dequant_f64(op.x, op.q, op.scale, op.zero, G)
    b = oracle.w4a16_f64(op.x, op.q, op.scale, op.zero, G)
    qk = np.empty((N, K), np.float64)
    qk[:, 0::2] = op.q & 0xF
    qk[:, 1::2] = op.q >> 4
    w = (qk - np.repeat(op.zero.astype(np.float64), G, axis=1)) * \
        np.repeat(oracle.bf16_bits_to_f32(op.scale).astype(np.float64), G, axis=1)
    bound = np.abs(oracle.bf16_bits_to_f32(op.x).astype(np.float64)) @ np.abs(w).T * 2.0 ** -8
    assert np.all(np.abs(a - b) <= bound * (1 + 1e-9))
    assert np.any(a != b)


def test_w4a16_weights_golden():
    """The weights themselves on the worked example: (q - z) s exactly, and
    the bf16 widening (3.0234375 -> 3.03125 by ties to even, 5.0390625 ->
    5.03125, -3.0234375 -> -3.03125)."""
    d = golden("w4a16_dequant_rounding.json")
    K, G = d["K"], d["group"]
    q = np.array([[b] * (K // 2) for b in d["row_byte"]], np.uint8)
    z = np.array(d["zero"], np.uint8)
    s = bits(d["scale"])
    w = oracle.w4a16_weights_f64(q, s, z, G)
    wd = oracle.w4a16_weights_f64(q, s, z, G, widen=True)
    assert w[0, 0] == 3.0234375 and wd[0, 0] == 3.03125
    assert w[1, 0] == 5.0390625 and wd[1, 0] == 5.03125
    assert w[2, 0] == -3.0234375 and wd[2, 0] == -3.03125
    assert w[3, :4].tolist() == [0.0, 3.0, 0.0, 3.0] and w[3, G:G + 2].tolist() == [0.0, 1.0078125]
    # summed over K with x = 1 they give the example's outputs
    assert w.sum(axis=1).tolist() == d["y_unrounded_weights"]
    assert wd.sum(axis=1).tolist() == d["y"]


def test_w4a16_weights_matmul_matches_layer_loops():
    """A library matrix product of x with the weights gives the oracle's
    per-output loops (both forms) up to fp64 rounding."""
    M, N, K, G = 5, 24, 512, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=36)
    x64 = oracle.bf16_bits_to_f32(op.x).astype(np.float64)
    for widen, loops in ((False, oracle.w4a16_f64), (True, oracle.w4a16_dequant_f64)):
        w = oracle.w4a16_weights_f64(op.q, op.scale, op.zero, G, widen=widen)
        ref = loops(op.x, op.q, op.scale, op.zero, G)
        mag = np.abs(x64) @ np.abs(w).T
        assert np.all(np.abs(x64 @ w.T - ref) <= 1e-13 * mag)


def test_tie_capacity_closed_forms():
    """A value exactly at a bf16 rounding midpoint can round either way with
    no evaluation error at all; a value on a bf16 number needs an error of
    half an ulp; a power of two has the finer spacing below it."""
    from oracle.compare import tie_capacity
    mid = 1.0 + 2.0 ** -8                      # midpoint of 1 and 1 + 2^-7
    assert tie_capacity(np.array([mid]), 0.0) == 1.0
    assert tie_capacity(np.array([1.5]), 2.0 ** -9) == 0.0
    assert tie_capacity(np.array([1.5]), 2.0 ** -8) == 1.0
    below = 1.0 - 2.0 ** -9                    # midpoint of 1 - 2^-8 and 1
    assert tie_capacity(np.array([below]), 0.0) == 1.0
    # 1 - 2^-11 rounds to 1; the midpoint below 1 is 3 2^-11 away
    assert tie_capacity(np.array([1.0 - 2.0 ** -11]), 3 * 2.0 ** -11 - 1e-12) == 0.0
    assert tie_capacity(np.array([1.0 - 2.0 ** -11]), 3 * 2.0 ** -11) == 1.0
    assert tie_capacity(np.array([mid, 1.5, 3.0, -mid]), 0.0) == 0.5


def _w4a16_stream_emulation(x_bits, q, scale, zero, G):
    """fp32 emulation of the streaming kernel's order (test of the bound):
    per group S1 = sum x (128 + q), S2 = sum x in fp32 in chunks of 16, then
    T = fma(-(128 + z), S2, S1) and a running fp32 sum of s T."""
    x = oracle.bf16_bits_to_f32(x_bits).astype(np.float32)
    M, K = x.shape
    N = q.shape[0]
    qk = np.empty((N, K), np.float32)
    qk[:, 0::2] = q & 0xF
    qk[:, 1::2] = q >> 4
    s = oracle.bf16_bits_to_f32(scale).astype(np.float32)
    y = np.zeros((M, N), np.float32)
    for j in range(K // G):
        sl = slice(j * G, (j + 1) * G)
        S1 = np.zeros((M, N), np.float32)
        S2 = np.zeros((M, 1), np.float32)
        for c in range(0, G, 16):
            cs = slice(j * G + c, j * G + c + 16)
            S1 = (S1 + (x[:, cs].astype(np.float64) @ (128.0 + qk[:, cs].astype(np.float64)).T)
                  .astype(np.float32)).astype(np.float32)
            S2 = (S2 + x[:, cs].astype(np.float64).sum(axis=1, keepdims=True).astype(np.float32))
        T = (S1.astype(np.float64) - (128.0 + zero[:, j].astype(np.float64)) * S2).astype(np.float32)
        y = (y.astype(np.float64) + s[:, j].astype(np.float64) * T).astype(np.float32)
    return y.astype(np.float64)


def test_w4a16_stream_bound_holds_for_an_fp32_evaluation():
    """The streaming kernel's error bound is not below what an fp32
    evaluation in its order actually makes, on ordinary and extreme tokens;
    and it scales with the offset terms (it is larger than sum |x| |w| alone
    allows)."""
    from oracle.compare import w4a16_stream_error
    M, N, K, G = 3, 40, 1024, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=37)
    x = oracle.bf16_bits_to_f32(op.x).astype(np.float64)
    x[1, 5] = 3.0e4
    x[2, 700] = 1.0e-30
    xb = inputs.f32_to_bf16_bits(x)
    ref = oracle.w4a16_f64(xb, op.q, op.scale, op.zero, G)
    emu = _w4a16_stream_emulation(xb, op.q, op.scale, op.zero, G)
    err = w4a16_stream_error(xb, op.q, op.scale, op.zero, G)
    assert np.all(np.abs(emu - ref) <= err)
    w = oracle.w4a16_weights_f64(op.q, op.scale, op.zero, G)
    assert np.all(err >= (K // G) * 2.0 ** -24 * (np.abs(x) @ np.abs(w).T))


def test_w4a16_tensor_core_bound_holds_for_an_fp32_evaluation():
    """The tcgen05 GEMM's bound against the 16-bit unpack form holds for an
    fp32 evaluation that rounds after every chunk of 16 products."""
    from oracle.compare import w4a16_tc_error
    M, N, K, G = 4, 32, 2048, 128
    op = inputs.w4a16_operands(M, N, K, G, seed=38)
    x = oracle.bf16_bits_to_f32(op.x).astype(np.float64)
    wd = oracle.w4a16_weights_f64(op.q, op.scale, op.zero, G, widen=True)
    acc = np.zeros((M, N), np.float32)
    for c in range(0, K, 16):
        acc = (acc.astype(np.float64) + x[:, c:c + 16] @ wd[:, c:c + 16].T).astype(np.float32)
    ref = x @ wd.T
    assert np.all(np.abs(acc - ref) <= w4a16_tc_error(op.x, wd))


# ---------------------------------------------------------------- fp16 scales

def test_round_f16_matches_ieee_half():
    """The oracle's fp16 rounding against numpy's IEEE half conversion (an
    independent implementation): random magnitudes over and past the whole
    fp16 range, subnormals, ties, and the overflow boundary (65504 stays,
    65520 becomes infinity)."""
    rng = np.random.default_rng(40)
    v = (rng.standard_normal(200000) * np.exp2(rng.uniform(-30, 18, 200000))).astype(np.float32)
    edges = np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
                      3 * 2.0 ** -25, 2.0 ** -14, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11,
                      -(1 + 2.0 ** -11)], np.float32)
    v = np.concatenate([v, edges])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16)
    got = oracle.round_f16(v)
    assert np.array_equal(got.view(np.uint32), ref.astype(np.float32).view(np.uint32))
    assert np.array_equal(oracle.f16_bits(got), ref.view(np.uint16))


def test_fp16_scale_golden():
    """Hand-derived rows where rounding the stored scale to fp16 changes a
    code (tests/golden/fp16_scale_codes.json): group-wise symmetric and
    asymmetric int4, and int8 (W8A8) weights."""
    d = golden("fp16_scale_codes.json")
    K, G = d["K"], d["group"]

    def row(head):
        W = np.zeros((1, K), np.float32)
        W[0, :2] = head
        return W

    for asym, key in ((False, "sym"), (True, "asym")):
        wp, sc, z, codes = oracle.pack_weights_groupwise(row(d["row_" + key]), 0, G, asym,
                                                         scale_f16=True)
        assert codes[0, :2].tolist() == d["codes_" + key] and not codes[0, 2:].any()
        assert sc[0, 0] == d["scale"] and oracle.f16_bits(sc)[0, 0] == d["scale_f16_bits"]
        assert wp[0, 0] == d["byte0_" + key]
        if asym:
            assert z[0, 0] == d["zero_asym"]
        _, sc32, _, codes32 = oracle.pack_weights_groupwise(row(d["row_" + key]), 0, G, asym)
        assert codes32[0, :2].tolist() == d["codes_" + key + "_f32_scale"]
        assert sc32[0, 0] == d["scale_f32"]
    codes, sc = oracle.quantize_weights_int8(row(d["row_int8"]), 0, scale_f16=True)
    assert codes[0, :2].tolist() == d["codes_int8"] and sc[0] == d["scale"]
    codes32, sc32 = oracle.quantize_weights_int8(row(d["row_int8"]), 0)
    assert codes32[0, :2].tolist() == d["codes_int8_f32_scale"] and sc32[0] == d["scale_f32"]


@pytest.mark.parametrize("g", [0, 64, 256])
def test_fp16_scale_quantization_error_bound(g):
    """With the stored fp16 scale s, every weight is within s / 2 of s (q - z)
    (s q for the symmetric forms), the scales lie on the fp16 grid, and the
    extremes still reach the end codes (the fp16 rounding moves a scale by at
    most 2^-11 of itself, far less than half a step of the codes)."""
    N, K = 24, 512
    W = inputs.weights(N, K, seed=41)
    v = oracle.rotate_rows_f32(W.copy(), g).astype(np.float64) if g else W.astype(np.float64)
    for asym in (False, True):
        _, sc, z, codes = oracle.pack_weights_groupwise(W, g, 128, asym, scale_f16=True)
        assert np.array_equal(oracle.round_f16(sc), sc)
        s = np.repeat(sc.astype(np.float64), 128, axis=1)
        zz = np.repeat(z.astype(np.float64), 128, axis=1) if asym else 0.0
        assert np.all(np.abs(v - s * (codes - zz)) <= s / 2 * (1 + 1e-6))
        if not asym:
            assert np.all(np.abs(codes).reshape(N, -1, 128).max(axis=2) == 7)
    codes, sc = oracle.quantize_weights_int8(W, g, scale_f16=True)
    assert np.array_equal(oracle.round_f16(sc), sc)
    assert np.all(np.abs(v - sc[:, None].astype(np.float64) * codes) <= sc[:, None] / 2 * (1 + 1e-6))
    assert np.all(np.abs(codes).max(axis=1) == 127)


# ---------------------------------------------------------------- fp64 outputs and the comparison

def test_unrounded_outputs_round_to_the_bf16_outputs():
    """The bf16 outputs are exactly the fp64 values rounded once."""
    g = 64
    x = inputs.activations(6, 128, seed=41)
    W = inputs.weights(32, 128, seed=42)
    wp, sr, _ = oracle.pack_weights(W, g)
    y64 = oracle.convrot_linear_f64(x, wp, sr, g, 8)
    assert np.array_equal(oracle.round_bf16(y64), oracle.convrot_linear(x, wp, sr, g, 8))
    op = inputs.w4a16_operands(3, 32, 256, 128, seed=43)
    w64 = oracle.w4a16_f64(op.x, op.q, op.scale, op.zero, 128)
    assert np.array_equal(oracle.round_bf16(w64), oracle.w4a16(op.x, op.q, op.scale, op.zero, 128))
    for v in w64.ravel()[:50]:
        assert oracle.double_to_bf16_bits(v) == oracle.round_bf16(np.array([v]))[0]


def test_compare_flags_errors_and_accepts_ties():
    from oracle.compare import check_bf16
    ref = np.array([1.0, 2.0, -3.0, 0.5], np.float64)
    exact = oracle.round_bf16(ref)
    c = check_bf16(exact, ref, 1e-9)
    assert c.ok and c.max_rel == 0 and c.ties == 0
    # a one-ulp difference far from any midpoint is an error, not a tie
    off = exact.copy()
    off[1] += 1
    c = check_bf16(off, ref, 1e-9)
    assert c.ties == 0 and c.max_rel == pytest.approx(2.0 ** -6 / np.sqrt(np.mean(ref ** 2)))
    off[1] += 1                                  # two ulps at 2.0: over the tolerance
    c = check_bf16(off, ref, 1e-9)
    assert c.ties == 0 and c.max_rel > 1e-2 and not c.ok
    # a value sitting on a rounding midpoint: either neighbour is a tie
    mid = 1.0 + 2.0 ** -8                       # halfway between 1 and 1 + 2^-7
    ref2 = np.full(2000, 1.0)
    ref2[0] = mid
    g = oracle.round_bf16(ref2)
    g[0] = oracle.double_to_bf16_bits(1.0 + 2.0 ** -7)   # the other neighbour
    c = check_bf16(g, ref2, 1e-6)
    assert c.ties == 1 and c.max_rel == 0 and c.ok
    # too many ties fail
    ref3 = np.full(100, mid)
    g3 = np.full(100, oracle.double_to_bf16_bits(1.0 + 2.0 ** -7), np.uint16)
    c = check_bf16(g3, ref3, 1e-6)
    assert c.ties == 100 and not c.ok


def test_compare_accepts_2d_inputs_and_error_arrays():
    from oracle.compare import check_bf16, gemm_eval_error
    g = 16
    x = inputs.activations(8, 64, seed=44)
    W = inputs.weights(32, 64, seed=45)
    wp, sr, _ = oracle.pack_weights(W, g)
    y64 = oracle.convrot_linear_f64(x, wp, sr, g, 8)
    y = oracle.convrot_linear(x, wp, sr, g, 8)
    c = check_bf16(y, y64, gemm_eval_error(y64))
    assert c.ok and c.ties == 0 and c.max_rel == 0
    c = check_bf16(y, y64, lambda i: gemm_eval_error(y64.ravel()[i]))   # bound given lazily
    assert c.ok and c.ties == 0
    bias = np.broadcast_to(inputs.f32_to_bf16_bits(np.ones(32)), (8, 32))
    c = check_bf16(y, y64, gemm_eval_error(y64, oracle.bf16_bits_to_f32(bias)))
    assert c.ok


# ------------------------------------------------------------------ group-wise W4A8

def _unpack_nibbles(packed, signed):
    """Independent nibble reader for the group-wise pins (numpy only)."""
    p = np.asarray(packed, np.uint8)
    q = np.empty((p.shape[0], 2 * p.shape[1]), np.int64)
    q[:, 0::2] = p & 0xF
    q[:, 1::2] = p >> 4
    if signed:
        q = np.where(q >= 8, q - 16, q)
    return q


def test_groupwise_weight_codes_golden():
    d = golden("groupwise_weight_codes.json")
    for mode in ("asym", "sym"):
        W = np.array(d["W_" + mode], np.float32)
        packed, s, z, codes = oracle.pack_weights_groupwise(W, d["group"], d["G"],
                                                            asym=(mode == "asym"))
        assert codes.tolist() == d["codes_" + mode]
        assert s.tolist() == d["scale_" + mode]
        if mode == "asym":
            assert z.tolist() == d["zero_asym"]
        else:
            assert z is None
        assert _unpack_nibbles(packed, mode == "sym").tolist() == d["codes_" + mode]


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("g", (0,) + GROUPS)
def test_groupwise_weight_quant_error_bound(g, asym):
    """Rotated rows (an independent fp64 rotation) within s/2 of s (q - z) in
    every group; the group extremes reach the end codes; every code and
    zero point in range."""
    G = 128
    K = 2 * max(g, G)
    W = inputs.weights(5, K, seed=14)
    W[1, :G] = np.abs(W[1, :G])        # a group with no negative value
    W[2, :G] = -np.abs(W[2, :G])       # and one with no positive value
    packed, s, z, codes = oracle.pack_weights_groupwise(W, g, G, asym)
    if g:
        H = oracle.hadamard(g)
        v = (W.astype(np.float64).reshape(5, -1, g) @ H.T).reshape(5, -1)
    else:
        v = W.astype(np.float64)
    q = _unpack_nibbles(packed, not asym)
    assert np.array_equal(q, codes)
    for n in range(5):
        for j in range(K // G):
            vg = v[n, j * G:(j + 1) * G]
            sg = np.float64(s[n, j])
            zg = int(z[n, j]) if asym else 0
            err = np.abs(vg - sg * (q[n, j * G:(j + 1) * G] - zg))
            assert err.max() <= 0.5 * sg * (1 + 1e-5) + 1e-6 * np.abs(vg).max()
            qg = q[n, j * G:(j + 1) * G]
            if asym:
                assert 0 <= qg.min() and qg.max() <= 15 and 0 <= zg <= 15
                assert qg.max() == 15 or qg.min() == 0
            else:
                assert np.abs(qg).max() == 7
    if asym and g == 0:
        assert z[1, 0] == 0 and z[2, 0] == 15


@pytest.mark.parametrize("asym", [False, True])
def test_groupwise_gemm_brute_force(asym):
    """The oracle's GEMM against the product written out with numpy: weights
    dequantized as s (q - z) from an independent nibble reader, an fp64
    matrix product, the token scale and the bias."""
    M, N, K, G = 5, 7, 256, 64
    rng = np.random.default_rng(21)
    a = rng.integers(-127, 128, (M, K)).astype(np.int8)
    st = rng.uniform(0.01, 0.1, M).astype(np.float32)
    W = inputs.weights(N, K, seed=22)
    packed, s, z, _ = oracle.pack_weights_groupwise(W, 0, G, asym)
    bias = inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32))
    y, mag = oracle.gemm_groupwise_f64(a, st, packed, s, z, bias, G)
    q = _unpack_nibbles(packed, not asym).astype(np.float64)
    zz = np.repeat(z.astype(np.float64), G, axis=1) if asym else 0.0
    w = np.repeat(s.astype(np.float64), G, axis=1) * (q - zz)
    b = oracle.bf16_bits_to_f32(bias).astype(np.float64)
    ref = st.astype(np.float64)[:, None] * (a.astype(np.float64) @ w.T) + b
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the magnitude: |s_tok| sum_j |s_j p_j| + |bias|, never below |y|
    p = np.einsum("mjk,njk->mnj", a.astype(np.float64).reshape(M, -1, G),
                  (q - zz).reshape(N, -1, G))
    mref = st.astype(np.float64)[:, None] * np.abs(p * s.astype(np.float64)[None]).sum(-1) + np.abs(b)
    assert np.allclose(mag, mref, rtol=1e-12) and np.all(mag >= np.abs(y) * (1 - 1e-12))
    pairs = np.array([[0, 0], [4, 6], [2, 3], [4, 0]], np.int64)
    ys, ms = oracle.gemm_groupwise_sampled_f64(a, st, packed, s, pairs, z, bias, G)
    assert np.array_equal(ys, y[pairs[:, 0], pairs[:, 1]])
    assert np.array_equal(ms, mag[pairs[:, 0], pairs[:, 1]])


def test_groupwise_gemm_reduces_to_per_row():
    """Symmetric codes with every group scale equal to the row scale: the
    group-wise GEMM is the per-row GEMM and epilogue."""
    M, N, K, G = 4, 6, 512, 128
    rng = np.random.default_rng(23)
    a = rng.integers(-127, 128, (M, K)).astype(np.int8)
    st = rng.uniform(0.01, 0.1, M).astype(np.float32)
    packed, sr, codes = oracle.pack_weights(inputs.weights(N, K, seed=24), 64)
    s = np.repeat(sr[:, None], K // G, axis=1)
    y, _ = oracle.gemm_groupwise_f64(a, st, packed, s, None, None, G)
    ref = oracle.epilogue_f64(oracle.gemm_i32(a, codes), st, sr)
    assert np.allclose(y, ref, rtol=1e-13, atol=0)


def test_groupwise_rejects_bad_shapes():
    W = np.zeros((2, 96), np.float32)
    with pytest.raises(ValueError):
        oracle.pack_weights_groupwise(W, 0, 64, False)     # K % G
    with pytest.raises(ValueError):
        oracle.gemm_groupwise_sampled_f64(np.zeros((2, 128), np.int8), np.ones(2, np.float32),
                                          np.zeros((3, 64), np.uint8), np.ones((3, 1), np.float32),
                                          np.array([[2, 0]], np.int64))
