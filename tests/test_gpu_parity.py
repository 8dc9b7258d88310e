"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every test feeds the same seeded inputs to both sides.  Bars:
  * packed weight bytes and int32 accumulators: bit-exact;
  * activation codes: equal except at rounding ties (<= 1e-4 of elements,
    each off by at most 1) -- both sides decide them in fp32;
  * bf16 outputs: max |gpu - oracle| / rms(oracle) <= 1e-2, where a one-ulp
    difference counts as a rounding tie (not an error) when the oracle's fp64
    value lies within the kernel's fp32 evaluation error of the bf16 rounding
    midpoint; ties must stay below 1e-3 of the outputs (oracle/compare.py).
Small cases span several tiles and ragged tails in M, N and K; a mid-size
case runs several tiles per persistent CTA; the full-size workloads are
checked on every output.
"""
import numpy as np
import pytest
import torch

import oracle
import int4_weight_quantized_block_b200 as t4
from int4_weight_quantized_block_b200 import inputs
from oracle.compare import (check_bf16, gemm_eval_error, tie_capacity, w4a16_stream_error,
                            w4a16_tc_error)
from gpu_util import CODE_MISMATCH_FRAC, bf16_from_gpu, bf16_to_gpu, code_mismatch, dev, to_gpu


def assert_gemm_output(y_gpu_bits, ref64, bias_bits=None):
    b64 = None if bias_bits is None else oracle.bf16_bits_to_f32(bias_bits).astype(np.float64)
    flat = np.asarray(ref64, np.float64).ravel()
    bflat = None if b64 is None else np.broadcast_to(b64, np.shape(ref64)).ravel()

    def err(i):   # the bound where the roundings differ (full-size outputs are large)
        return gemm_eval_error(flat[i], None if bflat is None else bflat[i])

    c = check_bf16(y_gpu_bits, ref64, err)
    assert c.ok, str(c)


pytestmark = pytest.mark.gpu


def assert_w4a16_stream(y_bits, x_bits, q, scale, zero, ref64=None):
    """The streaming W4A16 kernel against the exact layer: per element within
    the bound of its fp32 evaluation order (w4a16_stream_error); a one-ulp
    difference only where the exact value lies within that bound of a bf16
    rounding midpoint."""
    if ref64 is None:
        ref64 = oracle.w4a16_f64(x_bits, q, scale, zero, 128)
    err = w4a16_stream_error(x_bits, q, scale, zero, 128)
    c = check_bf16(y_bits, ref64, err, tie_capacity(ref64, err))
    assert c.ok, str(c)


# ------------------------------------------------------------------ weights

@pytest.mark.parametrize("N,K,g", [(16, 32, 0), (48, 352, 16), (272, 320, 64), (33 * 16, 768, 256),
                                   (256, 256, 256), (64, 16384, 16)])
def test_pack_weights_bit_exact(N, K, g):
    W = inputs.weights(N, K, seed=100 + K)
    W[3, :] = 0.0                                   # an all-zero row
    p_ref, s_ref, _ = oracle.pack_weights(W, g)
    p, s = t4.tint4_pack_weights(to_gpu(W), g)
    torch.cuda.synchronize()
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# ------------------------------------------------------------------ activations

@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,g", [(1, 32, 0), (7, 352, 16), (130, 320, 64), (64, 256, 256),
                                   (33, 3072, 256), (5, 12288, 64), (3, 16384, 256)])
def test_quantize_act(M, K, g, bits):
    x = inputs.activations(M, K, seed=200 + K)
    if M > 2:
        x[2, :] = 0                                  # an all-zero token
    c_ref, s_ref, p_ref = oracle.quantize_act(x, g, bits)
    codes, s = t4.convrot_quantize_act(bf16_to_gpu(x), g, bits)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    if bits == 8:
        frac, dmax = code_mismatch(codes.cpu().numpy(), c_ref)
    else:
        frac, dmax = code_mismatch(oracle.unpack_int4(codes.cpu().numpy()), c_ref)
    assert frac <= CODE_MISMATCH_FRAC and dmax <= 1


# ------------------------------------------------------------------ int32 GEMM

GEMM_SHAPES = [
    (1, 16, 32),        # minimum
    (64, 256, 256),     # the tiny layer
    (200, 272, 352),    # 2 M tiles (ragged), 2 N tiles (ragged 16), 3 K stages (ragged 96)
    (129, 512, 1024),
    (300, 768, 3072),
]


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_int32_accumulators_bit_exact(M, N, K, act_bits):
    Q = 127 if act_bits == 8 else 7
    qa = inputs.random_codes(M, K, -Q, Q, seed=300 + M)
    qw = inputs.random_codes(N, K, -7, 7, seed=301 + N)
    # extreme rows: all +Q against all +7 / -7
    qa[0, :] = Q
    qw[0, :] = 7
    qw[1 % N, :] = -7
    wp = oracle.pack_int4(qw)
    acc_ref = oracle.gemm_i32(qa, qw)
    a = to_gpu(qa) if act_bits == 8 else to_gpu(oracle.pack_int4(qa))
    acc = t4.tint4_debug_int32_gemm(a, act_bits, to_gpu(wp))
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES[1:4])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_bf16_epilogue(M, N, K, act_bits, with_bias):
    Q = 127 if act_bits == 8 else 7
    qa = inputs.random_codes(M, K, -Q, Q, seed=400 + M)
    qw = inputs.random_codes(N, K, -7, 7, seed=401 + N)
    st = inputs.positive_scales(M, seed=402)
    sr = inputs.positive_scales(N, seed=403)
    bias = inputs.f32_to_bf16_bits(np.linspace(-3, 3, N)) if with_bias else None
    y_ref = oracle.epilogue_f64(oracle.gemm_i32(qa, qw), st, sr, bias)
    wp = oracle.pack_int4(qw)
    b = bf16_to_gpu(bias) if with_bias else None
    if act_bits == 8:
        y = t4.w4a8_gemm(to_gpu(qa), to_gpu(st), to_gpu(wp), to_gpu(sr), b)
    else:
        y = t4.w4a4_gemm(to_gpu(oracle.pack_int4(qa)), to_gpu(st), to_gpu(wp), to_gpu(sr), b)
    torch.cuda.synchronize()
    assert_gemm_output(bf16_from_gpu(y), y_ref, np.broadcast_to(bias, (M, N)) if with_bias else None)


# ------------------------------------------------------------------ small-M GEMM
# M <= 16 runs the warp-MMA decode kernel (one pass over the packed weights).

SMALL_M_SHAPES = [
    (1, 16, 32),          # one block, one partial K chunk
    (3, 48, 288),         # odd block count (a half-used last box), K = 256 + 32
    (8, 272, 1088),       # one full token block, 17 blocks, ragged K chunk
    (9, 528, 4096),       # a second token block holding one token
    (16, 1024, 768),      # two full token blocks
    (5, 18960, 64),       # more row blocks than one wave of CTAs takes
    (2, 32, 16384),       # long K: sums of the x16 form near 2^28
]


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K", SMALL_M_SHAPES)
def test_small_m_int32_bit_exact(M, N, K, act_bits):
    Q = 127 if act_bits == 8 else 7
    qa = inputs.random_codes(M, K, -Q, Q, seed=350 + M)
    qw = inputs.random_codes(N, K, -7, 7, seed=351 + N)
    qa[0, :] = Q                                  # extreme sums: +Q against all +7 / all -7
    qw[0, :] = 7
    qw[1 % N, :] = -7
    acc_ref = oracle.gemm_i32(qa, qw)
    a = to_gpu(qa) if act_bits == 8 else to_gpu(oracle.pack_int4(qa))
    acc = t4.tint4_debug_int32_gemm(a, act_bits, to_gpu(oracle.pack_int4(qw)))
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K", SMALL_M_SHAPES[1:5])
@pytest.mark.parametrize("with_bias", [False, True])
def test_small_m_gemm_bf16(M, N, K, act_bits, with_bias):
    test_gemm_bf16_epilogue(M, N, K, act_bits, with_bias)


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_w4a8_full_size(M, act_bits):
    """The decode layer (K = 4096, N = 12288, group 256) through the fused
    linear, every output against the oracle, and the int32 sums bit-exact."""
    w = inputs.WORKLOADS["te_decode_w4a8"]
    N, K, g = w["N"], w["K"], w["group"]
    x = inputs.activations(M, K, seed=inputs.SEED)
    W = inputs.weights(N, K, seed=inputs.SEED)
    wp, sr, qw = oracle.pack_weights(W, g)
    fn = t4.convrot_w4a8_linear if act_bits == 8 else t4.convrot_w4a4_linear
    y = fn(bf16_to_gpu(x), to_gpu(wp), to_gpu(sr), g)
    qa, st, _ = oracle.quantize_act(x, g, act_bits)
    acc_ref = oracle.gemm_i32(qa, qw)
    a = to_gpu(qa) if act_bits == 8 else to_gpu(oracle.pack_int4(qa))
    acc = t4.tint4_debug_int32_gemm(a, act_bits, to_gpu(wp))
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_gemm_output(bf16_from_gpu(y), oracle.epilogue_f64(acc_ref, st, sr, None))


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K,g", [(1, 16, 32, 0), (2, 272, 352, 16), (3, 528, 1088, 64),
                                     (4, 1024, 4096, 256), (1, 12288, 4096, 256), (4, 96, 3840, 64)])
def test_fused_decode_linear(M, N, K, g, act_bits):
    """Decode-sized linears: at M = 1, K <= 4096 the GEMM kernel rotates and
    quantizes x itself (same codes as the separate rotate+quantize), larger M
    take the two launches; all against the oracle, with a bias."""
    x = inputs.activations(M, K, seed=830 + K)
    if M > 1:
        x[1, :] = 0                                 # an all-zero token
    W = inputs.weights(N, K, seed=831 + N)
    wp, sr, _ = oracle.pack_weights(W, g)
    bias = inputs.f32_to_bf16_bits(np.linspace(-2, 2, N))
    y_ref = oracle.convrot_linear_f64(x, wp, sr, g, act_bits, bias)
    fn = t4.convrot_w4a8_linear if act_bits == 8 else t4.convrot_w4a4_linear
    y = fn(bf16_to_gpu(x), to_gpu(wp), to_gpu(sr), g, bf16_to_gpu(bias))
    torch.cuda.synchronize()
    assert_gemm_output(bf16_from_gpu(y), y_ref, np.broadcast_to(bias, (M, N)))


@pytest.mark.parametrize("prefetch", [False, True])
def test_decode_weight_prefetch_switch(prefetch):
    """With the decode weight streaming switched on, the small-M kernels give
    the same bits: the activations (written by the kernel just before, the
    rotate + quantize of the fused linear) are still read after the wait."""
    M, N, K, g = 4, 2048, 1024, 256
    x = inputs.activations(M, K, seed=810)
    W = inputs.weights(N, K, seed=811)
    wp, sr, qw = oracle.pack_weights(W, g)
    op = inputs.w4a16_operands(M, N, K, 128, seed=812)
    xg, wpg, srg = bf16_to_gpu(x), to_gpu(wp), to_gpu(sr)
    q16, s16, z16, x16 = to_gpu(op.q), bf16_to_gpu(op.scale), to_gpu(op.zero), bf16_to_gpu(op.x)
    try:
        t4.tint4_set_decode_weight_prefetch(prefetch)
        outs = []
        for _ in range(3):   # back to back on one stream: each call follows a kernel
            outs.append((t4.convrot_w4a8_linear(xg, wpg, srg, g),
                         t4.convrot_w4a4_linear(xg, wpg, srg, g),
                         t4.w4a16_gemv_gemm(x16, q16, s16, z16, 128)))
        torch.cuda.synchronize()
    finally:
        t4.tint4_set_decode_weight_prefetch(False)
    y8, y4, y16 = (bf16_from_gpu(o) for o in outs[-1])
    for o in outs[:-1]:
        assert np.array_equal(bf16_from_gpu(o[0]), y8)
        assert np.array_equal(bf16_from_gpu(o[2]), y16)
    assert_gemm_output(y8, oracle.convrot_linear_f64(x, wp, sr, g, 8))
    assert_gemm_output(y4, oracle.convrot_linear_f64(x, wp, sr, g, 4))
    assert_w4a16_stream(y16, op.x, op.q, op.scale, op.zero)


# ------------------------------------------------------------------ fused linear

@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K,g", [(64, 256, 256, 256), (200, 272, 320, 64),
                                     (33, 512, 768, 16), (129, 256, 1024, 256)])
def test_convrot_linear_small(M, N, K, g, act_bits):
    x = inputs.activations(M, K, seed=500 + K)
    W = inputs.weights(N, K, seed=501 + N)
    wp, sr, _ = oracle.pack_weights(W, g)
    y_ref = oracle.convrot_linear_f64(x, wp, sr, g, act_bits)
    fn = t4.convrot_w4a8_linear if act_bits == 8 else t4.convrot_w4a4_linear
    y = fn(bf16_to_gpu(x), to_gpu(wp), to_gpu(sr), g)
    torch.cuda.synchronize()
    assert_gemm_output(bf16_from_gpu(y), y_ref)


@pytest.mark.parametrize("act_bits", [8, 4])
@pytest.mark.parametrize("M,N,K,g", [(17, 272, 320, 64), (200, 1040, 1024, 16),
                                     (333, 256, 768, 256)])
def test_fused_linear_even_odd_codes_match_gemm(M, N, K, g, act_bits):
    """Past the small-M kernel the fused linears keep their workspace codes in
    the tensor-core GEMM's even/odd K order; every fused entry gives, bit for
    bit, the output of the quantize entry followed by the GEMM entry (natural
    order codes), which the other tests hold to the oracle."""
    x = bf16_to_gpu(inputs.activations(M, K, seed=540 + M))
    wp, sr = t4.tint4_pack_weights(to_gpu(inputs.weights(N, K, seed=541 + N)), g)
    b = bf16_to_gpu(inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32)))
    codes, st = t4.convrot_quantize_act(x, g, act_bits)
    if act_bits == 8:
        y0 = t4.w4a8_gemm(codes, st, wp, sr, b)
        y1 = t4.convrot_w4a8_linear(x, wp, sr, g, b)
        y2 = t4.convrot_w4a8_linear_noalloc(x, wp, sr, g, b)
        y3 = t4.convrot_w4a8_linear_grouped(x, [(wp, sr, b, None)], g)[0]
        ys = (y1, y2, y3)
    else:
        y0 = t4.w4a4_gemm(codes, st, wp, sr, b)
        ys = (t4.convrot_w4a4_linear(x, wp, sr, g, b),)
    if act_bits == 8:
        # the test entry runs the same GEMM launch on codes permuted here
        ys += (t4.tint4_debug_w4a8_gemm_even_odd(t4.even_odd_codes(codes), st, wp, sr, b),)
    torch.cuda.synchronize()
    for y in ys:
        assert torch.equal(y, y0)


def test_quantized_linear_module_end_to_end():
    """Weights packed on the GPU, layer run on the GPU, both against the oracle."""
    M, N, K, g = 96, 320, 512, 64
    x = inputs.activations(M, K, seed=77)
    W = inputs.weights(N, K, seed=78)
    lin = t4.QuantizedLinear.from_float(to_gpu(W), g, act_bits=8)
    y = lin(bf16_to_gpu(x))
    wp, sr, _ = oracle.pack_weights(W, g)
    torch.cuda.synchronize()
    assert np.array_equal(lin.w_packed.cpu().numpy(), wp)
    assert_gemm_output(bf16_from_gpu(y), oracle.convrot_linear_f64(x, wp, sr, g, 8))


@pytest.mark.parametrize("name", ["dit_qkv_w4a8", "dit_qkv_w4a4", "dit_mlp_up_w4a8",
                                  "dit_mlp_down_w4a8"])
def test_full_size_workloads(name):
    """The full-size layers, every element: weights packed on the GPU
    (bit-exact against the oracle), activation codes and token scales, the
    fused linear's output against the oracle's epilogue of its exact int32
    sums, and those int32 sums themselves (bit-exact) from the GEMM that the
    persistent kernel runs over many tiles per CTA."""
    w = inputs.WORKLOADS[name]
    M, N, K, g, bits = w["M"], w["N"], w["K"], w["group"], w["act_bits"]
    x, W = inputs.layer_inputs(name)
    wp_ref, sr_ref, qw_ref = oracle.pack_weights(W, g)
    wp, sr = t4.tint4_pack_weights(to_gpu(W), g)
    codes, st = t4.convrot_quantize_act(bf16_to_gpu(x), g, bits)
    fn = t4.convrot_w4a8_linear if bits == 8 else t4.convrot_w4a4_linear
    y = fn(bf16_to_gpu(x), wp, sr, g)
    torch.cuda.synchronize()
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(sr.cpu().numpy().view(np.uint32), sr_ref.view(np.uint32))
    qa_ref, st_ref, _ = oracle.quantize_act(x, g, bits)
    qa_gpu = codes.cpu().numpy() if bits == 8 else oracle.unpack_int4(codes.cpu().numpy())
    frac, dmax = code_mismatch(qa_gpu, qa_ref)
    assert frac <= CODE_MISMATCH_FRAC and dmax <= 1
    assert np.array_equal(st.cpu().numpy().view(np.uint32), st_ref.view(np.uint32))
    acc = oracle.gemm_i32(qa_ref, qw_ref)
    assert_gemm_output(bf16_from_gpu(y), oracle.epilogue_f64(acc, st_ref, sr_ref))
    # int32 accumulators of the same codes, bit-exact everywhere
    a = to_gpu(qa_ref) if bits == 8 else to_gpu(oracle.pack_int4(qa_ref))
    acc_gpu = t4.tint4_debug_int32_gemm(a, bits, to_gpu(wp_ref))
    torch.cuda.synchronize()
    assert np.array_equal(acc_gpu.cpu().numpy(), acc)
    if bits == 4:
        # the packed-code GEMM entries on the same codes: every output
        y4 = t4.w4a4_gemm(a, to_gpu(st_ref), to_gpu(wp_ref), to_gpu(sr_ref))
        y4w = t4.w4a4_gemm_widened(a, to_gpu(st_ref), to_gpu(wp_ref), to_gpu(sr_ref))
        torch.cuda.synchronize()
        ref = oracle.epilogue_f64(acc, st_ref, sr_ref)
        assert_gemm_output(bf16_from_gpu(y4), ref)
        assert np.array_equal(bf16_from_gpu(y4w), bf16_from_gpu(y4))


@pytest.mark.parametrize("M,N,K", [(9, 272, 512), (17, 144, 256), (300, 768, 3072),
                                   (2048, 8192, 1024)])
def test_w4a4_gemm_widened(M, N, K):
    """Packed int4 codes widened once into a workspace, then the int8
    tensor-core GEMM: the bits of w4a4_gemm, which the oracle holds."""
    g = 256
    x = inputs.activations(M, K, seed=1400 + M)
    W = inputs.weights(N, K, seed=1401)
    wp, sr, qw = oracle.pack_weights(W, g)
    qa, st, packed = oracle.quantize_act(x, g, 4)
    b = inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32))
    a, stg, wpg, srg, bg = to_gpu(packed), to_gpu(st), to_gpu(wp), to_gpu(sr), bf16_to_gpu(b)
    y = t4.w4a4_gemm(a, stg, wpg, srg, bg)
    yw = t4.w4a4_gemm_widened(a, stg, wpg, srg, bg)
    yw2 = t4.w4a4_gemm_widened(a, stg, wpg, srg, bg)   # the workspace holds the last call's codes
    torch.cuda.synchronize()
    assert np.array_equal(bf16_from_gpu(yw), bf16_from_gpu(y))
    assert np.array_equal(bf16_from_gpu(yw2), bf16_from_gpu(y))
    assert_gemm_output(bf16_from_gpu(yw), oracle.epilogue_f64(oracle.gemm_i32(qa, qw), st, sr, b), b)


@pytest.mark.parametrize("bits", [8, 4])
def test_many_tiles_per_cta(bits):
    """A mid-size layer (2000 tokens, 12288 weight rows, K 1024), every
    element: 768 tiles of 128 x 256 for int8 codes (5 or 6 per persistent CTA,
    the single accumulator handed back and forth each tile, the last token
    tile ragged) and 1056 tiles of 128 x 192 for packed codes (7 or 8 per CTA,
    both accumulator buffers reused); each CTA crosses tile boundaries in its
    rings several times.  int32 sums bit-exact (packed and int8 codes), the
    fused linear and the GEMM entries against the oracle."""
    M, N, K, g = 2000, 12288, 1024, 256
    x = inputs.activations(M, K, seed=1300 + bits)
    W = inputs.weights(N, K, seed=1310)
    wp, sr, qw = oracle.pack_weights(W, g)
    qa, st, packed = oracle.quantize_act(x, g, bits)
    acc = oracle.gemm_i32(qa, qw)
    a = to_gpu(qa) if bits == 8 else to_gpu(packed)
    acc_gpu = t4.tint4_debug_int32_gemm(a, bits, to_gpu(wp))
    fn = t4.convrot_w4a8_linear if bits == 8 else t4.convrot_w4a4_linear
    y = fn(bf16_to_gpu(x), to_gpu(wp), to_gpu(sr), g)
    gemm = t4.w4a8_gemm if bits == 8 else t4.w4a4_gemm
    y2 = gemm(a, to_gpu(st), to_gpu(wp), to_gpu(sr))
    torch.cuda.synchronize()
    assert np.array_equal(acc_gpu.cpu().numpy(), acc)
    ref = oracle.epilogue_f64(acc, st, sr)
    assert_gemm_output(bf16_from_gpu(y), ref)
    assert np.array_equal(bf16_from_gpu(y), bf16_from_gpu(y2))


# ------------------------------------------------------------------ W8A8

@pytest.mark.parametrize("N,K,g", [(16, 32, 0), (272, 320, 64), (256, 4096, 256), (48, 352, 16)])
def test_quantize_weights_int8_bit_exact(N, K, g):
    W = inputs.weights(N, K, seed=150 + K)
    W[2, :] = 0.0
    c_ref, s_ref = oracle.quantize_weights_int8(W, g)
    c, s = t4.tint4_quantize_weights_int8(to_gpu(W), g)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), c_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("M,N,K,g", [(1, 256, 256, 256), (17, 272, 320, 64), (200, 1040, 1024, 16),
                                     (385, 128, 4096, 256)])
def test_w8a8_gemm_and_linear(M, N, K, g):
    x = inputs.activations(M, K, seed=160 + M)
    wc, sr = oracle.quantize_weights_int8(inputs.weights(N, K, seed=161 + N), g)
    codes, st, _ = oracle.quantize_act(x, g, 8)
    b = inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32))
    y = t4.w8a8_gemm(to_gpu(codes), to_gpu(st), to_gpu(wc), to_gpu(sr), bf16_to_gpu(b))
    yl = t4.convrot_w8a8_linear(bf16_to_gpu(x), to_gpu(wc), to_gpu(sr), g)
    torch.cuda.synchronize()
    acc = oracle.gemm_i32(codes, wc)
    assert_gemm_output(bf16_from_gpu(y), oracle.epilogue_f64(acc, st, sr, b), b)
    assert_gemm_output(bf16_from_gpu(yl), oracle.epilogue_f64(acc, st, sr))


def test_w8a8_full_size():
    """The DiT QKV layer as W8A8: all weight codes and scales bit-exact, every
    output against the oracle."""
    w = inputs.WORKLOADS["dit_qkv_w4a8"]
    M, N, K, g = w["M"], w["N"], w["K"], w["group"]
    x, W = inputs.layer_inputs("dit_qkv_w4a8")
    wc_ref, sr_ref = oracle.quantize_weights_int8(W, g)
    wc, sr = t4.tint4_quantize_weights_int8(to_gpu(W), g)
    y = t4.convrot_w8a8_linear(bf16_to_gpu(x), wc, sr, g)
    torch.cuda.synchronize()
    assert np.array_equal(wc.cpu().numpy(), wc_ref)
    assert np.array_equal(sr.cpu().numpy().view(np.uint32), sr_ref.view(np.uint32))
    qa_ref, st_ref, _ = oracle.quantize_act(x, g, 8)
    acc = oracle.gemm_i32(qa_ref, wc_ref)
    assert_gemm_output(bf16_from_gpu(y), oracle.epilogue_f64(acc, st_ref, sr_ref))


# ------------------------------------------------------------------ grouped GEMM

@pytest.mark.parametrize("M", [8, 200])
def test_gemm_grouped_matches_separate_calls(M):
    """One grouped launch over three weight matrices (Q, K, V of different
    widths) gives each group exactly the bits of its own w4a8_gemm, and those
    match the oracle."""
    K, g = 512, 64
    Ns = (1024, 256, 272)
    x = inputs.activations(M, K, seed=700 + M)
    codes, st, _ = oracle.quantize_act(x, g, 8)
    cg, sg = to_gpu(codes), to_gpu(st)
    groups, ref = [], []
    for i, N in enumerate(Ns):
        wp, sr, _ = oracle.pack_weights(inputs.weights(N, K, seed=710 + i), g)
        b = inputs.f32_to_bf16_bits(np.linspace(-0.5, 0.5, N, dtype=np.float32)) if i == 1 else None
        groups.append((to_gpu(wp), to_gpu(sr), None if b is None else bf16_to_gpu(b), None))
        ref.append((wp, sr, b))
    ys = t4.w4a8_gemm_grouped(cg, sg, groups)
    singles = [t4.w4a8_gemm(cg, sg, w, sr, b) for (w, sr, b, _) in groups]
    torch.cuda.synchronize()
    for y, y1, (wp, sr, b) in zip(ys, singles, ref):
        assert np.array_equal(bf16_from_gpu(y), bf16_from_gpu(y1))
        acc = oracle.gemm_i32(codes, oracle.unpack_int4(wp))
        y64 = oracle.epilogue_f64(acc, st, sr, b)
        assert_gemm_output(bf16_from_gpu(y), y64, b)


@pytest.mark.parametrize("M", [1, 64, 333])
def test_linear_grouped(M):
    K, g = 768, 256
    Ns = (512, 128)
    x = inputs.activations(M, K, seed=720 + M)
    groups, ref = [], []
    for i, N in enumerate(Ns):
        wp, sr, _ = oracle.pack_weights(inputs.weights(N, K, seed=730 + i), g)
        groups.append((to_gpu(wp), to_gpu(sr), None, None))
        ref.append((wp, sr))
    ys = t4.convrot_w4a8_linear_grouped(bf16_to_gpu(x), groups, g)
    torch.cuda.synchronize()
    for y, (wp, sr) in zip(ys, ref):
        assert_gemm_output(bf16_from_gpu(y), oracle.convrot_linear_f64(x, wp, sr, g, 8))


def test_gemm_grouped_full_size_qkv_split():
    """The DiT QKV layer with its 9216 weight rows split into separate Q, K
    and V matrices: the grouped launch reproduces the concatenated GEMM's
    columns bit for bit (that GEMM is itself held to the oracle)."""
    w = inputs.WORKLOADS["dit_qkv_w4a8"]
    M, N, K, g = w["M"], w["N"], w["K"], w["group"]
    x_np, W_np = inputs.layer_inputs("dit_qkv_w4a8")
    x = bf16_to_gpu(x_np)
    wp, sr = t4.tint4_pack_weights(torch.from_numpy(W_np).to(dev()), g)
    codes, st = t4.convrot_quantize_act(x, g, 8)
    y = t4.w4a8_gemm(codes, st, wp, sr)
    third = N // 3
    parts = [(wp[i * third:(i + 1) * third].contiguous(), sr[i * third:(i + 1) * third].contiguous(),
              None, None) for i in range(3)]
    ys = t4.w4a8_gemm_grouped(codes, st, parts)
    torch.cuda.synchronize()
    for i, yg in enumerate(ys):
        assert torch.equal(yg, y[:, i * third:(i + 1) * third])


# ------------------------------------------------------------------ group-wise W4A8

def assert_groupwise_output(y_gpu_bits, y64, mag, K):
    """bf16 outputs against the oracle: the fp32 evaluation (one rounding per
    weight group in a running sum, up to 16 partial sums added at the end by
    the streaming kernel, then the token scale and the bias) is within
    (K / 128 + 19) 2^-24 of the size of the terms it adds up."""
    err = (K // t4.WEIGHT_GROUP + 19) * 2.0 ** -24 * mag
    c = check_bf16(y_gpu_bits, y64, err)
    assert c.ok, str(c)


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("N,K,g", [(16, 128, 0), (48, 384, 16), (272, 640, 64), (400, 1024, 256)])
def test_pack_weights_groupwise_bit_exact(N, K, g, asym):
    W = inputs.weights(N, K, seed=800 + K)
    W[0, :128] = np.abs(W[0, :128])     # a group with no negative value
    W[1, :128] = -np.abs(W[1, :128])    # and one with no positive value
    W[2, 128:256 if K >= 256 else 128] = 0.0
    wp_ref, s_ref, z_ref, _ = oracle.pack_weights_groupwise(W, g, 128, asym)
    wp, s, z = t4.tint4_pack_weights_groupwise(to_gpu(W), g, asym)
    torch.cuda.synchronize()
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    if asym:
        assert np.array_equal(z.cpu().numpy(), z_ref)
    else:
        assert z is None


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (5, 272, 384), (130, 144, 256), (300, 400, 1024),
                                   (129, 128, 2048)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_groupwise(M, N, K, asym, with_bias):
    """Tiles, ragged M / N tails and 1 to 16 weight groups per row."""
    x = inputs.activations(M, K, seed=810 + M)
    codes, st, _ = oracle.quantize_act(x, 64, 8)
    wp, s, z, _ = oracle.pack_weights_groupwise(inputs.weights(N, K, seed=811 + N), 64, 128, asym)
    b = (inputs.f32_to_bf16_bits(np.linspace(-2, 2, N, dtype=np.float32)) if with_bias else None)
    y = t4.w4a8_gemm_groupwise(to_gpu(codes), to_gpu(st), to_gpu(wp), to_gpu(s),
                               to_gpu(z) if asym else None, bf16_to_gpu(b) if with_bias else None)
    torch.cuda.synchronize()
    y64, mag = oracle.gemm_groupwise_f64(codes, st, wp, s, z, b)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("M,N,K,g", [(1, 256, 256, 256), (17, 272, 384, 64), (200, 528, 1024, 16)])
def test_linear_groupwise(M, N, K, g, asym):
    """The fused linear (codes in the private even/odd order) gives the bits
    of quantize + GEMM (natural order), which match the oracle."""
    x_np = inputs.activations(M, K, seed=820 + M)
    x = bf16_to_gpu(x_np)
    wp, s, z = t4.tint4_pack_weights_groupwise(to_gpu(inputs.weights(N, K, seed=821 + N)), g, asym)
    b = bf16_to_gpu(inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32)))
    codes, st = t4.convrot_quantize_act(x, g, 8)
    y0 = t4.w4a8_gemm_groupwise(codes, st, wp, s, z, b)
    y1 = t4.convrot_w4a8_linear_groupwise(x, wp, s, g, z, b)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    qa, st_ref, _ = oracle.quantize_act(x_np, g, 8)
    frac, dmax = code_mismatch(codes.cpu().numpy(), qa)
    assert frac <= CODE_MISMATCH_FRAC and dmax <= 1
    y64, mag = oracle.gemm_groupwise_f64(codes.cpu().numpy(), st.cpu().numpy(), wp.cpu().numpy(),
                                         s.cpu().numpy(), None if z is None else z.cpu().numpy(),
                                         b.view(torch.int16).cpu().numpy().view(np.uint16))
    assert_groupwise_output(bf16_from_gpu(y1), y64, mag, K)


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_groupwise_decode_full_size(M, asym):
    """The text-encoder decode layer (K 4096, N 12288) with group-wise weights
    at 1, 4 and 16 tokens (the streaming kernel): every output against the
    oracle."""
    w = inputs.WORKLOADS["te_decode_w4a8"]
    N, K, g = w["N"], w["K"], w["group"]
    _, W = inputs.layer_inputs("te_decode_w4a8", M=1)
    x = inputs.activations(M, K, seed=840 + M)
    codes, st, _ = oracle.quantize_act(x, g, 8)
    wp, s, z, _ = oracle.pack_weights_groupwise(W, g, 128, asym)
    y = t4.w4a8_gemm_groupwise(to_gpu(codes), to_gpu(st), to_gpu(wp), to_gpu(s),
                               to_gpu(z) if asym else None)
    zg = to_gpu(z) if asym else None
    y1 = t4.convrot_w4a8_linear_groupwise(bf16_to_gpu(x), to_gpu(wp), to_gpu(s), g, zg)
    cg, sg = t4.convrot_quantize_act(bf16_to_gpu(x), g, 8)
    y2 = t4.w4a8_gemm_groupwise(cg, sg, to_gpu(wp), to_gpu(s), zg)
    torch.cuda.synchronize()
    y64, mag = oracle.gemm_groupwise_f64(codes, st, wp, s, z)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("asym", [False, True])
def test_groupwise_module_end_to_end(asym):
    """Weights packed on the GPU by the module, layer run on the GPU, both
    against the oracle (M spans a ragged tensor-core tile)."""
    M, N, K, g = 150, 272, 640, 64
    x = inputs.activations(M, K, seed=850)
    W = inputs.weights(N, K, seed=851)
    lin = t4.GroupwiseQuantizedLinear.from_float(to_gpu(W), g, asym=asym)
    y = lin(bf16_to_gpu(x))
    torch.cuda.synchronize()
    wp, s, z, _ = oracle.pack_weights_groupwise(W, g, 128, asym)
    assert np.array_equal(lin.w_packed.cpu().numpy(), wp)
    qa, st, _ = oracle.quantize_act(x, g, 8)
    y64, mag = oracle.gemm_groupwise_f64(qa, st, wp, s, z)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)


@pytest.mark.parametrize("M,N,K", [(4, 144, 12288), (40, 128, 128)])
def test_groupwise_routing_edges(M, N, K):
    """A small M with K past the streaming kernel's 8192 (the tensor-core
    kernel then runs it), and a single weight group (K = 128) at M > 16."""
    x = inputs.activations(M, K, seed=860 + K)
    codes, st, _ = oracle.quantize_act(x, 0, 8)
    wp, s, z, _ = oracle.pack_weights_groupwise(inputs.weights(N, K, seed=861), 0, 128, True)
    y = t4.w4a8_gemm_groupwise(to_gpu(codes), to_gpu(st), to_gpu(wp), to_gpu(s), to_gpu(z))
    y1 = t4.convrot_w4a8_linear_groupwise(bf16_to_gpu(x), to_gpu(wp), to_gpu(s), 0, to_gpu(z))
    torch.cuda.synchronize()
    y64, mag = oracle.gemm_groupwise_f64(codes, st, wp, s, z)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)
    assert_groupwise_output(bf16_from_gpu(y1), y64, mag, K)


def test_groupwise_equal_scales_match_per_row_gemm():
    """Symmetric group-wise weights whose group scales all equal the row
    scale compute the per-row W4A8 layer (same codes): outputs within the
    two kernels' evaluation bounds of each other."""
    M, N, K, g = 256, 384, 1024, 64
    x = bf16_to_gpu(inputs.activations(M, K, seed=830))
    wp, sr = t4.tint4_pack_weights(to_gpu(inputs.weights(N, K, seed=831)), g)
    s = sr[:, None].expand(N, K // 128).contiguous()
    codes, st = t4.convrot_quantize_act(x, g, 8)
    y_gw = t4.w4a8_gemm_groupwise(codes, st, wp, s)
    y_row = t4.w4a8_gemm(codes, st, wp, sr)
    torch.cuda.synchronize()
    d = (y_gw.float() - y_row.float()).abs().max().item()
    assert d <= 2 * 2.0 ** -8 * y_row.float().abs().max().item()


def test_groupwise_full_size():
    """The DiT QKV layer with asymmetric group-wise weights at full size:
    packing bit-exact, every output of the fused linear against the oracle."""
    name = "dit_qkv_w4a8_asym_g128"
    w = inputs.WORKLOADS[name]
    M, N, K, g = w["M"], w["N"], w["K"], w["group"]
    x_np, W = inputs.layer_inputs(name)
    wp_ref, s_ref, z_ref, _ = oracle.pack_weights_groupwise(W, g, 128, True)
    wp, s, z = t4.tint4_pack_weights_groupwise(to_gpu(W), g, True)
    x = bf16_to_gpu(x_np)
    y = t4.convrot_w4a8_linear_groupwise(x, wp, s, g, z)
    codes, st = t4.convrot_quantize_act(x, g, 8)
    torch.cuda.synchronize()
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(z.cpu().numpy(), z_ref)
    y64, mag = oracle.gemm_groupwise_f64(codes.cpu().numpy(), st.cpu().numpy(), wp_ref, s_ref,
                                         z_ref)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)


# ------------------------------------------------------------------ fp16 weight scales
# ("ComfyUI-INT-Crush", "Weight Format": the stored scales are fp16)

def _f16_to_gpu(scale_f32):
    """Oracle scales (float32 on the fp16 grid) -> a float16 device tensor."""
    return torch.from_numpy(np.ascontiguousarray(scale_f32).astype(np.float16)).to(dev())


def _fixture_rows(N, K):
    """Weights whose first rows hold the hand-derived cases where the fp16
    rounding of a scale changes a code (tests/golden/fp16_scale_codes.json)."""
    import json
    import os
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "fp16_scale_codes.json")))
    W = inputs.weights(N, K, seed=840 + K)
    for r, key in enumerate(("row_sym", "row_asym", "row_int8")):
        W[r, :] = 0.0
        W[r, :2] = d[key]
    W[3, :] = 1e-9           # scales below fp16's smallest subnormal: 0
    return W


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("N,K,g", [(16, 128, 0), (48, 384, 16), (272, 640, 64), (400, 1024, 256)])
def test_pack_weights_groupwise_f16_bit_exact(N, K, g, asym):
    W = _fixture_rows(N, K)
    wp_ref, s_ref, z_ref, _ = oracle.pack_weights_groupwise(W, g, 128, asym, scale_f16=True)
    wp, s, z = t4.tint4_pack_weights_groupwise(to_gpu(W), g, asym, scale_dtype=torch.float16)
    torch.cuda.synchronize()
    assert s.dtype == torch.float16
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), oracle.f16_bits(s_ref))
    if asym:
        assert np.array_equal(z.cpu().numpy(), z_ref)


@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (9, 272, 384), (130, 144, 256), (300, 400, 1024)])
def test_gemm_and_linear_groupwise_f16(M, N, K, asym):
    """GEMM (streaming and tensor-core kernels) and fused linear with fp16
    group scales against the oracle on the same fp16 scales."""
    g = 64
    x = inputs.activations(M, K, seed=850 + M)
    codes, st, _ = oracle.quantize_act(x, g, 8)
    wp, s, z, _ = oracle.pack_weights_groupwise(_fixture_rows(N, K), g, 128, asym, scale_f16=True)
    zg = to_gpu(z) if asym else None
    y = t4.w4a8_gemm_groupwise(to_gpu(codes), to_gpu(st), to_gpu(wp), _f16_to_gpu(s), zg)
    yl = t4.convrot_w4a8_linear_groupwise(bf16_to_gpu(x), to_gpu(wp), _f16_to_gpu(s), g, zg)
    torch.cuda.synchronize()
    y64, mag = oracle.gemm_groupwise_f64(codes, st, wp, s, z)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)
    assert_groupwise_output(bf16_from_gpu(yl), y64, mag, K)


@pytest.mark.parametrize("N,K,g", [(16, 128, 0), (272, 320, 64), (256, 4096, 256), (48, 352, 16)])
def test_quantize_weights_int8_f16_bit_exact(N, K, g):
    W = _fixture_rows(N, K)
    c_ref, s_ref = oracle.quantize_weights_int8(W, g, scale_f16=True)
    c, s = t4.tint4_quantize_weights_int8(to_gpu(W), g, scale_dtype=torch.float16)
    torch.cuda.synchronize()
    assert s.dtype == torch.float16
    assert np.array_equal(c.cpu().numpy(), c_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), oracle.f16_bits(s_ref))


@pytest.mark.parametrize("M,N,K,g", [(1, 256, 256, 256), (17, 272, 320, 64), (385, 128, 4096, 256)])
def test_w8a8_f16_gemm_and_linear(M, N, K, g):
    x = inputs.activations(M, K, seed=860 + M)
    wc, sr = oracle.quantize_weights_int8(inputs.weights(N, K, seed=861 + N), g, scale_f16=True)
    codes, st, _ = oracle.quantize_act(x, g, 8)
    b = inputs.f32_to_bf16_bits(np.linspace(-1, 1, N, dtype=np.float32))
    y = t4.w8a8_gemm(to_gpu(codes), to_gpu(st), to_gpu(wc), _f16_to_gpu(sr), bf16_to_gpu(b))
    yl = t4.convrot_w8a8_linear(bf16_to_gpu(x), to_gpu(wc), _f16_to_gpu(sr), g)
    torch.cuda.synchronize()
    acc = oracle.gemm_i32(codes, wc)
    assert_gemm_output(bf16_from_gpu(y), oracle.epilogue_f64(acc, st, sr, b), b)
    assert_gemm_output(bf16_from_gpu(yl), oracle.epilogue_f64(acc, st, sr))


def test_groupwise_f16_full_size():
    """The DiT QKV layer with asymmetric group-wise weights in the pages'
    stored format (fp16 scales): packing bit-exact, every output of the fused
    linear against the oracle."""
    name = "dit_qkv_w4a8_asym_g128"
    w = inputs.WORKLOADS[name]
    M, N, K, g = w["M"], w["N"], w["K"], w["group"]
    x_np, W = inputs.layer_inputs(name)
    wp_ref, s_ref, z_ref, _ = oracle.pack_weights_groupwise(W, g, 128, True, scale_f16=True)
    wp, s, z = t4.tint4_pack_weights_groupwise(to_gpu(W), g, True, scale_dtype=torch.float16)
    x = bf16_to_gpu(x_np)
    y = t4.convrot_w4a8_linear_groupwise(x, wp, s, g, z)
    codes, st = t4.convrot_quantize_act(x, g, 8)
    torch.cuda.synchronize()
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), oracle.f16_bits(s_ref))
    assert np.array_equal(z.cpu().numpy(), z_ref)
    y64, mag = oracle.gemm_groupwise_f64(codes.cpu().numpy(), st.cpu().numpy(), wp_ref, s_ref,
                                         z_ref)
    assert_groupwise_output(bf16_from_gpu(y), y64, mag, K)


# ------------------------------------------------------------------ W4A16

@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (4, 272, 384), (16, 512, 1024),
                                   (9, 128, 4096), (32, 64, 256), (17, 96, 512),
                                   (16, 2400, 1024), (3, 12288, 256)])
def test_w4a16(M, N, K):
    op = inputs.w4a16_operands(M, N, K, 128, seed=600 + M)
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(op.x), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), 128)
    torch.cuda.synchronize()
    assert_w4a16_stream(bf16_from_gpu(y), op.x, op.q, op.scale, op.zero)


@pytest.mark.parametrize("M", [1, 9])
def test_w4a16_extreme_token_values(M):
    """Token values far from the rest (tiny, and beyond the fp16 range) in a
    few groups, against the oracle."""
    N, K = 256, 2048
    op = inputs.w4a16_operands(M, N, K, 128, seed=820 + M)
    x = oracle.bf16_bits_to_f32(op.x).reshape(M, K).astype(np.float64)
    x[0, 300] = 3.0e-7          # pair 1: below fp16's exact range
    x[0, 1700] = 1.0e-30        # pair 6
    if M > 1:
        # pair 4: above fp16's largest finite value, in the last token only
        # (its outputs are then one dominant product each, often an exact
        # bf16 rounding midpoint: a tie the other token rows dilute)
        x[M - 1, 1100] = 7.0e4
    xb = inputs.f32_to_bf16_bits(x)
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(xb), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), 128)
    torch.cuda.synchronize()
    assert_w4a16_stream(bf16_from_gpu(y), xb, op.q, op.scale, op.zero)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_w4a16_full_size(M):
    w = inputs.WORKLOADS["te_decode_w4a16"]
    op = inputs.w4a16_operands(M, w["N"], w["K"], w["group"])
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(op.x), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), w["group"])
    torch.cuda.synchronize()
    assert_w4a16_stream(bf16_from_gpu(y), op.x, op.q, op.scale, op.zero)


# W4A16 above 32 tokens: one tensor-core GEMM, weights widened to bf16 first
# (the 16-bit unpack form); held to that form within the bound of its fp32
# accumulation, and to the exact form with the widening's and the output
# rounding's error added.  The reference is a library matrix product of x
# with the oracle's weights (every output).
def check_w4a16_large(y_bits, op):
    x64 = oracle.bf16_bits_to_f32(op.x).astype(np.float64)
    xa = np.abs(x64)
    w_dq = oracle.w4a16_weights_f64(op.q, op.scale, op.zero, 128, widen=True)
    ref_dq = x64 @ w_dq.T
    err = w4a16_tc_error(op.x, w_dq)
    c = check_bf16(y_bits, ref_dq, err, tie_capacity(ref_dq, err))
    assert c.ok, "16-bit unpack form: " + str(c)
    # against the exact form (q - z) * s: per element, the widening moves the
    # value by at most 2^-8 sum_k |x_k| |w_k|, the output rounding by half an
    # ulp (< 2^-8 |y|), the fp32 accumulation by the bound above
    w = oracle.w4a16_weights_f64(op.q, op.scale, op.zero, 128)
    ref = x64 @ w.T
    bound = (xa @ np.abs(w).T + np.abs(ref_dq)) * 2.0 ** -8 + err
    g = oracle.bf16_bits_to_f32(y_bits).astype(np.float64)
    excess = np.abs(g - ref) - bound
    assert np.all(excess <= 0), f"exact form: bound exceeded by {excess.max():.3e}"


@pytest.mark.parametrize("M,N,K", [(33, 16, 128), (64, 272, 384), (192, 128, 1024),
                                   (200, 1040, 256), (385, 512, 2048), (1000, 96, 640)])
def test_w4a16_large_m(M, N, K):
    op = inputs.w4a16_operands(M, N, K, 128, seed=900 + M)
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(op.x), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), 128)
    torch.cuda.synchronize()
    check_w4a16_large(bf16_from_gpu(y), op)


def test_w4a16_large_m_extreme_token_values():
    """Tiny and huge token values next to ordinary ones (bf16 range, not fp16's)."""
    M, N, K = 96, 256, 1024
    op = inputs.w4a16_operands(M, N, K, 128, seed=930)
    x = oracle.bf16_bits_to_f32(op.x).reshape(M, K).astype(np.float64)
    x[3, 17] = 1.0e-30
    x[40, 600] = 3.0e-7
    x[95, 1000] = 7.0e4
    xb = inputs.f32_to_bf16_bits(x)
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(xb), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), 128)
    torch.cuda.synchronize()
    ref_dq = oracle.w4a16_dequant_f64(xb, op.q, op.scale, op.zero, 128)
    err = w4a16_tc_error(xb, oracle.w4a16_weights_f64(op.q, op.scale, op.zero, 128, widen=True))
    c = check_bf16(bf16_from_gpu(y), ref_dq, err, tie_capacity(ref_dq, err))
    assert c.ok, str(c)


def test_w4a16_prefill_full_size():
    """The prefill workload (weights of the decode layer, thousands of tokens),
    every output checked."""
    w = inputs.WORKLOADS["te_prefill_w4a16"]
    M, N, K = w["M"], w["N"], w["K"]
    op = inputs.w4a16_operands(M, N, K, w["group"])
    y = t4.w4a16_gemv_gemm(bf16_to_gpu(op.x), to_gpu(op.q), bf16_to_gpu(op.scale),
                           to_gpu(op.zero), w["group"])
    torch.cuda.synchronize()
    check_w4a16_large(bf16_from_gpu(y), op)


# ------------------------------------------------------------------ edge cases

def test_empty_m_is_a_no_op():
    wp = to_gpu(np.zeros((256, 128), np.uint8))
    sr = to_gpu(np.ones(256, np.float32))
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=dev())
    y = t4.convrot_w4a8_linear(x, wp, sr, 256)
    assert y.shape == (0, 256)
    a = torch.empty((0, 256), dtype=torch.int8, device=dev())
    st = torch.empty((0,), dtype=torch.float32, device=dev())
    assert t4.w4a8_gemm(a, st, wp, sr).shape == (0, 256)


def test_zero_input_gives_zero_output():
    x = torch.zeros((64, 256), dtype=torch.bfloat16, device=dev())
    W = inputs.weights(256, 256, seed=5)
    wp, sr = t4.tint4_pack_weights(to_gpu(W), 256)
    y = t4.convrot_w4a8_linear(x, wp, sr, 256)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0


def test_misaligned_pointer_is_rejected():
    buf = torch.zeros(64 * 256 + 16, dtype=torch.int8, device=dev())
    a = buf[8:8 + 64 * 256].view(64, 256)
    st = torch.ones(64, dtype=torch.float32, device=dev())
    wp = torch.zeros((256, 128), dtype=torch.uint8, device=dev())
    sr = torch.ones(256, dtype=torch.float32, device=dev())
    with pytest.raises(t4.Tint4Error) as e:
        t4.w4a8_gemm(a, st, wp, sr)
    assert e.value.name == "TINT4_ERR_MISALIGNED"


def test_bounded_wait_reports_timeout_and_context_survives():
    """A device-side wait that nobody releases gives up after its limit and
    reports TINT4_ERR_TIMEOUT; the context stays usable afterwards."""
    assert t4.tint4_get_device_error() == 0
    t4.tint4_debug_bounded_wait(2_000_000)       # 2 ms
    assert t4.tint4_get_device_error() == 5
    assert t4.tint4_get_device_error() == 0     # the read cleared it
    qa = inputs.random_codes(64, 256, -127, 127, seed=1)
    qw = inputs.random_codes(256, 256, -7, 7, seed=2)
    acc = t4.tint4_debug_int32_gemm(to_gpu(qa), 8, to_gpu(oracle.pack_int4(qw)))
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i32(qa, qw))
    assert t4.tint4_get_device_error() == 0


def test_quantize_exact_ties():
    """Values that sit exactly on rounding midpoints (scale exactly 1 or 1/127):
    the kernel's codes must equal the oracle's round-half-to-even codes."""
    ties = np.arange(-126.5, 127.0, 1.0)                      # 254 exact ties
    row = np.concatenate([[127.0, -127.0], ties]).astype(np.float32)
    x = inputs.f32_to_bf16_bits(np.stack([row, row[::-1], row * 0.5]))
    for bits in (8, 4):
        c_ref, s_ref, _ = oracle.quantize_act(x, 0, bits)
        codes, s = t4.convrot_quantize_act(bf16_to_gpu(x), 0, bits)
        torch.cuda.synchronize()
        got = codes.cpu().numpy() if bits == 8 else oracle.unpack_int4(codes.cpu().numpy())
        assert np.array_equal(got, c_ref)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    wt = np.concatenate([[7.0, -7.0], np.arange(-6.5, 7.0, 1.0), np.arange(-6.5, 7.0, 1.0)[::-1],
                         [0.5, -0.5]]).astype(np.float32)
    W = np.stack([wt, -wt])
    p_ref, s_ref, _ = oracle.pack_weights(W, 0)
    p, s = t4.tint4_pack_weights(to_gpu(W), 0)
    torch.cuda.synchronize()
    assert np.array_equal(p.cpu().numpy(), p_ref)
