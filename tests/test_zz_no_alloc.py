"""The allocation-free fused linear, called through the C ABI.

convrot_w4a8_linear_noalloc serves callers that cannot allocate device memory
where they call the layer (a fixed memory budget, a host program or plug-in
whose host application owns all allocations): its scratch is a fixed 16 MiB
array inside the library instead of a caller workspace.  Its results must be
those of convrot_w4a8_linear, call after call, although every call reuses the
same array.  This file is collected last, and also passes on its own in a
fresh process (the first call on the device resolves the array's address).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import int4_weight_quantized_block_b200 as t4
from int4_weight_quantized_block_b200 import _native, inputs
from oracle.compare import bits_to_f64, check_bf16, gemm_eval_error

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(x, wp, sr, g, y, bias=None):
    """Direct C-ABI call (no Python-side allocation in between)."""
    lib = _native.load()
    M, K = x.shape
    N = wp.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.convrot_w4a8_linear_noalloc(
        x.data_ptr(), wp.data_ptr(), sr.data_ptr(), None if bias is None else bias.data_ptr(),
        y.data_ptr(), M, N, K, g, ctypes.c_void_p(stream))


@pytest.mark.parametrize("case", [
    # (M, N, K, group, with_bias): two different layers back to back each time
    [(200, 272, 320, 64, False), (4608, 1024, 3072, 256, True)],
    [(64, 256, 256, 256, True), (129, 512, 1024, 16, False)],
])
def test_noalloc_matches_workspace_entry_two_calls(case):
    for i, (M, N, K, g, with_bias) in enumerate(case):
        x = _bf16(inputs.activations(M, K, seed=900 + i))
        W = torch.from_numpy(inputs.weights(N, K, seed=901 + i)).cuda()
        wp, sr = t4.tint4_pack_weights(W, g)
        bias = _bf16(inputs.f32_to_bf16_bits(np.linspace(-1, 1, N))) if with_bias else None
        y_ref = t4.convrot_w4a8_linear(x, wp, sr, g, bias)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(x, wp, sr, g, y, bias) == 0
        torch.cuda.synchronize()
        ref64 = bits_to_f64(y_ref.view(torch.int16).cpu().numpy().view(np.uint16))
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        c = check_bf16(got, ref64, gemm_eval_error(ref64))
        assert c.ok, f"call {i}: {c}"
    assert t4.tint4_get_device_error() == 0


@pytest.mark.parametrize("M", [1, 9])
def test_noalloc_small_m_against_oracle(M):
    """Decode-sized calls: one token runs the one-launch small-M path of
    convrot_w4a8_linear (the GEMM's CTAs rotate and quantize x themselves),
    nine tokens the quantize grid and the streaming GEMM with natural-order
    codes in the fixed array.  Both are checked against the oracle, on two
    calls in a row, and against the workspace entry."""
    N, K, g = 256, 4096, 256
    xb = inputs.activations(M, K, seed=90 + M)
    W = inputs.weights(N, K, seed=91 + M)
    wp_ref, sr_ref, _ = oracle.pack_weights(W, g)
    x = _bf16(xb)
    wp = torch.from_numpy(wp_ref).cuda()
    sr = torch.from_numpy(sr_ref).cuda()
    ref64 = oracle.convrot_linear_f64(xb, wp_ref, sr_ref, g, 8)
    y_ws = t4.convrot_w4a8_linear(x, wp, sr, g)
    for _ in range(2):
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(x, wp, sr, g, y) == 0
        torch.cuda.synchronize()
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        c = check_bf16(got, ref64, gemm_eval_error(ref64))
        assert c.ok, str(c)
        assert np.array_equal(got, y_ws.view(torch.int16).cpu().numpy().view(np.uint16))
    assert t4.tint4_get_device_error() == 0


def test_noalloc_against_oracle_and_size_limit():
    M, N, K, g = 96, 320, 512, 64
    xb = inputs.activations(M, K, seed=77)
    W = inputs.weights(N, K, seed=78)
    wp_ref, sr_ref, _ = oracle.pack_weights(W, g)
    x = _bf16(xb)
    wp = torch.from_numpy(wp_ref).cuda()
    sr = torch.from_numpy(sr_ref).cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        assert _noalloc(x, wp, sr, g, y) == 0
        torch.cuda.synchronize()
        ref64 = oracle.convrot_linear_f64(xb, wp_ref, sr_ref, g, 8)
        c = check_bf16(y.view(torch.int16).cpu().numpy().view(np.uint16), ref64,
                       gemm_eval_error(ref64))
        assert c.ok, str(c)
    # M * K beyond the fixed scratch: rejected before any launch
    Mbig, Kbig = 4608, 4096
    assert t4.convrot_linear_workspace_size(Mbig, Kbig, 8) > SCRATCH_BYTES
    xbig = torch.zeros((Mbig, Kbig), dtype=torch.bfloat16, device="cuda")
    wbig = torch.zeros((256, Kbig // 2), dtype=torch.uint8, device="cuda")
    sbig = torch.ones(256, dtype=torch.float32, device="cuda")
    ybig = torch.empty((Mbig, 256), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(xbig, wbig, sbig, 256, ybig) == 6          # TINT4_ERR_WORKSPACE
