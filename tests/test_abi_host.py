"""Host-side checks of the C ABI library (no GPU needed).

The library must load on a machine without a GPU, export every entry point
that include/tint4.h declares, and reject bad arguments before it touches the
CUDA runtime.  No compute call is made here.
"""
import ctypes
import os
import re

import pytest

from int4_weight_quantized_block_b200 import _native, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tint4.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_lists_the_entry_points():
    names = declared_functions()
    for n in ("tint4_pack_weights", "convrot_quantize_act", "w4a8_gemm", "w4a4_gemm",
              "convrot_w4a8_linear", "convrot_w4a4_linear", "w4a16_gemv_gemm",
              "tint4_debug_int32_gemm", "tint4_get_device_error", "tint4_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _native.SIGNATURES, f"binding lacks {name}"


def test_binding_names_match_header():
    assert sorted(_native.SIGNATURES) == declared_functions()


def test_library_does_not_link_the_oracle():
    out = open(build.LIB, "rb").read()
    assert b"oracle_" not in out


def test_version_and_status_strings(lib):
    assert lib.tint4_abi_version() == 1
    for code in range(8):
        s = lib.tint4_status_string(code)
        assert s and isinstance(s, bytes)
    assert lib.tint4_status_string(99) == b"unknown status"


def test_workspace_size(lib):
    # codes | token scales, each part 256-aligned
    assert lib.convrot_linear_workspace_size(4608, 3072, 8) == 4608 * 3072 + 4608 * 4
    assert lib.convrot_linear_workspace_size(4608, 3072, 4) == 4608 * 3072 + 4608 * 4
    assert lib.convrot_linear_workspace_size(3, 64, 8) == 256 + 256
    assert lib.convrot_linear_workspace_size(3, 64, 5) == 0
    assert lib.convrot_linear_workspace_size(-1, 64, 8) == 0
    # the boundary specification's name for the W4A8 size
    for M, K in ((4608, 3072), (3, 64), (1, 4096)):
        assert lib.convrot_w4a8_linear_workspace(M, K) == lib.convrot_linear_workspace_size(M, K, 8)


NULL = None


@pytest.mark.parametrize("M,N,K,expect", [
    (-1, 256, 256, 1),      # negative size
    (64, 8, 256, 2),        # N < 16
    (64, 24, 256, 2),       # N % 16
    (64, 256, 48, 2),       # K % 32
    (64, 256, 16, 2),       # K < 32
    (64, 256, 131072, 2),   # K too large for int32 accumulation headroom
])
def test_gemm_shape_rules(lib, M, N, K, expect):
    assert lib.w4a8_gemm(16, 16, 16, 16, NULL, 16, M, N, K, NULL) == expect
    assert lib.w4a4_gemm(16, 16, 16, 16, NULL, 16, M, N, K, NULL) == expect


def test_gemm_null_and_alignment(lib):
    assert lib.w4a8_gemm(NULL, 16, 16, 16, NULL, 16, 4, 256, 256, NULL) == 1
    assert lib.w4a8_gemm(16 + 8, 16, 16, 16, NULL, 16, 4, 256, 256, NULL) == 3
    assert lib.w4a8_gemm(16, 16, 16, 16, 16 + 2, 16, 4, 256, 256, NULL) == 3   # bias


@pytest.mark.parametrize("group,K,expect", [(32, 256, 1), (128, 256, 1), (64, 96, 2),
                                            (256, 128, 2), (16, 16384 + 32, 2)])
def test_quantize_shape_rules(lib, group, K, expect):
    assert lib.convrot_quantize_act(16, 4, K, group, 8, 16, 16, NULL) == expect
    assert lib.tint4_pack_weights(16, 4, K, group, 16, 16, NULL) == expect


def test_quantize_bits_rule(lib):
    assert lib.convrot_quantize_act(16, 4, 256, 16, 6, 16, 16, NULL) == 1


def test_linear_workspace_rules(lib):
    need = lib.convrot_linear_workspace_size(4, 256, 8)
    assert lib.convrot_w4a8_linear(16, 16, 16, NULL, 16, 4, 256, 256, 16, NULL, need,
                                   NULL) == 6
    assert lib.convrot_w4a8_linear(16, 16, 16, NULL, 16, 4, 256, 256, 16, 256, need - 1,
                                   NULL) == 6
    assert lib.convrot_w4a8_linear(16, 16, 16, NULL, 16, 4, 256, 256, 16, 256 + 16, need,
                                   NULL) == 3


def test_w4a16_rules(lib):
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 64, 16, 1, 256, 256, NULL) == 2   # group
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 32, 256, 16512, NULL) == 2  # decode K
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 33, 256, 65664, NULL) == 2  # GEMM K
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 65535 * 128 + 1, 256, 256,
                               NULL) == 2                                          # M
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 0, 256, 256, NULL) == 2    # M
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 33, 8, 256, NULL) == 2     # N % 16
    assert lib.w4a16_gemv_gemm(16, 16, 16, 16, 128, 16, 1, 256, 192, NULL) == 2  # K % 128
    assert lib.w4a16_gemv_gemm(NULL, 16, 16, 16, 128, 16, 1, 256, 256, NULL) == 1
    assert lib.w4a16_gemv_gemm(16, 24, 16, 16, 128, 16, 1, 256, 256, NULL) == 3


def test_grouped_rules(lib):
    from int4_weight_quantized_block_b200._native import WeightGroup
    G = WeightGroup * 5
    ok = G(*[WeightGroup(16, 16, None, 16, 256) for _ in range(5)])
    assert lib.w4a8_gemm_grouped(16, 16, NULL, 1, 4, 256, NULL) == 1                 # null groups
    assert lib.w4a8_gemm_grouped(16, 16, ctypes.addressof(ok), 0, 4, 256, NULL) == 1  # none
    assert lib.w4a8_gemm_grouped(16, 16, ctypes.addressof(ok), 5, 4, 256, NULL) == 2  # too many
    bad_n = G(WeightGroup(16, 16, None, 16, 256), WeightGroup(16, 16, None, 16, 8))
    assert lib.w4a8_gemm_grouped(16, 16, ctypes.addressof(bad_n), 2, 4, 256, NULL) == 2
    bad_p = G(WeightGroup(16, 16, None, 16, 256), WeightGroup(None, 16, None, 16, 256))
    assert lib.w4a8_gemm_grouped(16, 16, ctypes.addressof(bad_p), 2, 4, 256, NULL) == 1
    mis = G(WeightGroup(16, 16, None, 24, 256))
    assert lib.w4a8_gemm_grouped(16, 16, ctypes.addressof(mis), 1, 4, 256, NULL) == 3
    assert lib.w4a8_gemm_grouped(NULL, 16, ctypes.addressof(ok), 1, 4, 256, NULL) == 1
    need = lib.convrot_linear_workspace_size(4, 256, 8)
    assert lib.convrot_w4a8_linear_grouped(16, ctypes.addressof(ok), 1, 4, 256, 16, NULL, need,
                                           NULL) == 6
    assert lib.convrot_w4a8_linear_grouped(16, ctypes.addressof(ok), 1, 4, 256, 32, 256, need,
                                           NULL) == 1                                  # group value


def test_groupwise_rules(lib):
    assert lib.tint4_pack_weights_groupwise(16, 4, 256, 0, 2, 16, 16, 16, NULL) == 1   # asym
    assert lib.tint4_pack_weights_groupwise(16, 4, 96, 0, 0, 16, 16, NULL, NULL) == 2  # K % 128
    assert lib.tint4_pack_weights_groupwise(16, 4, 256, 0, 1, 16, 16, NULL, NULL) == 1  # no zero
    assert lib.tint4_pack_weights_groupwise(16, 4, 256, 0, 0, 16, 17, NULL, NULL) == 3
    assert lib.w4a8_gemm_groupwise(16, 16, 16, 16, NULL, NULL, 16, 4, 32, 160, NULL) == 2
    assert lib.w4a8_gemm_groupwise(16, 16, 16, 16, NULL, NULL, 16, 4, 24, 256, NULL) == 2
    assert lib.w4a8_gemm_groupwise(NULL, 16, 16, 16, NULL, NULL, 16, 4, 32, 256, NULL) == 1
    assert lib.w4a8_gemm_groupwise(16, 16, 16, 16, 17, NULL, 16, 4, 32, 256, NULL) == 3
    need = lib.convrot_linear_workspace_size(4, 256, 8)
    assert lib.convrot_w4a8_linear_groupwise(16, 16, 16, NULL, NULL, 16, 4, 32, 256, 256, 256,
                                             need - 1, NULL) == 6
    assert lib.convrot_w4a8_linear_groupwise(16, 16, 16, NULL, NULL, 16, 4, 32, 256, 32, 256,
                                             need, NULL) == 1                           # group value


def test_debug_entries_rules(lib):
    assert lib.tint4_debug_int32_gemm(16, 6, 16, 16, 4, 256, 256, NULL) == 1
    assert lib.tint4_debug_bounded_wait(10, NULL) == 1
    # the even/odd GEMM entry: M > 16 only, then the GEMM rules
    assert lib.tint4_debug_w4a8_gemm_even_odd(16, 16, 16, 16, NULL, 16, 16, 256, 256, NULL) == 2
    assert lib.tint4_debug_w4a8_gemm_even_odd(NULL, 16, 16, 16, NULL, 16, 17, 256, 256, NULL) == 1
    assert lib.tint4_debug_w4a8_gemm_even_odd(16, 16, 16, 16, NULL, 16, 17, 256, 100, NULL) == 2
    assert lib.tint4_set_wait_limit_ns(10) == 1
    assert lib.tint4_set_wait_limit_ns(10 ** 11) == 1
    assert lib.tint4_set_wait_limit_ns(4 * 10 ** 9) == 0


def test_decode_prefetch_switch_rules(lib):
    assert lib.tint4_set_decode_weight_prefetch(2) == 1
    assert lib.tint4_set_decode_weight_prefetch(-1) == 1
    assert lib.tint4_set_decode_weight_prefetch(1) == 0
    assert lib.tint4_set_decode_weight_prefetch(0) == 0


def test_even_odd_code_order():
    """The test helper's permutation: within each block of 8 codes along K,
    positions 0, 2, 4, 6 first, then 1, 3, 5, 7 (the order the fused linears
    store and the tensor-core GEMM's weight unpack produces)."""
    import torch
    import int4_weight_quantized_block_b200 as t4
    codes = torch.arange(2 * 16, dtype=torch.int8).view(2, 16)
    eo = t4.even_odd_codes(codes)
    assert eo[0].tolist() == [0, 2, 4, 6, 1, 3, 5, 7, 8, 10, 12, 14, 9, 11, 13, 15]
    assert eo[1].tolist() == [v + 16 for v in eo[0].tolist()]
    # a dot product over K does not depend on the order
    w = torch.randint(-7, 8, (16,), dtype=torch.int32)
    a = torch.randint(-127, 128, (16,), dtype=torch.int32)
    perm = t4.even_odd_codes(torch.arange(16, dtype=torch.int8).view(1, 16))[0].long()
    assert int((a * w).sum()) == int((a[perm] * w[perm]).sum())
