"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function include/lynx.h declares, rejects bad arguments before touching the
device, and converts metadata between the canonical and hardware layouts the
same way as the test's own reading of the layout."""
import ctypes

import numpy as np
import pytest

from activation_sparse_gemm_lynx_b200 import build as lynx_build
from activation_sparse_gemm_lynx_b200 import lynx

import helpers


@pytest.fixture(scope="module")
def lib():
    lynx_build.build()
    return lynx.library()


def test_exports_every_header_function(lib):
    names = lynx.header_functions()
    assert len(names) >= 14
    raw = ctypes.CDLL(lynx.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_status_strings(lib):
    assert lynx.lynx_status_string(0) == "LYNX_OK"
    assert lynx.lynx_status_string(6) == "LYNX_ERR_DEVICE_TIMEOUT"
    assert lynx.lynx_status_string(99) == "LYNX_ERR_UNKNOWN"
    assert lynx.lynx_version() >> 16 == 1
    assert lynx.lynx_lora_rank() == 64


def test_lora_rank_rules(lib):
    ok = [16, 32, 48, 64, 128, 240, 256]
    bad = [0, 8, 24, 63, 65, 272, 512, -16]
    assert all(lynx.lynx_lora_rank_supported(r) for r in ok)
    assert not any(lynx.lynx_lora_rank_supported(r) for r in bad)
    for r in ok:  # accepted by the checks; the call then fails only for want of a device
        assert linear(lib, A=P, B=P, r=r) in (lynx.LYNX_ERR_CUDA, lynx.LYNX_OK), r
    for r in bad:
        assert linear(lib, A=P, B=P, r=r) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE, r
    # without A and B, r only sizes nothing: 0 or any supported rank
    assert linear(lib, r=17) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("r", [16, 64, 256])
def test_workspace_grows_with_rank(lib, r):
    M, K = 4608, 3072
    ws = lynx.lynx_workspace_bytes(M, 512, K, r)
    # kept values, metadata, s, T [M,r] bf16, 8 split partials (sums and T),
    # one state word per 32-row slice
    floor = M * K + lynx.lynx_meta_bytes(M, K) + 4 * M + 2 * M * r + 8 * M * 8 + 8 * M * r * 4 + \
        4 * -(-M // 32)
    assert floor <= ws <= floor + 8 * 256


def test_profile_part_hook(lib):
    assert lynx.lynx_profile_set_part(1) == 0
    assert lynx.lynx_profile_set_part(2) == 1
    assert lib.lynx_profile_set_part(3) == -1
    assert lynx.lynx_profile_set_part(0) == 2


@pytest.mark.parametrize("M,K", [(1, 64), (128, 128), (129, 192), (4608, 3072), (4608, 12288)])
def test_sizes(lib, M, K):
    assert lynx.lynx_vals_bytes(M, K) == M * K
    assert lynx.lynx_meta_bytes(M, K) == -(-M // 256) * 2 * -(-K // 128) * 2048
    ws = lynx.lynx_workspace_bytes(M, 512, K, 64)
    assert ws >= M * K + lynx.lynx_meta_bytes(M, K) + 4 * M + 128 * M
    assert ws % 256 == 0


# fake, never dereferenced device addresses: every check below fails on the host
P = 0x10000000


def vp(x):
    return ctypes.c_void_p(x)


def linear(lib, X=P, W=P, bias=None, A=None, B=None, M=256, N=512, K=512, r=64, skip=0, Y=P,
           ws=P, ws_bytes=1 << 30):
    return lib.lynx_linear(vp(X), vp(W), vp(bias), vp(A), vp(B), M, N, K, r, skip, vp(Y), vp(ws),
                           ws_bytes, None)


def test_linear_argument_errors(lib):
    assert linear(lib, X=None) == lynx.LYNX_ERR_INVALID_ARG
    assert linear(lib, W=None) == lynx.LYNX_ERR_INVALID_ARG
    assert linear(lib, Y=None) == lynx.LYNX_ERR_INVALID_ARG
    assert linear(lib, A=P, B=None) == lynx.LYNX_ERR_INVALID_ARG
    assert linear(lib, A=P, B=P, r=40) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert linear(lib, K=100) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert linear(lib, K=32) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert linear(lib, N=12) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert linear(lib, M=0) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert linear(lib, X=P + 8) == lynx.LYNX_ERR_MISALIGNED
    assert linear(lib, bias=P + 2) == lynx.LYNX_ERR_MISALIGNED
    assert linear(lib, ws=None) == lynx.LYNX_ERR_INVALID_ARG
    need = lynx.lynx_workspace_bytes(256, 512, 512, 64)
    assert linear(lib, ws_bytes=need - 1) == lynx.LYNX_ERR_WORKSPACE_TOO_SMALL
    # dense path without LoRA needs no workspace at all: the checks pass and the
    # call then fails only because there is no device here
    r = linear(lib, ws=None, skip=1, r=0)
    assert r in (lynx.LYNX_ERR_CUDA, lynx.LYNX_OK)


def test_sparsify_argument_errors(lib):
    f = lib.lynx_sparsify
    big = 1 << 30
    assert f(None, 128, 512, vp(P), vp(P), None, vp(P), big, None) == lynx.LYNX_ERR_INVALID_ARG
    assert f(vp(P), 128, 512, vp(P), vp(P), None, None, big, None) == lynx.LYNX_ERR_INVALID_ARG
    assert f(vp(P), 128, 500, vp(P), vp(P), None, vp(P), big, None) == \
        lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert f(vp(P), 128, 512, vp(P + 4), vp(P), None, vp(P), big, None) == lynx.LYNX_ERR_MISALIGNED
    assert f(vp(P), 128, 512, vp(P), vp(P), vp(P + 2), vp(P), big, None) == \
        lynx.LYNX_ERR_MISALIGNED
    need = lynx.lynx_sparsify_workspace_bytes(128, 512)
    assert need >= 8 * 128 * 8
    assert f(vp(P), 128, 512, vp(P), vp(P), None, vp(P), need - 1, None) == \
        lynx.LYNX_ERR_WORKSPACE_TOO_SMALL


def test_linear_host_argument_errors(lib):
    f = lib.lynx_linear_host
    need = lynx.lynx_linear_host_workspace_bytes(256, 512, 512, 64)
    assert need >= 2 * 256 * 512 * 2 + lynx.lynx_workspace_bytes(256, 512, 512, 64)

    def call(X=P, W=P, Y=P, ws=P, ws_bytes=need, M=256, K=512, A=None, B=None, r=0):
        return f(vp(X), vp(W), None, vp(A), vp(B), M, 512, K, r, 0, vp(Y), vp(ws), ws_bytes, None)

    assert call(X=None) == lynx.LYNX_ERR_INVALID_ARG
    assert call(Y=None) == lynx.LYNX_ERR_INVALID_ARG
    assert call(ws=None) == lynx.LYNX_ERR_INVALID_ARG
    assert call(A=P) == lynx.LYNX_ERR_INVALID_ARG
    assert call(K=100) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert call(ws=P + 8) == lynx.LYNX_ERR_MISALIGNED
    assert call(ws_bytes=need - 1) == lynx.LYNX_ERR_WORKSPACE_TOO_SMALL


def test_linear_act_argument_errors(lib):
    def call(act=lynx.LYNX_ACT_GELU_TANH, X=P, Y=P, ws_bytes=1 << 30):
        return lib.lynx_linear_act(vp(X), vp(P), None, vp(P), vp(P), 256, 512, 512, 64, 0, act,
                                   vp(Y), vp(P), ws_bytes, None)

    assert call(act=2) == lynx.LYNX_ERR_INVALID_ARG
    assert call(act=-1) == lynx.LYNX_ERR_INVALID_ARG
    assert call(X=None) == lynx.LYNX_ERR_INVALID_ARG
    assert call(Y=P + 8) == lynx.LYNX_ERR_MISALIGNED
    need = lynx.lynx_workspace_bytes(256, 512, 512, 64)
    assert call(ws_bytes=need - 1) == lynx.LYNX_ERR_WORKSPACE_TOO_SMALL
    # the host form checks the activation too
    hneed = lynx.lynx_linear_host_workspace_bytes(256, 512, 512, 64)
    assert lib.lynx_linear_host_act(vp(P), vp(P), None, None, None, 256, 512, 512, 0, 0, 7, vp(P),
                                    vp(P), hneed, None) == lynx.LYNX_ERR_INVALID_ARG


def test_sparse_gemm_argument_errors(lib):
    f = lib.lynx_sparse_gemm
    assert f(vp(P), None, None, vp(P), None, None, 128, 256, 512, 0, vp(P), None) == \
        lynx.LYNX_ERR_INVALID_ARG
    assert f(vp(P), vp(P), vp(P), vp(P), None, None, 128, 256, 512, 64, vp(P), None) == \
        lynx.LYNX_ERR_INVALID_ARG
    assert f(vp(P), vp(P), None, vp(P), None, None, 128, 256, 96, 0, vp(P), None) == \
        lynx.LYNX_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("M,K", [(1, 64), (128, 128), (200, 192), (300, 576), (130, 1024)])
def test_meta_layout_roundtrip_and_formula(lib, M, K):
    rng = np.random.default_rng(M * 7 + K)
    valid = np.array([0x4, 0x8, 0xC, 0x9, 0xD, 0xE], dtype=np.uint8)
    nib = valid[rng.integers(0, 6, size=(M, K // 4))]
    canon = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    hw = lynx.lynx_meta_canonical_to_hw(canon, M, K)
    assert hw.size == lynx.lynx_meta_bytes(M, K)
    # the library's layout equals the test's own reading of the definition
    # (padding columns of a last, half-filled K block are zero in both)
    mine = helpers.hw_from_canonical(canon, M, K)
    assert np.array_equal(hw, mine)
    back = lynx.lynx_meta_hw_to_canonical(hw, M, K)
    assert np.array_equal(back, canon)
    assert np.array_equal(helpers.canonical_from_hw(hw, M, K), canon)


def test_meta_padding_rows_hold_zero_row_pattern(lib):
    M, K = 130, 256
    canon = np.full((M, K // 8), 0xEE, dtype=np.uint8)   # (2,3) everywhere
    hw = lynx.lynx_meta_canonical_to_hw(canon, M + 0, K)
    pad = helpers.canonical_from_hw(hw, 256, K)[M:]  # padded to 256 rows
    assert np.all(pad == 0x44)


def test_specific_bit_positions(lib):
    # row 9 (second 8-row half of block row 0 -> upper 16 bits), column 16..19
    # (second K16 half -> lane + 8), word 0: lane = 1 + 8 + 0 = 9, bit 16
    M, K = 128, 128
    canon = np.full((M, K // 8), 0x44, dtype=np.uint8)
    canon[9, 2] = 0x4E   # group 4 (k = 16..19) -> nibble 0xE, group 5 -> 0x4
    hw = lynx.lynx_meta_canonical_to_hw(canon, M, K)
    word = int.from_bytes(hw[9 * 16: 9 * 16 + 4].tobytes(), "little")
    assert (word >> 16) & 0xF == 0xE
