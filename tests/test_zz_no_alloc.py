"""lynx_sparsify_noalloc: S(X) with the library's fixed device scratch.

The entry point is compared with lynx_sparsify (caller workspace) on two calls
in a row on one stream, so the second call reuses the scratch the first one
wrote.  The file is collected last, and passes alone as well.
"""
import ctypes

import numpy as np
import pytest

from activation_sparse_gemm_lynx_b200 import build as lynx_build
from activation_sparse_gemm_lynx_b200 import lynx, workloads

# fake, never dereferenced device addresses for the host-side checks
P = 0x10000000


def vp(x):
    return ctypes.c_void_p(x)


@pytest.fixture(scope="module")
def lib():
    lynx_build.build()
    return lynx.library()


def test_noalloc_host_checks(lib):
    f = lib.lynx_sparsify_noalloc
    mx = lynx.lynx_sparsify_noalloc_max_rows()
    assert mx == 16384
    # one row past the fixed scratch is refused before anything is launched
    assert f(vp(P), mx + 1, 512, vp(P), vp(P), None, None) == lynx.LYNX_ERR_WORKSPACE_TOO_SMALL
    assert f(None, 128, 512, vp(P), vp(P), None, None) == lynx.LYNX_ERR_INVALID_ARG
    assert f(vp(P), 128, 500, vp(P), vp(P), None, None) == lynx.LYNX_ERR_UNSUPPORTED_SHAPE
    assert f(vp(P), 128, 512, vp(P + 4), vp(P), None, None) == lynx.LYNX_ERR_MISALIGNED
    assert f(vp(P), 128, 512, vp(P), vp(P), vp(P + 2), None) == lynx.LYNX_ERR_MISALIGNED


def _dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda:0")


def _canonical(meta, M, K):
    # the defined part of the metadata: every group of rows < M (a half-filled
    # last 128-K block leaves its unused columns unwritten)
    return lynx.lynx_meta_hw_to_canonical(meta.cpu().numpy(), M, K)


def _bufs(M, K):
    import torch

    return (torch.empty((M, K // 2), dtype=torch.bfloat16, device="cuda:0"),
            torch.empty(lynx.lynx_meta_bytes(M, K), dtype=torch.uint8, device="cuda:0"),
            torch.empty(M, dtype=torch.float32, device="cuda:0"))


@pytest.mark.gpu
@pytest.mark.parametrize("M,K", [(300, 576), (4608, 3072), (16384, 1024)])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(lib, M, K):
    import torch

    assert torch.cuda.is_available(), "this test needs a GPU"
    torch.cuda.set_device(0)
    lynx.lynx_check_error()  # start from a clear device status word
    x1 = _dev(workloads.make_linear_inputs(M, K, 8, seed=[11, M, K])["X"])
    x2 = _dev(workloads.make_linear_inputs(M, K, 8, seed=[12, M, K], x_kind="gelu")["X"])

    # the existing entry point, with its own workspace
    ref = [lynx.lynx_sparsify(x) for x in (x1, x2)]
    torch.cuda.synchronize()

    a, b = _bufs(M, K), _bufs(M, K)
    lynx.lynx_sparsify_noalloc(x1, *a)
    lynx.lynx_sparsify_noalloc(x2, *b)  # same stream, right after: the scratch is reused
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)

    for (rv, rm, rs), (v, m, s) in zip(ref, (a, b)):
        assert torch.equal(v.view(torch.int16), rv.view(torch.int16))
        assert np.array_equal(_canonical(m, M, K), _canonical(rm, M, K))
        assert torch.equal(s, rs)


@pytest.mark.gpu
def test_noalloc_without_row_scale(lib):
    import torch

    torch.cuda.set_device(0)
    lynx.lynx_check_error()
    M, K = 1000, 3072
    x = _dev(workloads.make_linear_inputs(M, K, 8, seed=13)["X"])
    rv, rm, _ = lynx.lynx_sparsify(x)
    v, m, _ = _bufs(M, K)
    # s then lives in the library's scratch; the compensated values still carry it
    lynx.lynx_sparsify_noalloc(x, v, m, None)
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    assert torch.equal(v.view(torch.int16), rv.view(torch.int16))
    assert np.array_equal(_canonical(m, M, K), _canonical(rm, M, K))
