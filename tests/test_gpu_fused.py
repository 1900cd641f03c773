"""The fully fused variant (lynx_linear_fused): the 2:4 selection and the
compression run inside the GEMM on dense X tiles, after a slim pass that
computes only the row sums and T.  It must match the oracle within the layer's
bar, and it must give the two-pass lynx_linear's Y bit for bit (the same s and
T/s from the same partial sums, the same kept values in the same MMAs)."""
import numpy as np
import pytest
import torch

from activation_sparse_gemm_lynx_b200 import lynx, workloads

import oracle_checks

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def dev(bits):
    if bits is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def host(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "these tests need a GPU"
    torch.cuda.set_device(0)
    lynx.library()
    yield
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)


def run_both(inp, act=lynx.LYNX_ACT_NONE):
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    Yf = lynx.lynx_linear_fused(*args, act=act)
    if act == lynx.LYNX_ACT_NONE:
        Yl = lynx.lynx_linear(*args)
    else:
        Yl = lynx.lynx_linear_act(*args, act=act)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    return host(Yf), host(Yl)


@pytest.mark.parametrize("M,N,K,r,bias,lora", [
    (256, 512, 512, 64, True, True),      # the tiny config's shape
    (300, 768, 1024, 64, True, True),     # ragged M: a partial CTA-pair row block
    (512, 1024, 3072, 48, True, True),    # r % 32 == 16
    (384, 512, 1024, 64, False, False),   # no bias, no LoRA
    (200, 136, 576, 64, True, True),      # not a pair-kernel shape: the two-pass layer
])
def test_fused_matches_oracle_and_two_pass_layer(M, N, K, r, bias, lora):
    inp = workloads.make_linear_inputs(M, K, N, r=r, seed=M + N + K + r, bias=bias, lora=lora)
    yf, yl = run_both(inp)
    worst, fro = oracle_checks.linear_all_rows(yf, inp)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)
    assert np.array_equal(yf, yl), "fused and two-pass layers differ"


def test_fused_ties_zeros_and_all_keep_rows():
    """Groups with ties, signed zeros, an all-zero row and rows that already
    have two zeros per group, through the in-kernel selection."""
    rng = np.random.default_rng(12)
    M, K, N = 256, 512, 256
    alphabet = np.array([0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5], dtype=np.float32)
    x = alphabet[rng.integers(0, len(alphabet), size=(M, K))]
    x[7] = 0.0
    keep = rng.standard_normal((M // 2, K // 4, 4)).astype(np.float32)
    for m in range(M // 2):
        for g in range(K // 4):
            keep[m, g, rng.choice(4, 2, replace=False)] = 0.0
    x[M // 2:] = keep.reshape(M // 2, K)
    inp = workloads.make_linear_inputs(M, K, N, seed=3)
    inp["X"] = workloads.f32_to_bf16_bits(x)
    yf, yl = run_both(inp)
    worst, fro = oracle_checks.linear_all_rows(yf, inp)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)
    assert np.array_equal(yf, yl)


def test_fused_with_gelu_epilogue():
    inp = workloads.make_linear_inputs(512, 1024, 768, seed=44)
    yf, yl = run_both(inp, act=lynx.LYNX_ACT_GELU_TANH)
    worst, fro = oracle_checks.linear_all_rows(yf, inp, act="gelu_tanh")
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)
    assert np.array_equal(yf, yl)


@pytest.mark.parametrize("name", ["attn_out", "mlp_up"])
def test_fused_full_size_every_row(name):
    inp = workloads.make_config_inputs(name)
    yf, yl = run_both(inp)
    assert np.array_equal(yf, yl)
    worst, fro = oracle_checks.linear_all_rows(yf, inp)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)
