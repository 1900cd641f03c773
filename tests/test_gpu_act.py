"""The layer with GELU (tanh form) applied in the GEMM epilogue
(lynx_linear_act), against the CPU oracle's gelu_tanh(linear(...)).

Bar, derived from the layer's own: GELU (tanh form) is Lipschitz with constant
1.13 (its largest slope, near v = 1.5), so a pre-activation error within e
leaves the activated output within 1.13 e; evaluating GELU in fp32 with the
hardware exp and divide approximations adds a few fp32 ulps of the value, far
below that.  Hence elementwise |dY| <= 1.13 * 2e-2 * ||S(X)_m||_2 ||W_n||_2 and
||dY||_F <= 1.13 * 5e-3 * ||Y_pre||_F, with Y_pre the oracle's output before
the activation.  Inputs come from the seeded generators; expected values only
from the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gemm_lynx_b200 import lynx, workloads

import helpers

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LIP = 1.13


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


def act_check(y_gpu_bits, inp, skip, rows=None):
    X = inp["X"] if rows is None else inp["X"][rows]
    y_pre, _, sx = oracle.linear(X, inp["W"], inp["bias"], inp["A"], inp["B"], skip=skip, want_sx=True)
    y_ref = oracle.gelu_tanh(y_pre)
    y = helpers.f32(y_gpu_bits).astype(np.float64)
    if rows is not None:
        y = y[rows]
    bound = LIP * 2e-2 * np.outer(np.linalg.norm(sx, axis=1),
                                  np.linalg.norm(helpers.f32(inp["W"]).astype(np.float64), axis=1))
    worst = float((np.abs(y - y_ref) / np.maximum(bound, 1e-30)).max())
    fro = float(np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_pre), 1e-30))
    assert worst <= 1.0 and fro <= LIP * 5e-3, (worst, fro)
    # the activation did act: a fair share of the outputs is negative-side
    # GELU (small magnitude), not the identity
    assert np.mean(y_ref < 0) > 0.05


def run_act(inp, skip, act=lynx.LYNX_ACT_GELU_TANH):
    Y = lynx.lynx_linear_act(dev(inp["X"]), dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]),
                             dev(inp["B"]), skip_sparsify=skip, act=act)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    return host(Y)


@pytest.mark.parametrize("M,N,K", [(300, 200, 576),     # one-CTA GEMM (N < 256, K % 128 != 0)
                                   (520, 1024, 768),    # CTA-pair GEMM, ragged last row block
                                   (256, 512, 512)])
@pytest.mark.parametrize("skip", [False, True])
def test_gelu_epilogue_matches_oracle(M, N, K, skip):
    inp = workloads.make_linear_inputs(M, K, N, seed=[11, M, N, K])
    act_check(run_act(inp, skip), inp, skip)


def test_gelu_epilogue_tiny_config():
    inp = workloads.make_config_inputs("tiny")
    act_check(run_act(inp, False), inp, False)


@pytest.mark.parametrize("M,N,K", [(300, 200, 576), (520, 1024, 768)])
def test_act_none_is_the_plain_layer(M, N, K):
    inp = workloads.make_linear_inputs(M, K, N, seed=[12, M])
    y_none = run_act(inp, False, act=lynx.LYNX_ACT_NONE)
    Y = lynx.lynx_linear(dev(inp["X"]), dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert np.array_equal(y_none, host(Y))


def bf16_ulp(v):
    """Spacing of bf16 values at |v| (normal range)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


@pytest.mark.parametrize("M,N,K", [(300, 200, 576), (520, 1024, 768)])
def test_activation_sits_between_bias_and_rounding(M, N, K):
    """act output == bf16(gelu(s*acc + bias)) up to the one extra rounding of
    the plain layer's bf16 output: |Y_act - gelu(Y_plain)| <= 1.13 * ulp(Y_plain)/2
    + ulp(Y_act)/2 (+ the fp32 evaluation), checked element by element."""
    inp = workloads.make_linear_inputs(M, K, N, seed=[13, M])
    y_act = helpers.f32(run_act(inp, False)).astype(np.float64)
    Y = lynx.lynx_linear(dev(inp["X"]), dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]), dev(inp["B"]))
    torch.cuda.synchronize()
    y_plain = helpers.f32(host(Y)).astype(np.float64)
    g = oracle.gelu_tanh(y_plain)
    tol = LIP * bf16_ulp(y_plain) / 2 + bf16_ulp(g) / 2 + 1e-5 * np.abs(g) + 1e-37
    assert np.all(np.abs(y_act - g) <= tol), float(np.max(np.abs(y_act - g) / tol))


def test_full_size_mlp_up_with_gelu_sampled_rows():
    """The MLP up-projection at full size (M = 4608, in the launch configuration
    the benchmark times), GELU in the epilogue, on sampled rows."""
    inp = workloads.make_config_inputs("mlp_up")
    M = inp["X"].shape[0]
    y = run_act(inp, False)
    rng = np.random.default_rng(21)
    rows = np.unique(np.concatenate([[0, 255, 256, M - 1], rng.choice(M, 16, replace=False)]))
    act_check(y, inp, False, rows=rows)


def test_host_entry_matches_device_entry():
    inp = workloads.make_linear_inputs(1100, 768, 1024, seed=[14])
    y_dev = run_act(inp, False)
    Xh = torch.from_numpy(inp["X"].view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = lynx.lynx_linear_host_act(Xh, dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert np.array_equal(Yh.view(torch.int16).numpy().view(np.uint16), y_dev)
