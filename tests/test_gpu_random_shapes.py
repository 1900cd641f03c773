"""Seeded random layer configurations against the oracle, on every row.

Each case draws a shape (M from 1 to 700 rows, N a multiple of 8 up to 1536, K a
multiple of 64 up to 2048, so both the 1-CTA GEMM and the CTA-pair GEMM with
ragged tiles are reached), a LoRA rank (none, or r % 16 == 0 up to 256), bias
or none, the sparse or the dense (skip) path, the GELU epilogue or none, and
the activation distribution.  Y is checked on every row against the oracle's
fp64 layer with the layer's bar (times GELU's largest slope, 1.13, with the
activation); the layer's two halves on two streams must give the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gemm_lynx_b200 import lynx, workloads

import helpers

pytestmark = pytest.mark.gpu

N_CASES = 120


def dev(bits):
    if bits is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda:0")


def host(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def draw_case(i):
    rng = np.random.default_rng([20261203, i])
    M = int(rng.integers(1, 129)) if rng.random() < 0.3 else int(rng.integers(129, 701))
    N = 8 * int(rng.integers(1, 193))
    K = 128 * int(rng.integers(1, 17)) if rng.random() < 0.6 else 64 * int(rng.integers(1, 33))
    r = int(rng.choice([0, 16, 32, 48, 64, 96, 128, 256]))
    return dict(M=M, N=N, K=K, r=r, bias=bool(rng.random() < 0.7), skip=bool(rng.random() < 0.3),
                gelu=bool(rng.random() < 0.3), kind=str(rng.choice(["mixture", "gelu"])), seed=[77, i])


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_layer_matches_oracle(i):
    torch.cuda.set_device(0)
    lynx.library()
    c = draw_case(i)
    lora = c["r"] > 0
    inp = workloads.make_linear_inputs(c["M"], c["K"], c["N"], r=c["r"] if lora else 64, seed=c["seed"],
                                       x_kind=c["kind"], bias=c["bias"], lora=lora)
    X, W, bias, A, B = (dev(inp[k]) for k in ("X", "W", "bias", "A", "B"))
    act = lynx.LYNX_ACT_GELU_TANH if c["gelu"] else lynx.LYNX_ACT_NONE
    Y = lynx.lynx_linear_act(X, W, bias, A, B, skip_sparsify=c["skip"], act=act)
    # the two halves on two streams, after an event
    ws = torch.full((lynx.lynx_workspace_bytes(c["M"], c["N"], c["K"], c["r"] if lora else 64),), 0x5A,
                    dtype=torch.uint8, device="cuda:0")
    Y2 = torch.zeros_like(Y)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    lynx.lynx_linear_begin(X, W, bias, A, B, skip_sparsify=c["skip"], act=act, Y=Y2, workspace=ws, stream=s1)
    ev = torch.cuda.Event()
    ev.record(s1)
    s2.wait_event(ev)
    lynx.lynx_linear_finish(X, W, bias, A, B, skip_sparsify=c["skip"], act=act, Y=Y2, workspace=ws, stream=s2)
    torch.cuda.synchronize()
    for s in (None, s1, s2):
        st, code = lynx.lynx_check_error(s)
        assert st == lynx.LYNX_OK, (c, st, code)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)), c
    y_pre, _, sx = oracle.linear(inp["X"], inp["W"], inp["bias"], inp["A"], inp["B"], skip=c["skip"],
                                 want_sx=True)
    y_ref = oracle.gelu_tanh(y_pre) if c["gelu"] else y_pre
    slope = 1.13 if c["gelu"] else 1.0
    y = helpers.f32(host(Y)).astype(np.float64)
    bound = slope * 2e-2 * np.outer(np.linalg.norm(sx, axis=1),
                                    np.linalg.norm(helpers.f32(inp["W"]).astype(np.float64), axis=1))
    worst = float((np.abs(y - y_ref) / np.maximum(bound, 1e-30)).max())
    fro = float(np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_pre), 1e-30)) / slope
    assert worst <= 1.0 and fro <= 5e-3, (c, worst, fro)
