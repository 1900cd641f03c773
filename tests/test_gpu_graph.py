"""One lynx_linear captured in a CUDA graph and replayed with new activations.

A graph fixes every kernel parameter at capture, so nothing a call needs to be
fresh may come from the host: the layer is replayed three times on the
mlp_up shape (4608 x 3072 -> 12288, a full-device CTA-pair grid), each time
after copying a newly drawn X into the captured input buffer, and Y is checked
on every row against the oracle for that X.  The workspace is the graph's own
and is not touched between replays."""
import numpy as np
import pytest
import torch

from activation_sparse_gemm_lynx_b200 import lynx, workloads

import oracle_checks

pytestmark = pytest.mark.gpu


def host(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda:0")


@pytest.mark.parametrize("skip", [False, True])
def test_graph_replay_with_new_inputs_every_row(skip):
    torch.cuda.set_device(0)
    lynx.library()
    name = "mlp_up"
    c = workloads.CONFIGS[name]
    inp = workloads.make_config_inputs(name)
    X, W, bias, A, B = (dev(inp[k]) for k in ("X", "W", "bias", "A", "B"))
    Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda:0")
    ws = torch.empty(lynx.lynx_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device="cuda:0")
    lynx.lynx_linear(X, W, bias, A, B, skip_sparsify=skip, Y=Y, workspace=ws)  # set-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            lynx.lynx_linear(X, W, bias, A, B, skip_sparsify=skip, Y=Y, workspace=ws)
    torch.cuda.synchronize()
    for rep in range(3):
        rng = np.random.default_rng([c.seed, 1000 + rep])
        xb = workloads.f32_to_bf16_bits(workloads.draw_activations(rng, c.M, c.K, c.x_kind))
        X.copy_(dev(xb))
        Y.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        st, code = lynx.lynx_check_error(s)
        assert st == lynx.LYNX_OK, (rep, st, code)
        worst, fro = oracle_checks.linear_all_rows(host(Y), dict(inp, X=xb), skip=skip)
        assert worst <= 1.0 and fro <= 5e-3, (rep, worst, fro)
    del g
