"""The block sweep replayed from a CUDA graph: every layer's Y from the graph
equals the eagerly launched sequence bit for bit, and sampled rows of one
layer of each kind (a dense, skip_sparsify block among them) match the oracle
within the layer's tolerance."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gemm_lynx_b200 import lynx, workloads
from activation_sparse_gemm_lynx_b200.sweep import LinearSweep

import helpers

pytestmark = pytest.mark.gpu


def host(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module")
def sweep_and_plan():
    assert torch.cuda.is_available(), "these tests need a GPU"
    torch.cuda.set_device(0)
    lynx.library()
    lynx.lynx_check_error()
    # the sweep's layer shapes and skip pattern at a reduced token count
    # (384 rows: one and a half CTA-pair row blocks)
    plan = workloads.sweep_plan(M=384)
    layers = []
    for (_b, _n, M, K, N, kind, skip, seed) in plan:
        inp = workloads.make_linear_inputs(M, K, N, seed=seed, x_kind=kind)
        inp["skip"] = skip
        layers.append(inp)
    return LinearSweep(layers, device="cuda:0"), plan, layers


def test_graph_replay_equals_eager_pass(sweep_and_plan):
    sweep, plan, _ = sweep_and_plan
    sweep.run()
    torch.cuda.synchronize()
    eager = [t["Y"].clone() for t in sweep.layers]
    for t in sweep.layers:
        t["Y"].zero_()
    sweep.capture()
    sweep.replay()
    sweep.replay()  # twice: the shared workspace is reused in place
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    for i, (t, e) in enumerate(zip(sweep.layers, eager)):
        assert torch.equal(t["Y"].view(torch.int16), e.view(torch.int16)), plan[i][:2]


def test_graph_layers_match_oracle(sweep_and_plan):
    sweep, plan, layers = sweep_and_plan
    if sweep.graph is None:
        sweep.run()
        sweep.capture()
    sweep.replay()
    torch.cuda.synchronize()
    skipped = {b for (b, _n, *_r, skip, _s) in plan if skip}
    assert len(skipped) == 2
    first_dense = min(skipped)
    picked = [i for i, p in enumerate(plan) if p[0] == 0] + \
             [i for i, p in enumerate(plan) if p[0] == first_dense]
    rows = np.array([0, 1, 127, 128, 255, 256, 383])
    for i in picked:
        inp = layers[i]
        y = helpers.f32(host(sweep.layers[i]["Y"])).astype(np.float64)[rows]
        y_ref, _, sx = oracle.linear(inp["X"][rows], inp["W"], inp["bias"], inp["A"], inp["B"],
                                     skip=inp["skip"], want_sx=True)
        worst, fro = helpers.y_tolerance_check(y, y_ref, sx, helpers.f32(inp["W"]).astype(np.float64))
        assert worst <= 1.0 and fro <= 5e-3, (plan[i][:2], worst, fro)


# qkv 3072->9216, out 3072->3072, up 3072->12288, down 12288->3072 (GELU inputs)
@pytest.mark.parametrize("layer", [0, 1, 2, 3])
@pytest.mark.parametrize("skip", [False, True])
def test_full_size_sweep_layer_sampled_rows(layer, skip):
    """One linear of the sweep at its full size (M = 8192), in the launch
    configuration the sweep times, on sampled rows; the dense path too."""
    torch.cuda.set_device(0)
    lynx.lynx_check_error()
    _b, _n, M, K, N, kind, _skip, seed = workloads.sweep_plan()[layer]
    inp = workloads.make_linear_inputs(M, K, N, seed=seed, x_kind=kind)
    dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda:0")
    Y = lynx.lynx_linear(dev(inp["X"]), dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]), dev(inp["B"]),
                         skip_sparsify=skip)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    rng = np.random.default_rng(layer * 2 + int(skip))
    rows = np.unique(np.concatenate([[0, 255, 256, M - 1], rng.choice(M, 20, replace=False)]))
    y = helpers.f32(host(Y)).astype(np.float64)[rows]
    y_ref, _, sx = oracle.linear(inp["X"][rows], inp["W"], inp["bias"], inp["A"], inp["B"], skip=skip,
                                 want_sx=True)
    worst, fro = helpers.y_tolerance_check(y, y_ref, sx, helpers.f32(inp["W"]).astype(np.float64))
    assert worst <= 1.0 and fro <= 5e-3, (layer, skip, worst, fro)


def test_sweep_with_gelu_on_up_layers():
    """The sweep with the MLP up-projections' GELU in their GEMM epilogue: the
    graph replays the eager pass bit for bit, and an up layer matches the
    oracle's gelu_tanh(linear) within the layer's bar times GELU's largest
    slope (1.13)."""
    torch.cuda.set_device(0)
    plan = workloads.sweep_plan(M=384)[:8]  # two blocks
    layers = []
    for (_b, name, M, K, N, kind, skip, seed) in plan:
        inp = workloads.make_linear_inputs(M, K, N, seed=seed, x_kind=kind)
        inp["skip"] = skip
        if name == "up":
            inp["act"] = lynx.LYNX_ACT_GELU_TANH
        layers.append(inp)
    sweep = LinearSweep(layers, device="cuda:0")
    sweep.run()
    torch.cuda.synchronize()
    eager = [t["Y"].clone() for t in sweep.layers]
    for t in sweep.layers:
        t["Y"].zero_()
    sweep.capture()
    sweep.replay()
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    for t, e in zip(sweep.layers, eager):
        assert torch.equal(t["Y"].view(torch.int16), e.view(torch.int16))
    i = next(i for i, p in enumerate(plan) if p[1] == "up")
    inp = layers[i]
    rows = np.array([0, 5, 127, 128, 255, 256, 383])
    y = helpers.f32(host(sweep.layers[i]["Y"])).astype(np.float64)[rows]
    y_pre, _, sx = oracle.linear(inp["X"][rows], inp["W"], inp["bias"], inp["A"], inp["B"],
                                 skip=inp["skip"], want_sx=True)
    y_ref = oracle.gelu_tanh(y_pre)
    bound = 1.13 * 2e-2 * np.outer(np.linalg.norm(sx, axis=1),
                                   np.linalg.norm(helpers.f32(inp["W"]).astype(np.float64), axis=1))
    assert float((np.abs(y - y_ref) / bound).max()) <= 1.0
    assert np.linalg.norm(y - y_ref) <= 1.13 * 5e-3 * np.linalg.norm(y_pre)


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda:0")


@pytest.mark.parametrize("skip,act,lora", [(False, lynx.LYNX_ACT_NONE, True), (True, lynx.LYNX_ACT_NONE, True),
                                           (False, lynx.LYNX_ACT_GELU_TANH, True),
                                           (False, lynx.LYNX_ACT_NONE, False),
                                           (True, lynx.LYNX_ACT_NONE, False)])
def test_begin_then_finish_on_two_streams_equals_linear(skip, act, lora):
    """lynx_linear_begin on one stream and lynx_linear_finish on another (after
    an event) give the same Y bits as lynx_linear_act, on the mlp_up shape."""
    torch.cuda.set_device(0)
    c = workloads.CONFIGS["mlp_up"]
    inp = workloads.make_config_inputs("mlp_up")
    X, W, bias, A, B = (dev(inp[k]) for k in ("X", "W", "bias", "A", "B"))
    if not lora:
        A = B = None
    ref = lynx.lynx_linear_act(X, W, bias, A, B, skip_sparsify=skip, act=act)
    s_begin, s_finish = torch.cuda.Stream(), torch.cuda.Stream()
    ws = torch.full((lynx.lynx_workspace_bytes(c.M, c.N, c.K, c.r),), 0xA5, dtype=torch.uint8, device="cuda:0")
    Y = torch.zeros_like(ref)
    torch.cuda.synchronize()
    lynx.lynx_linear_begin(X, W, bias, A, B, skip_sparsify=skip, act=act, Y=Y, workspace=ws, stream=s_begin)
    ev = torch.cuda.Event()
    ev.record(s_begin)
    s_finish.wait_event(ev)
    lynx.lynx_linear_finish(X, W, bias, A, B, skip_sparsify=skip, act=act, Y=Y, workspace=ws, stream=s_finish)
    torch.cuda.synchronize()
    for s in (s_begin, s_finish, None):
        st, code = lynx.lynx_check_error(s)
        assert st == lynx.LYNX_OK, (st, code)
    assert torch.equal(Y.view(torch.int16), ref.view(torch.int16))


def test_overlapped_schedules_equal_serial_calls(sweep_and_plan):
    """The overlapped sweep (passes on a side stream, GEMMs on the main one, two
    workspaces) eagerly and from a graph gives the serial pass's Y bits; with
    row blocks (384 rows: a 256-row block and a 128-row tail) every block
    equals a lynx_linear call on the same rows."""
    sweep, plan, layers = sweep_and_plan
    sweep.run()
    torch.cuda.synchronize()
    serial = [t["Y"].clone() for t in sweep.layers]

    def check(expected, what):
        torch.cuda.synchronize()
        st, code = lynx.lynx_check_error()
        assert st == lynx.LYNX_OK, (what, st, code)
        for side in sweep.side_streams():
            st, code = lynx.lynx_check_error(side)
            assert st == lynx.LYNX_OK, (what, st, code)
        for i, (t, e) in enumerate(zip(sweep.layers, expected)):
            assert torch.equal(t["Y"].view(torch.int16), e.view(torch.int16)), (what, plan[i][:2])

    for t in sweep.layers:
        t["Y"].zero_()
    sweep.run_overlapped(1)
    check(serial, "overlap eager")
    for t in sweep.layers:
        t["Y"].zero_()
    sweep.capture(overlapped=True, chunks=1)
    sweep.replay()
    sweep.replay()
    check(serial, "overlap graph")

    blocks = []
    for t in sweep.layers:
        y = torch.empty_like(t["Y"])
        for (tt, r0, r1) in sweep.work_items(2):
            if tt is t:
                y[r0:r1] = lynx.lynx_linear_act(t["X"][r0:r1], t["W"], t["bias"], t["A"], t["B"],
                                                skip_sparsify=t["skip"], act=t["act"])
        blocks.append(y)
    assert [(r0, r1) for (tt, r0, r1) in sweep.work_items(2) if tt is sweep.layers[0]] == [(0, 256), (256, 384)]
    for t in sweep.layers:
        t["Y"].zero_()
    sweep.run_overlapped(2)
    check(blocks, "row blocks eager")
    for t in sweep.layers:
        t["Y"].zero_()
    sweep.capture(overlapped=True, chunks=2)
    sweep.replay()
    check(blocks, "row blocks graph")
    sweep.graph = None
