"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars (the layer's stated tolerances):
  * metadata (kept positions) bit-exact, compared in the canonical layout;
  * compressed values within 1 bf16 ulp (the fp32 row sums are added in a
    different order on the GPU);
  * Y: elementwise |dY| <= 2e-2 * ||S(X)_m||_2 * ||W_n||_2 and relative
    Frobenius error <= 5e-3 (fp32 accumulation, one bf16 rounding).
Inputs come from the seeded generators; expected values only from the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gemm_lynx_b200 import lynx, workloads

import helpers
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


def run_sparsify(X):
    vals, meta, scale = lynx.lynx_sparsify(dev(X))
    torch.cuda.synchronize()
    return host(vals), meta.cpu().numpy(), scale.cpu().numpy()


def check_sparsify(X, vals, meta, scale):
    M, K = X.shape
    ref = oracle.sparsify(X)
    canon = helpers.canonical_from_hw(meta, M, K)
    assert np.array_equal(canon, ref["meta"]), "metadata differs from the oracle"
    # the library's own converter agrees with the test's reading of the layout
    assert np.array_equal(lynx.lynx_meta_hw_to_canonical(meta, M, K), canon)
    d = helpers.bf16_ulp_distance(vals, ref["vals"])
    assert int(d.max()) <= 1, f"values differ by {int(d.max())} ulp"
    assert np.allclose(scale, ref["scale"], rtol=4e-6, atol=0)
    return ref


# ---------------------------------------------------------------------------
# S(X)


def test_sparsify_tiny_config():
    inp = workloads.make_config_inputs("tiny")
    X = inp["X"]
    check_sparsify(X, *run_sparsify(X))


@pytest.mark.parametrize("M,K", [(1, 64), (130, 192), (300, 576), (257, 1024), (64, 3072),
                                 (129, 12288)])
def test_sparsify_shapes(M, K):
    X = workloads.make_linear_inputs(M, K, 8, seed=M + K)["X"]
    check_sparsify(X, *run_sparsify(X))


def test_sparsify_ties_and_zeros():
    rng = np.random.default_rng(3)
    M, K = 192, 512
    alphabet = np.array([0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5], dtype=np.float32)
    x = alphabet[rng.integers(0, len(alphabet), size=(M, K))]
    x[5] = 0.0                                        # an all-zero row: s = 1
    X = workloads.f32_to_bf16_bits(x)
    vals, meta, scale = run_sparsify(X)
    check_sparsify(X, vals, meta, scale)
    assert scale[5] == 1.0


def test_sparsify_all_keep_is_identity():
    rng = np.random.default_rng(4)
    M, K = 130, 256
    x = rng.standard_normal((M, K // 4, 4)).astype(np.float32)
    for m in range(M):
        for g in range(K // 4):
            x[m, g, rng.choice(4, 2, replace=False)] = 0.0
    X = workloads.f32_to_bf16_bits(x.reshape(M, K))
    vals, meta, scale = run_sparsify(X)
    check_sparsify(X, vals, meta, scale)
    assert np.all(scale == 1.0)
    dense = helpers.dense_from_canonical(vals, helpers.canonical_from_hw(meta, M, K), K)
    assert np.array_equal(dense, helpers.f32(X).astype(np.float64))


# ---------------------------------------------------------------------------
# the sparse product alone, on an oracle-made S(X)


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (200, 136, 576), (130, 1024, 256)])
def test_sparse_gemm_on_oracle_sx(M, N, K):
    inp = workloads.make_linear_inputs(M, K, N, seed=7)
    ref = oracle.sparsify(inp["X"])
    hw = helpers.hw_from_canonical(ref["meta"], M, K)
    Y = lynx.lynx_sparse_gemm(dev(ref["vals"]), torch.from_numpy(hw).to(DEV), dev(inp["W"]),
                              bias=dev(inp["bias"]))
    y = helpers.f32(host(Y)).astype(np.float64)
    SX = helpers.dense_from_canonical(ref["vals"], ref["meta"], K)
    Wd = helpers.f32(inp["W"]).astype(np.float64)
    y_ref = SX @ Wd.T + helpers.f32(inp["bias"]).astype(np.float64)
    worst, fro = helpers.y_tolerance_check(y, y_ref, SX, Wd)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)


def test_identity_weight_probe_pins_operand_layout():
    """W = I: Y must reproduce S(X) exactly (each output is one exact product),
    which pins the value and metadata layouts end to end."""
    M, K = 256, 512
    X = workloads.make_linear_inputs(M, K, 8, seed=31)["X"]
    eye = workloads.f32_to_bf16_bits(np.eye(K, dtype=np.float32))
    Y = lynx.lynx_linear(dev(X), dev(eye))
    vals, meta, _ = run_sparsify(X)
    dense = helpers.dense_from_canonical(vals, helpers.canonical_from_hw(meta, M, K), K)
    y = helpers.f32(host(Y)).astype(np.float64)
    assert np.array_equal(y, dense)
    ref = oracle.sparsify(X)
    ref_dense = helpers.dense_from_canonical(ref["vals"], ref["meta"], K)
    assert np.array_equal(y != 0, ref_dense != 0)


# ---------------------------------------------------------------------------
# the whole layer


def check_linear(inp, skip=False, rows=None):
    X, W = inp["X"], inp["W"]
    Y = lynx.lynx_linear(dev(X), dev(W), dev(inp["bias"]), dev(inp["A"]), dev(inp["B"]),
                         skip_sparsify=skip)
    torch.cuda.synchronize()
    y = helpers.f32(host(Y)).astype(np.float64)
    if rows is not None:
        X = X[rows]
        y = y[rows]
    y_ref, _, sx = oracle.linear(X, W, inp["bias"], inp["A"], inp["B"], skip=skip, want_sx=True)
    worst, fro = helpers.y_tolerance_check(y, y_ref, sx, helpers.f32(W).astype(np.float64))
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)
    return worst, fro


def test_linear_tiny_config():
    check_linear(workloads.make_config_inputs("tiny"))


def test_linear_dense_path_tiny_config():
    check_linear(workloads.make_config_inputs("tiny"), skip=True)


@pytest.mark.parametrize("M,N,K,bias,lora", [
    (300, 200, 576, True, True),     # ragged M and N, K % 128 == 64
    (1, 8, 64, True, True),          # smallest shape
    (129, 264, 1024, False, True),   # no bias
    (256, 1024, 512, True, False),   # no LoRA, BN = 256
    (200, 2048, 3072, True, True),   # cluster-split sparsify, several N tiles
])
def test_linear_shapes(M, N, K, bias, lora):
    inp = workloads.make_linear_inputs(M, K, N, seed=M * 3 + N, bias=bias, lora=lora)
    check_linear(inp)


@pytest.mark.parametrize("M,N,K", [(300, 200, 576), (256, 1024, 512)])
def test_linear_dense_shapes(M, N, K):
    inp = workloads.make_linear_inputs(M, K, N, seed=11)
    check_linear(inp, skip=True)


def test_linear_is_deterministic():
    inp = workloads.make_linear_inputs(384, 3072, 1024, seed=5)
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    y1 = host(lynx.lynx_linear(*args))
    y2 = host(lynx.lynx_linear(*args))
    assert np.array_equal(y1, y2)


def check_workspace(ws, inp, rows=None, r=64):
    """lynx_linear leaves in its workspace: the uncompensated kept values (exact
    copies of X), the metadata, s per row and T/s.  Checked on `rows`."""
    X = inp["X"]
    M, K = X.shape
    vals, meta, scale, t = helpers.workspace_views(ws.cpu().numpy(), M, K, r)
    rows = np.arange(M) if rows is None else rows
    canon = helpers.canonical_from_hw(meta, M, K)[rows]
    ref = oracle.sparsify(X[rows])
    assert np.array_equal(canon, ref["meta"])
    assert np.array_equal(vals[rows], helpers.kept_from_x(X[rows], canon, K))
    assert np.allclose(scale[rows], ref["scale"], rtol=4e-6, atol=0)
    _, t_ref, _ = oracle.linear(X[rows], inp["W"][:8], None, inp["A"], inp["B"][:8])
    assert t_ref.shape[1] == r
    s64 = ref["scale"].astype(np.float64)[:, None]
    t_over_s = t_ref / s64
    T = helpers.f32(t[rows]).astype(np.float64)
    # T/s rounded once to bf16 (2^-9 relative, plus the division) on top of a
    # K-term fp32 tensor-core accumulation, whose error is bounded by K * 2^-24
    # times the sum of |x_k a_k| (<= 2^-10 of it for K <= 16384)
    xa = np.abs(helpers.f32(X[rows]).astype(np.float64)) @ \
        np.abs(helpers.f32(inp["A"]).astype(np.float64)).T
    bound = 2 ** -8 * np.abs(t_over_s) + 2 ** -10 * xa / s64
    ratio = np.abs(T - t_over_s) / bound
    assert ratio.max() <= 1.0, f"T/s off: worst {ratio.max():.3g} of the bound"


def test_workspace_holds_kept_values_scale_and_t():
    inp = workloads.make_linear_inputs(200, 576, 64, seed=17)
    M, K = inp["X"].shape
    ws = torch.zeros(lynx.lynx_workspace_bytes(M, 64, K, 64), dtype=torch.uint8, device=DEV)
    lynx.lynx_linear(dev(inp["X"]), dev(inp["W"]), dev(inp["bias"]), dev(inp["A"]),
                     dev(inp["B"]), workspace=ws)
    torch.cuda.synchronize()
    check_workspace(ws, inp)


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times: Y on
# every row against the oracle, the workspace (selection, kept values, s, T/s)
# on sampled rows


@pytest.mark.parametrize("name", ["attn_out", "mlp_up", "mlp_down"])
def test_full_size_every_row(name):
    c = workloads.CONFIGS[name]
    inp = workloads.make_config_inputs(name)
    M, K = inp["X"].shape
    ws = torch.empty(lynx.lynx_workspace_bytes(M, c.N, K, 64), dtype=torch.uint8, device=DEV)
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    Y = lynx.lynx_linear(*args, workspace=ws)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    worst, fro = oracle_checks.linear_all_rows(host(Y), inp)
    assert worst <= 1.0 and fro <= 5e-3, (name, worst, fro)
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.choice(M, 28, replace=False)]))
    check_workspace(ws, inp, rows=rows)


# ---------------------------------------------------------------------------
# the dense path's own entry point


@pytest.mark.parametrize("M,N,K,lora", [
    (300, 200, 576, True),     # 1-CTA GEMM, ragged
    (512, 1024, 1024, True),   # CTA-pair GEMM, LoRA T combined inside the GEMM
    (384, 768, 512, False),    # CTA-pair GEMM, no LoRA: one kernel
])
def test_linear_dense_entry_point(M, N, K, lora):
    inp = workloads.make_linear_inputs(M, K, N, seed=M + N + K, lora=lora)
    Y = lynx.lynx_linear_dense(*[dev(inp[k]) for k in ("X", "W", "bias", "A", "B")])
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    worst, fro = oracle_checks.linear_all_rows(host(Y), inp, skip=True)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)


# ---------------------------------------------------------------------------
# LoRA ranks other than the pages' 64: r % 16 == 0 up to 256 (r = 48 leaves the
# last K = 32 step of the up-projection half empty)


@pytest.mark.parametrize("r", [16, 48, 128, 256])
@pytest.mark.parametrize("M,N,K", [(300, 200, 576), (512, 768, 1024)])
@pytest.mark.parametrize("skip", [False, True])
def test_linear_lora_ranks(r, M, N, K, skip):
    inp = workloads.make_linear_inputs(M, K, N, r=r, seed=r * 7 + M)
    ws = torch.empty(lynx.lynx_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=DEV)
    Y = lynx.lynx_linear(*[dev(inp[k]) for k in ("X", "W", "bias", "A", "B")], skip_sparsify=skip,
                         workspace=ws)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    worst, fro = oracle_checks.linear_all_rows(host(Y), inp, skip=skip)
    assert worst <= 1.0 and fro <= 5e-3, (r, worst, fro)
    if not skip:
        _, _, _, t = helpers.workspace_views(ws.cpu().numpy(), M, K, r)
        assert t.shape == (M, r)
        check_workspace(ws, inp, rows=np.array([0, 1, M // 2, M - 1]), r=r)


def test_garbage_workspace_and_stale_state_words():
    """The workspace needs no initial contents: with every 32-bit word set to 2
    (the 'combined' state of the GEMM's per-row-block words) and to -1, the
    layer still matches the oracle, since each call clears those words first."""
    inp = workloads.make_linear_inputs(512, 1024, 768, seed=21)
    ws = torch.empty(lynx.lynx_workspace_bytes(512, 768, 1024, 64), dtype=torch.uint8, device=DEV)
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    for fill in (2, -1):
        for skip in (False, True):
            ws.view(torch.int32).fill_(fill)
            Y = lynx.lynx_linear(*args, skip_sparsify=skip, workspace=ws)
            torch.cuda.synchronize()
            worst, fro = oracle_checks.linear_all_rows(host(Y), inp, skip=skip)
            assert worst <= 1.0 and fro <= 5e-3, (fill, skip, worst, fro)
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)


def test_layer_with_sms_held_by_another_stream():
    """The CTA-pair GEMM needs no co-residency of its grid: while kernels on
    other streams hold some SMs for about 20 ms, the layer at the mlp_up shape
    (a full-device grid) completes without a timeout and matches the oracle."""
    inp = workloads.make_config_inputs("mlp_up")
    M = inp["X"].shape[0]
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    Y = lynx.lynx_linear(*args)  # one-time set-up outside the contended run
    torch.cuda.synchronize()
    side = [torch.cuda.Stream() for _ in range(6)]
    cycles = 40_000_000  # about 20 ms at the B200's 1.965 GHz
    for sstream in side:
        with torch.cuda.stream(sstream):
            torch.cuda._sleep(cycles)  # one block spinning for about 20 ms
    Y.zero_()
    lynx.lynx_linear(*args, Y=Y)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    rows = np.unique(np.concatenate([[0, 1, 255, 256, M - 1], np.arange(7, M, 97)]))
    worst, fro = oracle_checks.linear_all_rows(host(Y)[rows], inp, rows=rows)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)


# ---------------------------------------------------------------------------
# errors


def test_bad_workspace_is_rejected_before_launch():
    inp = workloads.make_linear_inputs(128, 512, 256, seed=2)
    ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(lynx.LynxError) as e:
        lynx.lynx_linear(dev(inp["X"]), dev(inp["W"]), workspace=ws)
    assert e.value.status == lynx.LYNX_ERR_WORKSPACE_TOO_SMALL


def test_device_timeout_is_reported_and_context_survives():
    X = workloads.make_linear_inputs(256, 512, 8, seed=1)["X"]
    lynx.lynx_debug_set_stall(True)
    try:
        lynx.lynx_sparsify(dev(X))
        st, code = lynx.lynx_check_error()
    finally:
        lynx.lynx_debug_set_stall(False)
    assert st == lynx.LYNX_ERR_DEVICE_TIMEOUT
    assert code != 0
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK and code == 0
    # the context is still usable and the next call is correct
    check_sparsify(X, *run_sparsify(X))


def test_device_timeout_in_the_fused_layer():
    inp = workloads.make_linear_inputs(256, 512, 256, seed=6)
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    lynx.lynx_debug_set_stall(True)
    try:
        lynx.lynx_linear(*args)
        st, code = lynx.lynx_check_error()
    finally:
        lynx.lynx_debug_set_stall(False)
    assert st == lynx.LYNX_ERR_DEVICE_TIMEOUT and code != 0
    check_linear(inp)


def test_device_timeout_stays_with_its_stream():
    """A timeout raised by a call on one stream is reported by lynx_check_error
    on that stream only; a call on another stream reports OK and is correct."""
    inp = workloads.make_linear_inputs(256, 512, 256, seed=8)
    args = [dev(inp[k]) for k in ("X", "W", "bias", "A", "B")]
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    lynx.lynx_debug_set_stall(True)
    try:
        with torch.cuda.stream(a):
            lynx.lynx_linear(*args)
    finally:
        lynx.lynx_debug_set_stall(False)
    with torch.cuda.stream(b):
        Y = lynx.lynx_linear(*args)
    st_b, code_b = lynx.lynx_check_error(b)
    st_a, code_a = lynx.lynx_check_error(a)
    assert st_b == lynx.LYNX_OK and code_b == 0
    assert st_a == lynx.LYNX_ERR_DEVICE_TIMEOUT and code_a != 0
    assert lynx.lynx_check_error(a) == (lynx.LYNX_OK, 0)
    torch.cuda.synchronize()
    worst, fro = oracle_checks.linear_all_rows(host(Y), inp)
    assert worst <= 1.0 and fro <= 5e-3, (worst, fro)


def check_selection_all_rows(inp, chunk=1024):
    """lynx_linear in the benchmark's launch configuration, then its workspace on
    every row: metadata bit-exact, kept values exact copies of X, s within a few
    fp32 ulps of the oracle's (rows in chunks, to bound host memory)."""
    X = inp["X"]
    M, K = X.shape
    N = inp["W"].shape[0]
    ws = torch.empty(lynx.lynx_workspace_bytes(M, N, K, 64), dtype=torch.uint8, device=DEV)
    lynx.lynx_linear(*[dev(inp[k]) for k in ("X", "W", "bias", "A", "B")], workspace=ws)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    assert st == lynx.LYNX_OK, (st, code)
    vals, meta, scale, _ = helpers.workspace_views(ws.cpu().numpy(), M, K)
    for m0 in range(0, M, chunk):
        rows = np.arange(m0, min(M, m0 + chunk))
        ref = oracle.sparsify(X[rows])
        canon = helpers.canonical_from_hw(meta, M, K, rows)
        assert np.array_equal(canon, ref["meta"]), f"metadata differs in rows {m0}.."
        assert np.array_equal(vals[rows], helpers.kept_from_x(X[rows], canon, K)), f"values, rows {m0}.."
        assert np.allclose(scale[rows], ref["scale"], rtol=4e-6, atol=0), f"s, rows {m0}.."


@pytest.mark.parametrize("name", ["attn_out", "mlp_up", "mlp_down"])
def test_full_size_selection_on_every_row(name):
    check_selection_all_rows(workloads.make_config_inputs(name))


@pytest.mark.parametrize("layer", [0, 3])  # the sweep's qkv (K = 3072) and down (K = 12288) at M = 8192
def test_sweep_size_selection_on_every_row(layer):
    _b, _n, M, K, N, kind, _skip, seed = workloads.sweep_plan()[layer]
    check_selection_all_rows(workloads.make_linear_inputs(M, K, N, seed=seed, x_kind=kind))
