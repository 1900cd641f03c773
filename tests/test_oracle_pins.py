"""Pins of the CPU oracle against what the RT-Lynx pages and mathematics fix.

None of these compares the oracle with itself: each check is a brute force,
a closed form, an invariant, a metamorphic relation, an independent library
routine (torch's bf16 rounding, numpy fp64 matmul) or a hand-derived worked
example (tests/golden).  Passages: qingkeai.online article 'RT-Lynx' sections
02-03 (Y = S(X) W^T, 2:4 Top-K on activations, norm compensation, LoRA
residual on the frozen backbone, selective layer skipping); ai-feeds.com
summary 'core module 1' (pruned L1 returned to the kept values in proportion).
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from activation_sparse_gemm_lynx_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sparsify_worked_examples.json")


def bits(x):
    return workloads.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f32(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def canon_nibbles(meta_row, K):
    """canonical bytes of one row -> list of (lo, hi) per group"""
    out = []
    for g in range(K // 4):
        byte = int(meta_row[g // 2])
        nib = (byte >> 4) if g & 1 else (byte & 0xF)
        out.append((nib & 3, (nib >> 2) & 3))
    return out


def brute_force_pair(mags):
    """All 6 masks of a group: the kept pair maximising the kept L1; among equal
    sums the lexicographically smallest sorted index pair.  For top-2 with ties
    to the lower index this is the same choice: a tie of sums can only come from
    a tie of magnitudes at the boundary of the top two.  Sums are exact
    rationals, so no rounding can create or hide a tie."""
    best = None
    for i, j in itertools.combinations(range(4), 2):
        sc = Fraction(mags[i]) + Fraction(mags[j])
        if best is None or sc > best[0]:
            best = (sc, (i, j))
    return best[1]


# --------------------------------------------------------------------------
# bf16 rounding


def test_bf16_rne_matches_torch(oracle_mod):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.389531389e38], dtype=np.float32),
    ])
    # exact midpoints between neighbouring bf16 values, both parities
    base = rng.integers(0x0080, 0x7F00, size=4000, dtype=np.uint32)
    mids = ((base << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, mids, -mids])
    got = oracle_mod.bf16_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rne_ties_go_to_even(oracle_mod):
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even neighbour is 1.0
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)], dtype=np.float32)
    got = f32(oracle_mod.bf16_rne(x))
    assert got.tolist() == [1.0, 1 + 2.0 ** -6, -1.0]


# --------------------------------------------------------------------------
# group selection (2:4 Top-K by magnitude, ties to the lower index)


def test_select_exhaustive_small_alphabet(oracle_mod):
    alphabet = [0.0, 1.0, -1.0, 2.0, -2.0, 3.0, -3.0]
    groups = np.array(list(itertools.product(alphabet, repeat=4)), dtype=np.float32)
    assert groups.shape == (7 ** 4, 4)
    lo, hi = oracle_mod.select_groups(bits(groups))
    for g, l, h in zip(groups, lo, hi):
        assert (l, h) == brute_force_pair(np.abs(g).tolist()), g


def test_select_signed_zero_is_a_tie(oracle_mod):
    g = np.array([[-0.0, 0.0, 0.0, -0.0], [0.0, -0.0, 1.0, 0.0], [0.0, 0.0, -0.0, -5.0]],
                 dtype=np.float32)
    lo, hi = oracle_mod.select_groups(bits(g))
    assert list(zip(lo.tolist(), hi.tolist())) == [(0, 1), (0, 2), (0, 3)]


def test_select_random_bf16_groups(oracle_mod):
    rng = np.random.default_rng(5)
    # raw bf16 bit patterns of finite values, with forced magnitude ties
    mag = rng.integers(0, 0x7F80, size=(30000, 4), dtype=np.uint16)
    tie = rng.random((30000, 4)) < 0.3
    mag = np.where(tie, mag[:, :1], mag)
    sign = (rng.random((30000, 4)) < 0.5).astype(np.uint16) << 15
    g = (mag | sign).astype(np.uint16)
    lo, hi = oracle_mod.select_groups(g)
    a = np.abs(f32(g)).astype(np.float64)
    for i in range(0, 30000, 7):
        assert (lo[i], hi[i]) == brute_force_pair(a[i].tolist())


# --------------------------------------------------------------------------
# S(X): invariants and closed forms


@pytest.fixture(scope="module")
def mix():
    inp = workloads.make_linear_inputs(96, 1024, 160, seed=123)
    return inp


def test_exactly_two_kept_per_group(oracle_mod, mix):
    X = mix["X"]
    r = oracle_mod.sparsify(X)
    M, K = X.shape
    for m in range(0, M, 5):
        for lo, hi in canon_nibbles(r["meta"][m], K):
            assert 0 <= lo < hi <= 3


def test_scale_closed_form_bounds(oracle_mod, mix):
    r = oracle_mod.sparsify(mix["X"])
    la64, lk64 = r["sums"][:, 2], r["sums"][:, 3]
    s64 = la64 / lk64
    # the top two of each group carry at least half of its L1
    assert np.all(s64 >= 1.0) and np.all(s64 <= 2.0)
    # fp32 s agrees with the exact ratio to fp32 sum accuracy
    assert np.allclose(r["scale"].astype(np.float64), s64, rtol=2e-5, atol=0)
    assert np.all((r["scale"] >= 1.0) & (r["scale"] <= 2.0 * (1 + 2 ** -20)))


def test_l1_norm_preserved(oracle_mod, mix):
    X = mix["X"]
    r = oracle_mod.sparsify(X)
    l1_dense = np.abs(f32(X).astype(np.float64)).sum(1)
    l1_sparse = np.abs(f32(r["vals"]).astype(np.float64)).sum(1)
    # each kept value is rounded once to bf16 (rel. error <= 2^-9)
    assert np.all(np.abs(l1_sparse - l1_dense) <= 2.0 ** -8 * l1_dense)


def test_vals_within_one_ulp_of_exact_scaling(oracle_mod, mix):
    X = mix["X"]
    M, K = X.shape
    r = oracle_mod.sparsify(X)
    s_exact = r["sums"][:, 2] / r["sums"][:, 3]
    xf = f32(X).astype(np.float64)
    got = f32(r["vals"]).astype(np.float64)
    for m in range(0, M, 3):
        pairs = canon_nibbles(r["meta"][m], K)
        kept = np.array([4 * g + p for g, (lo, hi) in enumerate(pairs) for p in (lo, hi)])
        want = xf[m, kept] * s_exact[m]
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
        assert np.all(np.abs(got[m] - want) <= ulp)


def test_kept_values_are_the_largest(oracle_mod, mix):
    X = mix["X"]
    M, K = X.shape
    r = oracle_mod.sparsify(X)
    a = np.abs(f32(X)).reshape(M, K // 4, 4)
    for m in range(0, M, 4):
        for g, (lo, hi) in enumerate(canon_nibbles(r["meta"][m], K)):
            drop = [i for i in range(4) if i not in (lo, hi)]
            assert min(a[m, g, lo], a[m, g, hi]) >= max(a[m, g, d] for d in drop)


def test_sign_flip_is_exact(oracle_mod, mix):
    X = mix["X"]
    r1 = oracle_mod.sparsify(X)
    r2 = oracle_mod.sparsify((X ^ np.uint16(0x8000)).astype(np.uint16))
    assert np.array_equal(r1["meta"], r2["meta"])
    assert np.array_equal(r1["scale"], r2["scale"])
    assert np.array_equal(r1["vals"] ^ np.uint16(0x8000), r2["vals"])


@pytest.mark.parametrize("p", [-3, 4])
def test_power_of_two_scaling_is_exact(oracle_mod, mix, p):
    X = mix["X"]
    Xs = bits(f32(X) * np.float32(2.0 ** p))
    assert np.array_equal(f32(Xs), f32(X) * np.float32(2.0 ** p))  # exact in bf16
    r1 = oracle_mod.sparsify(X)
    r2 = oracle_mod.sparsify(Xs)
    assert np.array_equal(r1["meta"], r2["meta"])
    assert np.array_equal(r1["scale"], r2["scale"])
    assert np.array_equal(f32(r1["vals"]) * np.float32(2.0 ** p), f32(r2["vals"]))


def test_group_permutation_invariance(oracle_mod, mix):
    X, W = mix["X"], mix["W"]
    M, K = X.shape
    rng = np.random.default_rng(9)
    perm_g = rng.permutation(K // 4)
    cols = (perm_g[:, None] * 4 + np.arange(4)[None, :]).reshape(-1)
    Y1, _, S1 = oracle_mod.linear(X, W, mix["bias"], want_sx=True)
    Y2, _, S2 = oracle_mod.linear(np.ascontiguousarray(X[:, cols]),
                                  np.ascontiguousarray(W[:, cols]), mix["bias"], want_sx=True)
    # same kept positions; values agree to one bf16 ulp (fp32 sum order moved)
    assert np.array_equal(S1[:, cols] != 0, S2 != 0)
    assert np.allclose(S1[:, cols], S2, rtol=2 ** -7, atol=0)
    ref = np.abs(S1) @ np.abs(f32(W).astype(np.float64)).T
    assert np.all(np.abs(Y1 - Y2) <= 2 ** -7 * ref + 1e-12)


# --------------------------------------------------------------------------
# reductions to textbook operations


def _all_keep_matrix(rng, M, K):
    x = rng.standard_normal((M, K)).astype(np.float32)
    z = np.zeros((M, K // 4, 4), dtype=bool)
    for m in range(M):
        for g in range(K // 4):
            z[m, g, rng.choice(4, 2, replace=False)] = True
    x = x.reshape(M, K // 4, 4)
    x[z] = 0.0
    return bits(x.reshape(M, K))


def test_all_keep_input_reduces_to_plain_gemm(oracle_mod):
    rng = np.random.default_rng(21)
    M, K, N = 48, 256, 72
    X = _all_keep_matrix(rng, M, K)
    inp = workloads.make_linear_inputs(M, K, N, seed=4)
    r = oracle_mod.sparsify(X)
    assert np.all(r["scale"] == np.float32(1.0))
    Y, T, SX = oracle_mod.linear(X, inp["W"], inp["bias"], want_sx=True)
    Xd = f32(X).astype(np.float64)
    assert np.array_equal(SX, Xd)
    ref = Xd @ f32(inp["W"]).astype(np.float64).T + f32(inp["bias"]).astype(np.float64)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    assert T is None


def test_skipped_layer_is_dense_linear_plus_lora(oracle_mod):
    M, K, N = 40, 320, 96
    inp = workloads.make_linear_inputs(M, K, N, r=64, seed=8)
    Y, T, SX = oracle_mod.linear(inp["X"], inp["W"], inp["bias"], inp["A"], inp["B"], skip=True,
                                 want_sx=True)
    Xd = f32(inp["X"]).astype(np.float64)
    Wd, Ad, Bd = (f32(inp[k]).astype(np.float64) for k in ("W", "A", "B"))
    bd = f32(inp["bias"]).astype(np.float64)
    assert np.array_equal(SX, Xd)
    assert np.allclose(T, Xd @ Ad.T, rtol=1e-12, atol=1e-14)
    assert np.allclose(Y, Xd @ Wd.T + bd + (Xd @ Ad.T) @ Bd.T, rtol=1e-12, atol=1e-12)


def test_lora_branch_reads_dense_x(oracle_mod):
    M, K, N = 40, 256, 80
    inp = workloads.make_linear_inputs(M, K, N, r=64, seed=10)
    Y, T, SX = oracle_mod.linear(inp["X"], inp["W"], inp["bias"], inp["A"], inp["B"],
                                 want_sx=True)
    Xd = f32(inp["X"]).astype(np.float64)
    Wd, Ad, Bd = (f32(inp[k]).astype(np.float64) for k in ("W", "A", "B"))
    bd = f32(inp["bias"]).astype(np.float64)
    assert not np.array_equal(SX, Xd)
    assert np.allclose(T, Xd @ Ad.T, rtol=1e-12, atol=1e-14)
    assert np.allclose(Y, SX @ Wd.T + bd + (Xd @ Ad.T) @ Bd.T, rtol=1e-12, atol=1e-12)


def test_dense_sx_matches_vals_and_meta(oracle_mod, mix):
    X = mix["X"]
    M, K = X.shape
    r = oracle_mod.sparsify(X)
    _, _, SX = oracle_mod.linear(X, mix["W"][:8], want_sx=True)
    v = f32(r["vals"]).astype(np.float64)
    for m in range(0, M, 7):
        dense = np.zeros(K)
        for g, (lo, hi) in enumerate(canon_nibbles(r["meta"][m], K)):
            dense[4 * g + lo] = v[m, 2 * g]
            dense[4 * g + hi] = v[m, 2 * g + 1]
        assert np.array_equal(dense, SX[m])


# --------------------------------------------------------------------------
# hand-derived worked examples


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_worked_examples(oracle_mod, case):
    x = np.array(case["x"], dtype=np.float32)
    xb = bits(x)
    assert np.array_equal(f32(xb), x), "fixture inputs must be exact bf16 values"
    K = len(x)
    pad = (-K) % 8  # metadata rows are whole bytes: pad with a zero group
    xp = np.concatenate([xb, np.zeros(pad, dtype=np.uint16)])[None, :]
    r = oracle_mod.sparsify(xp)
    pairs = canon_nibbles(r["meta"][0], K + pad)[: K // 4]
    assert [lo | (hi << 2) for lo, hi in pairs] == case["nibbles"]
    assert int(r["scale"].view(np.uint32)[0]) == int(case["s_bits"], 16)
    want = np.array(case["vals"], dtype=np.float32)
    got = f32(r["vals"][0, : K // 2])
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))  # -0 vs +0 too


# --------------------------------------------------------------------------
# GELU (tanh form), the optional output activation: pinned to torch's own
# fp64 GELU, to the function's odd-part identity, to its value and slope at 0
# and to its distance from the exact (erf) GELU it approximates.

def test_gelu_matches_torch_fp64(oracle_mod):
    v = np.concatenate([np.linspace(-4.0, 8.0, 2401),
                        np.random.default_rng(7).normal(-0.5, 1.0, 4000).clip(-4.0, None)])
    want = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    got = oracle_mod.gelu_tanh(v)
    # torch evaluates v/2 (1 + tanh u): its own rounding error relative to the
    # result grows like 1e-16 / (1 + tanh u) = 1e-16 / (2 e^(2u)), about 3e-12
    # at v = -4 (and 1e-9 at v = -5, where the comparison would test torch)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-300)


def test_gelu_odd_part_is_identity(oracle_mod):
    # (1 + tanh u)/2 - (1 - tanh u)/2 = tanh u ... so gelu(v) - gelu(-v) = v
    v = np.random.default_rng(8).normal(0.0, 3.0, 5000)
    d = oracle_mod.gelu_tanh(v) - oracle_mod.gelu_tanh(-v)
    np.testing.assert_allclose(d, v, rtol=1e-13, atol=1e-15)


def test_gelu_at_zero_and_tails(oracle_mod):
    g = oracle_mod.gelu_tanh(np.array([0.0, -1e-6, 1e-6, 40.0, -40.0]))
    assert g[0] == 0.0
    # slope 1/2 at the origin
    assert abs((g[2] - g[1]) / 2e-6 - 0.5) < 1e-9
    assert g[3] == 40.0 and g[4] == 0.0


def test_gelu_tanh_form_is_close_to_erf_gelu(oracle_mod):
    # the tanh form approximates v * Phi(v); the two stay within 1e-3 everywhere
    v = np.linspace(-8.0, 8.0, 16001)
    exact = torch.nn.functional.gelu(torch.from_numpy(v)).numpy()
    assert np.max(np.abs(oracle_mod.gelu_tanh(v) - exact)) < 1e-3
