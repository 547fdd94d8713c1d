"""Pins for the CPU oracle, each against something other than the oracle itself.

* exact rational brute force (``fractions.Fraction``) on tiny inputs, written here from the
  definitions out[r,n] = sum_k A[r,k] W[e,k,n], dX[r,k] = sum_n dY[r,n] W[e,k,n],
  dW[e,k,n] = sum_{r in e} A[r,k] dY[r,n];
* the concatenation identity: the grouped result equals the row-concatenation of per-group
  dense GEMMs done by ``numpy`` float64 matmul;
* special cases that reduce to one dense GEMM (all experts equal; sum over experts of dW);
* invariances (expert relabelling; masked layout == packed contiguous layout);
* exact small-integer probes of group membership;
* the shapes and offsets printed in PyTorch issue 152668 ("Easy repro scenario").
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_shapes.json")


def _f64(t):
    return oracle.bf16_to_f64(oracle.as_u16(t))


def _bounds_plain(offs, rows_alloc):
    """Group bounds written out independently: start = previous end, end = offs[e]."""
    starts, ends, prev = [], [], 0
    for o in offs:
        t = min(max(int(o), prev), rows_alloc)
        starts.append(prev)
        ends.append(t)
        prev = t
    return starts, ends


def _brute_forward(A, W, offs):
    A, W = _f64(A), _f64(W)
    starts, ends = _bounds_plain(offs, A.shape[0])
    out = {}
    for e, (s, t) in enumerate(zip(starts, ends)):
        for r in range(s, t):
            for n in range(W.shape[2]):
                acc = Fraction(0)
                for k in range(A.shape[1]):
                    acc += Fraction(A[r, k]) * Fraction(W[e, k, n])
                out[(r, n)] = float(acc)
    return out


def _brute_dgrad(dY, W, offs):
    dY, W = _f64(dY), _f64(W)
    starts, ends = _bounds_plain(offs, dY.shape[0])
    out = {}
    for e, (s, t) in enumerate(zip(starts, ends)):
        for r in range(s, t):
            for k in range(W.shape[1]):
                acc = Fraction(0)
                for n in range(dY.shape[1]):
                    acc += Fraction(dY[r, n]) * Fraction(W[e, k, n])
                out[(r, k)] = float(acc)
    return out


def _brute_wgrad(A, dY, offs, E):
    A, dY = _f64(A), _f64(dY)
    starts, ends = _bounds_plain(offs, A.shape[0])
    out = np.zeros((E, A.shape[1], dY.shape[1]))
    for e, (s, t) in enumerate(zip(starts, ends)):
        for k in range(A.shape[1]):
            for n in range(dY.shape[1]):
                acc = Fraction(0)
                for r in range(s, t):
                    acc += Fraction(A[r, k]) * Fraction(dY[r, n])
                out[e, k, n] = float(acc)
    return out


def _fp64_bound(terms_abs_sum, n):
    """Rigorous bound on recursive fp64 summation error of n exact products."""
    u = 2.0 ** -53
    g = n * u / (1 - n * u)
    return g * terms_abs_sum + 1e-300


TINY_OFFSET_CASES = [
    (8, 16, 32, 40), (8, 8, 32, 40), (0, 16, 32, 40), (8, 16, 32, 32),
    (0, 0, 0, 0), (40, 40, 40, 40), (48, 48, 48, 48),
]


@pytest.mark.parametrize("offs", TINY_OFFSET_CASES)
def test_forward_dgrad_wgrad_match_exact_bruteforce_tiny(offs):
    t = workloads.make_tiny(offs)
    out, g = oracle.forward(t.A, t.W, t.offs)
    bf = _brute_forward(t.A, t.W, offs)
    for (r, n), v in bf.items():
        assert out[r, n] == v, (r, n, out[r, n], v)
    covered = {r for (r, _) in bf}
    for r in range(48):
        if r not in covered:
            assert g[r] == -1 and np.all(np.isnan(out[r]))
    dx, _ = oracle.dgrad(t.dY, t.W, t.offs)
    for (r, k), v in _brute_dgrad(t.dY, t.W, offs).items():
        assert dx[r, k] == v
    dw = oracle.wgrad(t.A, t.dY, t.offs)
    np.testing.assert_array_equal(dw, _brute_wgrad(t.A, t.dY, offs, 4))


SWEEP = [0, 1, 7, 8, 9, 15, 16, 17]


@pytest.mark.parametrize("K,N", [(8, 16), (16, 8), (32, 24)])
def test_size_sweep_within_rigorous_fp64_bound_of_exact(K, N):
    sizes = SWEEP
    r = workloads.make_ragged_custom(len(sizes), K, N, sizes, seed=11 + K, tail=5)
    offs = r.offs
    out, _ = oracle.forward(r.A, r.W, offs)
    A, W, dY = _f64(r.A), _f64(r.W), _f64(r.dY)
    for (row, n), v in _brute_forward(r.A, r.W, offs).items():
        e = int(np.searchsorted(offs, row, side="right"))
        bound = _fp64_bound(float(np.sum(np.abs(A[row] * W[e, :, n]))), K)
        assert abs(out[row, n] - v) <= bound
    dx, _ = oracle.dgrad(r.dY, r.W, offs)
    for (row, k), v in _brute_dgrad(r.dY, r.W, offs).items():
        e = int(np.searchsorted(offs, row, side="right"))
        bound = _fp64_bound(float(np.sum(np.abs(dY[row] * W[e, k, :]))), N)
        assert abs(dx[row, k] - v) <= bound
    dw = oracle.wgrad(r.A, r.dY, offs)
    ex = _brute_wgrad(r.A, r.dY, offs, len(sizes))
    assert np.all(np.abs(dw - ex) <= 1e-12 * (1 + np.abs(ex)))
    # empty group -> exact zeros
    assert np.all(dw[0] == 0.0)


def _concat_reference(A, W, offs):
    A, W = _f64(A), _f64(W)
    parts = []
    prev = 0
    for e, t in enumerate(offs):
        parts.append(A[prev:t] @ W[e])
        prev = t
    return np.concatenate(parts, axis=0)


@pytest.mark.parametrize("sizes", [[37, 0, 64, 129, 5], [0, 0, 200], [300]])
def test_concatenation_identity_against_numpy(sizes):
    r = workloads.make_ragged_custom(len(sizes), 96, 40, sizes, seed=5, tail=7)
    T = r.T
    out, _ = oracle.forward(r.A, r.W, r.offs)
    ref = _concat_reference(r.A, r.W, r.offs)
    np.testing.assert_allclose(out[:T], ref, rtol=1e-12, atol=1e-12)
    assert np.all(np.isnan(out[T:]))
    dx, _ = oracle.dgrad(r.dY, r.W, r.offs)
    Wt = torch.stack([r.W[e].t().contiguous() for e in range(r.E)])
    ref_dx = _concat_reference(r.dY, Wt, r.offs)
    np.testing.assert_allclose(dx[:T], ref_dx, rtol=1e-12, atol=1e-12)
    dw = oracle.wgrad(r.A, r.dY, r.offs)
    A, dY = _f64(r.A), _f64(r.dY)
    prev = 0
    for e, t in enumerate(r.offs):
        np.testing.assert_allclose(dw[e], A[prev:t].T @ dY[prev:t], rtol=1e-12, atol=1e-12)
        prev = t


def test_equal_experts_reduce_to_dense_gemm():
    sizes = [50, 0, 77, 13]
    r = workloads.make_ragged_custom(4, 64, 48, sizes, seed=21, tail=3)
    W = r.W.clone()
    W[:] = W[0]
    out, _ = oracle.forward(r.A, W, r.offs)
    A, Wd, dY = _f64(r.A), _f64(W[0]), _f64(r.dY)
    T = r.T
    np.testing.assert_allclose(out[:T], A[:T] @ Wd, rtol=1e-12, atol=1e-12)
    dx, _ = oracle.dgrad(r.dY, W, r.offs)
    np.testing.assert_allclose(dx[:T], dY[:T] @ Wd.T, rtol=1e-12, atol=1e-12)


def test_wgrad_sums_to_dense_over_experts():
    sizes = [31, 0, 90, 1, 17]
    r = workloads.make_ragged_custom(5, 40, 24, sizes, seed=23, tail=9)
    dw = oracle.wgrad(r.A, r.dY, r.offs)
    A, dY = _f64(r.A), _f64(r.dY)
    T = r.T
    np.testing.assert_allclose(dw.sum(0), A[:T].T @ dY[:T], rtol=1e-11, atol=1e-11)


def test_expert_relabelling_permutes_results_bit_exactly():
    sizes = np.array([20, 0, 33, 7, 41])
    r = workloads.make_ragged_custom(5, 32, 24, sizes, seed=29, tail=0)
    perm = np.array([3, 0, 4, 2, 1])  # new expert j is old expert perm[j]
    old_starts = np.concatenate([[0], np.cumsum(sizes)[:-1]])
    rows = np.concatenate([np.arange(old_starts[p], old_starts[p] + sizes[p]) for p in perm])
    A2, dY2, W2 = r.A[rows], r.dY[rows], r.W[perm]
    offs2 = np.cumsum(sizes[perm]).astype(np.int32)
    out, _ = oracle.forward(r.A, r.W, r.offs)
    out2, _ = oracle.forward(A2, W2, offs2)
    np.testing.assert_array_equal(out2, out[rows])
    dx, _ = oracle.dgrad(r.dY, r.W, r.offs)
    dx2, _ = oracle.dgrad(dY2, W2, offs2)
    np.testing.assert_array_equal(dx2, dx[rows])
    dw = oracle.wgrad(r.A, r.dY, r.offs)
    dw2 = oracle.wgrad(A2, dY2, offs2)
    np.testing.assert_array_equal(dw2, dw[perm])


def test_masked_equals_packed_contiguous_bit_exactly():
    m = workloads.make_masked(E=4, mmax=32, K=64, N=40, masked_m=[5, 0, 32, 17], seed=31)
    out, act, bad = oracle.masked_forward(m.A, m.W, m.masked_m)
    assert not bad
    rows = np.concatenate([e * 32 + np.arange(c) for e, c in enumerate(m.masked_m)])
    packed = m.A.reshape(-1, 64)[rows]
    offs = np.cumsum(m.masked_m).astype(np.int32)
    ref, _ = oracle.forward(packed, m.W, offs)
    np.testing.assert_array_equal(out[rows], ref)
    assert act.sum() == len(rows)
    inactive = np.setdiff1d(np.arange(4 * 32), rows)
    assert np.all(np.isnan(out[inactive])) and not act[inactive].any()


def test_masked_clamps_out_of_range_counts():
    m = workloads.make_masked(E=3, mmax=16, K=32, N=8, masked_m=[-3, 40, 7], seed=33,
                              nan_inactive=False)
    out, act, bad = oracle.masked_forward(m.A, m.W, m.masked_m)
    assert bad
    assert act.reshape(3, 16).sum(1).tolist() == [0, 16, 7]


def test_group_id_probe_is_exact():
    """A[:,0]=1, rest 0; W[e][0,n]=e+1, rest 0 -> out[r,n] = e(r)+1 exactly; the wgrad
    probe dW[e][0,n] = m_e*(e+1) with dY[r,:] = e(r)+1."""
    sizes = [3, 0, 9, 1, 12]
    E, K, N = 5, 16, 8
    offs = np.cumsum(sizes).astype(np.int32)
    rows_alloc = int(offs[-1]) + 4
    A = torch.zeros(rows_alloc, K, dtype=torch.bfloat16)
    A[:, 0] = 1
    W = torch.zeros(E, K, N, dtype=torch.bfloat16)
    for e in range(E):
        W[e, 0, :] = e + 1
    out, g = oracle.forward(A, W, offs)
    expect_group = np.concatenate([np.full(s, e) for e, s in enumerate(sizes)] + [[-1] * 4])
    np.testing.assert_array_equal(g, expect_group)
    for r in range(int(offs[-1])):
        assert np.all(out[r] == g[r] + 1)
    dY = torch.zeros(rows_alloc, N, dtype=torch.bfloat16)
    for r in range(int(offs[-1])):
        dY[r, :] = int(expect_group[r]) + 1
    dw = oracle.wgrad(A, dY, offs)
    for e in range(E):
        assert np.all(dw[e, 0] == sizes[e] * (e + 1))
        assert np.all(dw[e, 1:] == 0)


def test_clamp_rule_for_invalid_offsets():
    s, e, bad = oracle.group_bounds([8, 4, 60, -1], 48)
    assert bad
    assert s.tolist() == [0, 8, 8, 48] and e.tolist() == [8, 8, 48, 48]
    s, e, bad = oracle.group_bounds([8, 16, 32, 40], 48)
    assert not bad and s.tolist() == [0, 8, 16, 32] and e.tolist() == [8, 16, 32, 40]


def test_page_pins_tiny_repro():
    g = json.load(open(GOLDEN))["tiny_repro"]
    for key, rows_key in (("offsets_ok", "expect_group_rows_ok"),
                          ("offsets_empty_expert", "expect_group_rows_empty_expert")):
        t = workloads.make_tiny(tuple(g[key]))
        assert tuple(t.A.shape) == (g["M"], g["K"])
        assert tuple(t.W.shape) == (g["E"], g["K"], g["N"])
        out, grp = oracle.forward(t.A, t.W, t.offs)
        dx, _ = oracle.dgrad(t.dY, t.W, t.offs)
        dw = oracle.wgrad(t.A, t.dY, t.offs)
        assert list(out.shape) == g["expect_out_shape"]
        assert list(dx.shape) == g["expect_dx_shape"]
        assert list(dw.shape) == g["expect_dw_shape"]
        counts = [int((grp == e).sum()) for e in range(g["E"])]
        assert counts == g[rows_key]
        lo, hi = g["unused_rows"]
        assert np.all(grp[lo:hi] == -1)
        assert oracle.untouched_rows(t.offs, g["M"]).tolist() == list(range(lo, hi))
        assert np.all(np.isfinite(out[:lo])) and np.all(np.isfinite(dw))
        if key == "offsets_empty_expert":
            assert np.all(dw[1] == 0.0)


def test_nan_in_unused_rows_never_reaches_results():
    t = workloads.make_tiny(nan_tail=True)
    t2 = workloads.make_tiny(nan_tail=False)
    a, _ = oracle.forward(t.A, t.W, t.offs)
    b, _ = oracle.forward(t2.A, t2.W, t2.offs)
    np.testing.assert_array_equal(a[:40], b[:40])
    np.testing.assert_array_equal(oracle.wgrad(t.A, t.dY, t.offs),
                                  oracle.wgrad(t2.A, t2.dY, t2.offs))


def test_round_bf16_matches_torch_on_float_values_and_ties():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        [0.0, -0.0, 1e-39, -3e-40, 3.3e38, 3.4e38, -3.5e38, np.inf]])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.round_bf16(x32.astype(np.float64)), ref)
    # ties to even, and a double just above a tie must round up (no double rounding)
    assert oracle.round_bf16([1 + 2 ** -8])[0] == 0x3F80
    assert oracle.round_bf16([1 + 3 * 2 ** -8])[0] == 0x3F82
    assert oracle.round_bf16([1 + 2 ** -8 + 2 ** -40])[0] == 0x3F81


def test_wgrad_accumulate_reduces_and_is_exact_on_integers():
    """The fp32 accumulating wgrad: alpha=1,beta=0 is plain wgrad; alpha=0 leaves beta*old;
    small integers give exact values; NaN in `old` is ignored when beta == 0."""
    sizes = [5, 0, 9]
    r = workloads.make_ragged_custom(3, 16, 24, sizes, seed=71, tail=2)
    old = np.random.default_rng(1).standard_normal((3, 16, 24)).astype(np.float32)
    base = oracle.wgrad(r.A, r.dY, r.offs)
    np.testing.assert_array_equal(oracle.wgrad_accumulate(r.A, r.dY, r.offs, old, 1.0, 0.0), base)
    np.testing.assert_array_equal(oracle.wgrad_accumulate(r.A, r.dY, r.offs, old, 0.0, 2.0),
                                  2.0 * old.astype(np.float64))
    nan_old = np.full((3, 16, 24), np.nan, np.float32)
    assert np.all(np.isfinite(oracle.wgrad_accumulate(r.A, r.dY, r.offs, nan_old, 0.5, 0.0)))
    # integer probe: A = 1, dY = 2 on group rows; old = 3 -> dW = alpha*2*m_e + beta*3
    A = torch.ones(16, 4, dtype=torch.bfloat16)
    dY = torch.full((16, 8), 2.0, dtype=torch.bfloat16)
    offs = np.array([5, 5, 14], np.int32)
    got = oracle.wgrad_accumulate(A, dY, offs, np.full((3, 4, 8), 3.0, np.float32), 0.5, -1.0)
    for e, m in enumerate([5, 0, 9]):
        assert np.all(got[e] == 0.5 * 2 * m - 3.0)


def test_epilogue_bias_and_scale_reduce_exactly():
    """Zero weights leave s[r]*bias[e] exactly; no bias and act 0 is the plain forward."""
    sizes = [3, 0, 5]
    r = workloads.make_ragged_custom(3, 16, 256, sizes, seed=77, tail=2)
    bias = torch.randn(3, 256).to(torch.bfloat16)
    scale = np.linspace(-2, 2, r.rows_alloc)
    out, g = oracle.forward_ex(r.A, torch.zeros_like(r.W), r.offs, bias, scale)
    b = _f64(bias)
    for row in range(r.T):
        assert np.all(out[row] == scale[row] * b[g[row]])
    plain, _ = oracle.forward(r.A, r.W, r.offs)
    same, _ = oracle.forward_ex(r.A, r.W, r.offs)
    np.testing.assert_array_equal(same, plain)


def test_epilogue_silu_mul_layout_and_closed_form():
    """A one-hot, W[0,0,n] a distinct bf16-exact label per column: output column 128b+i must
    be silu(gate) * up of gate column 256b+i and up column 256b+128+i (silu by math.exp)."""
    import math
    N, K = 512, 16
    A = torch.zeros(4, K, dtype=torch.bfloat16)
    A[:, 0] = 1
    n = torch.arange(N, dtype=torch.float32)
    labels = torch.where(n < 256, n / 64.0, (n - 384.0) / 64.0)  # <= 8 significant bits
    W = torch.zeros(1, K, N, dtype=torch.bfloat16)
    W[0, 0, :] = labels
    assert torch.equal(W[0, 0].float(), labels)
    out, _ = oracle.forward_ex(A, W, [4], act=1)
    assert out.shape == (4, N // 2)
    for b in range(N // 256):
        for i in range(128):
            gte = float(labels[256 * b + i])
            up = float(labels[256 * b + 128 + i])
            want = gte / (1.0 + math.exp(-gte)) * up
            assert abs(out[3, 128 * b + i] - want) <= 1e-15 * max(1.0, abs(want))


def test_epilogue_silu_mul_concatenated_halves():
    """The same exact labels with gate and up as the two halves of N: output column j must be
    silu(gate column j) * up column N/2 + j; and permuting W's columns from the concatenated
    order into the 128-block interleaved order gives the interleaved result bit for bit."""
    import math
    N, K = 512, 16
    A = torch.zeros(4, K, dtype=torch.bfloat16)
    A[:, 0] = 1
    n = torch.arange(N, dtype=torch.float32)
    labels = torch.where(n < 256, n / 64.0, (n - 384.0) / 64.0)  # <= 8 significant bits
    W = torch.zeros(1, K, N, dtype=torch.bfloat16)
    W[0, 0, :] = labels
    out, _ = oracle.forward_ex(A, W, [4], act=1, concat=True)
    assert out.shape == (4, N // 2)
    for j in range(N // 2):
        gte, up = float(labels[j]), float(labels[N // 2 + j])
        want = gte / (1.0 + math.exp(-gte)) * up
        assert abs(out[3, j] - want) <= 1e-15 * max(1.0, abs(want))
    # concatenated column c -> interleaved position: gate j -> 256 (j // 128) + j % 128,
    # up j -> that + 128
    perm = torch.empty(N, dtype=torch.long)
    j = torch.arange(N // 2)
    perm[256 * (j // 128) + j % 128] = j
    perm[256 * (j // 128) + 128 + j % 128] = N // 2 + j
    inter, _ = oracle.forward_ex(A, W[:, :, perm], [4], act=1)
    np.testing.assert_array_equal(inter, out)


def _route_brute(ids, X, E):
    """Obviously-correct routing: for each expert in order, every assignment in order."""
    ids = np.asarray(ids)
    T, k = ids.shape
    rows, row_of, offs = [], np.full(T * k, -1, np.int32), []
    for e in range(E):
        for t in range(T):
            for s in range(k):
                if ids[t, s] == e:
                    row_of[t * k + s] = len(rows)
                    rows.append(t)
        offs.append(len(rows))
    Xu = oracle.as_u16(X)
    return np.array(offs, np.int32), row_of, Xu[rows] if rows else Xu[:0]


def test_route_matches_brute_force_and_invariants():
    ids, X = workloads.make_routing(37, 3, 6, 16, seed=5, dropped=4)
    ids[0, 0] = 9  # out of range: dropped and flagged
    offs, row_of, Ap, bad = oracle.route(ids, X, 6)
    boffs, brow, bA = _route_brute(ids, X, 6)
    np.testing.assert_array_equal(offs, boffs)
    np.testing.assert_array_equal(row_of, brow)
    np.testing.assert_array_equal(Ap, bA)
    assert bad
    # every packed row of group e came from an assignment to expert e
    flat = ids.reshape(-1)
    starts = np.concatenate([[0], offs[:-1]])
    for i, r in enumerate(row_of):
        if r >= 0:
            e = flat[i]
            assert starts[e] <= r < offs[e]
    assert offs[-1] == np.count_nonzero((flat >= 0) & (flat < 6))
