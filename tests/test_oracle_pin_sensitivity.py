"""The pins catch plausible oracle mistakes. Each test plants one mistake in a numpy
restatement of an oracle pass (on the CPU) and checks that the exact brute-force pin of
test_oracle_pins rejects it on the PyTorch issue 152668 repro (4 experts, x[48,8],
w[4,8,16], offsets (8,16,32,40) and the empty-expert (8,8,32,40)), while the same
restatement without the mistake, and the oracle itself, agree with the pin."""
import numpy as np
import pytest

import oracle
import workloads
from test_oracle_pins import _brute_dgrad, _brute_forward, _brute_wgrad, _f64

OFFSETS = [(8, 16, 32, 40), (8, 8, 32, 40)]


def _groups(offs, rows, mistake):
    """(start, end) of every group; mistakes of the group arithmetic are planted here."""
    out, prev = [], 0
    for e, o in enumerate(offs):
        s, t = prev, min(max(int(o), prev), rows)
        if mistake == "offsets_read_as_starts":
            s, t = int(o), (int(offs[e + 1]) if e + 1 < len(offs) else rows)
        if mistake == "last_row_dropped":
            t = max(s, t - 1)
        out.append((s, t))
        prev = min(max(int(o), prev), rows)
    return out


def _forward(A, W, offs, mistake=None):
    A, W = _f64(A), _f64(W)
    E = W.shape[0]
    out = {}
    for e, (s, t) in enumerate(_groups(offs, A.shape[0], mistake)):
        we = W[(e + 1) % E] if mistake == "wrong_expert" else W[e]
        for r in range(s, t):
            row = A[r] @ we
            for n in range(W.shape[2]):
                out[(r, n)] = row[n]
    return out


def _dgrad(dY, W, offs, mistake=None):
    dY, W = _f64(dY), _f64(W)
    E = W.shape[0]
    out = {}
    for e, (s, t) in enumerate(_groups(offs, dY.shape[0], mistake)):
        we = W[(e + 1) % E] if mistake == "wrong_expert" else W[e]
        for r in range(s, t):
            row = we @ dY[r]
            for k in range(W.shape[1]):
                out[(r, k)] = row[k]
    return out


def _wgrad(A, dY, offs, E, mistake=None):
    A, dY = _f64(A), _f64(dY)
    out = np.zeros((E, A.shape[1], dY.shape[1]))
    groups = _groups(offs, A.shape[0], mistake)
    for e in range(E):
        s, t = groups[e - 1] if (mistake == "previous_group" and e > 0) else groups[e]
        out[e] = A[s:t].T @ dY[s:t]
    return out


def _agree(got, want):
    if isinstance(want, dict):
        if set(got) != set(want):
            return False
        return all(abs(got[k] - want[k]) <= 1e-12 * max(1.0, abs(want[k])) for k in want)
    return np.allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("offs", OFFSETS)
def test_restatements_without_mistakes_agree_with_the_pins(offs):
    r = workloads.make_tiny(offs)
    assert _agree(_forward(r.A, r.W, offs), _brute_forward(r.A, r.W, offs))
    assert _agree(_dgrad(r.dY, r.W, offs), _brute_dgrad(r.dY, r.W, offs))
    assert _agree(_wgrad(r.A, r.dY, offs, r.E), _brute_wgrad(r.A, r.dY, offs, r.E))


@pytest.mark.parametrize("offs", OFFSETS)
@pytest.mark.parametrize("mistake", ["wrong_expert", "offsets_read_as_starts", "last_row_dropped"])
def test_pins_reject_forward_and_dgrad_mistakes(offs, mistake):
    r = workloads.make_tiny(offs)
    assert not _agree(_forward(r.A, r.W, offs, mistake), _brute_forward(r.A, r.W, offs))
    assert not _agree(_dgrad(r.dY, r.W, offs, mistake), _brute_dgrad(r.dY, r.W, offs))


@pytest.mark.parametrize("offs", OFFSETS)
@pytest.mark.parametrize("mistake", ["previous_group", "offsets_read_as_starts", "last_row_dropped"])
def test_pins_reject_wgrad_mistakes(offs, mistake):
    r = workloads.make_tiny(offs)
    assert not _agree(_wgrad(r.A, r.dY, offs, r.E, mistake),
                      _brute_wgrad(r.A, r.dY, offs, r.E))


def test_the_oracle_itself_agrees_with_the_pins():
    r = workloads.make_tiny((8, 8, 32, 40))
    out, grp = oracle.forward(r.A, r.W, r.offs)
    want = _brute_forward(r.A, r.W, r.offs)
    assert all(out[rn[0], rn[1]] == v for rn, v in want.items())
    assert all(grp[row] < 0 for row in range(40, 48))
