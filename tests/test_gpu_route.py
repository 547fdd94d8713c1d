"""Device token routing (gg_route) against the oracle: offsets, packed rows and packed
activations bit for bit, dropped and invalid assignments, and routing followed by the
grouped GEMM."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import cuda_ok
from helpers import assert_close, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")


def _route(ids, X, E):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = ids.shape[0] * ids.shape[1]
    A_packed = torch.full((n, X.shape[1]), float("nan"), dtype=torch.bfloat16, device="cuda")
    Ap, row_of, offs = gg.route(torch.from_numpy(ids).cuda(), X.cuda(), E, A_packed=A_packed,
                                status=st)
    torch.cuda.synchronize()
    return Ap, row_of.cpu().numpy(), offs.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("T,k,E,K,dropped", [(37, 3, 6, 16, 4), (4096, 8, 64, 2048, 0),
                                             (1000, 4, 1024, 64, 100), (5, 1, 1, 8, 0),
                                             (300, 2, 33, 136, 599), (4096, 4, 8, 64, 0),
                                             (20000, 2, 3, 16, 50)])
def test_route_bit_exact(T, k, E, K, dropped):
    """Stable routing equal to the oracle's; the last two cases split each expert's 64 and
    157 per-block histograms into 4 and 8 scan segments (the last one partial)."""
    ids, X = workloads.make_routing(T, k, E, K, seed=T + E, dropped=min(dropped, T * k))
    Ap, row_of, offs, st = _route(ids, X, E)
    roffs, rrow, rA, bad = oracle.route(ids, X, E)
    assert not bad and (st & gg.DEV_ERROR_MASK) == 0
    np.testing.assert_array_equal(offs, roffs)
    np.testing.assert_array_equal(row_of, rrow)
    total = int(roffs[-1])
    got = oracle.as_u16(Ap[:total])
    np.testing.assert_array_equal(got, rA)


def test_route_flags_out_of_range_ids():
    ids, X = workloads.make_routing(64, 2, 8, 32, seed=9)
    ids[3, 1] = 8
    ids[10, 0] = 1000
    Ap, row_of, offs, st = _route(ids, X, 8)
    roffs, rrow, _, bad = oracle.route(ids, X, 8)
    assert bad and st & gg.DEV_BAD_ROUTE
    np.testing.assert_array_equal(offs, roffs)
    np.testing.assert_array_equal(row_of, rrow)
    assert row_of[3 * 2 + 1] == -1 and row_of[10 * 2] == -1


def test_route_of_no_tokens():
    ids = np.zeros((0, 4), np.int32)
    X = torch.zeros(0, 64, dtype=torch.bfloat16)
    _, row_of, offs, st = _route(ids, X, 7)
    assert offs.tolist() == [0] * 7 and row_of.size == 0


def test_route_then_grouped_gemm():
    """The routed layout feeds the grouped GEMM directly (offsets never leave the device)."""
    ids, X = workloads.make_routing(512, 4, 16, 256, seed=13)
    W = (torch.randn(16, 256, 384) / 16).to(torch.bfloat16)
    Ap, row_of, offs = gg.route(torch.from_numpy(ids).cuda(), X.cuda(), 16)
    out = torch.empty(Ap.shape[0], 384, dtype=torch.bfloat16, device="cuda")
    gg.forward(Ap, W.cuda(), offs, out)
    torch.cuda.synchronize()
    roffs, _, rA, _ = oracle.route(ids, X, 16)
    ref, _ = oracle.forward(rA, W, roffs)
    assert_close(to_f64(out), ref, "route + forward")
