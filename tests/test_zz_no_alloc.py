"""gg_route_noalloc: token routing for callers that cannot allocate device memory where they
route (a runtime whose device memory is all reserved by its own allocator, or code that must
not enter the CUDA allocator at that point). It takes no workspace: its histograms live in a
fixed array inside the library, shared by every call.

Checked through the C ABI against gg_route (which takes a caller-provided workspace) and
against the oracle's routing: the offsets, packed rows and packed activations must be
identical, on two calls in a row with different inputs (the shared array keeps the first
call's contents), and at the largest size the array admits. This file is collected last so
that a run stopping at its first failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import cuda_ok

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")


def _noalloc_fn():
    L = gg.lib()
    fn = L.gg_route_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_int64, P, P,
                   P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _route_noalloc(ids, X, E):
    T, k = ids.shape
    n = T * k
    A_packed = torch.full((n, X.shape[1]), float("nan"), dtype=torch.bfloat16, device="cuda")
    row_of = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    offs = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _noalloc_fn()(ids.data_ptr(), T, k, E, X.data_ptr(), X.shape[1], A_packed.data_ptr(),
                       row_of.data_ptr(), offs.data_ptr(), st.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0, gg.status_string(rc)
    return A_packed, row_of, offs, st


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    for call, (T, k, E, K) in enumerate([(4096, 8, 64, 512), (777, 3, 37, 136)]):
        ids_np, X = workloads.make_routing(T, k, E, K, seed=100 + call, dropped=11)
        ids, X = torch.from_numpy(ids_np).cuda(), X.cuda()
        ref_A, ref_row, ref_offs = gg.route(ids, X, E)
        A, row_of, offs, st = _route_noalloc(ids, X, E)
        torch.cuda.synchronize()
        assert (int(st.item()) & gg.DEV_ERROR_MASK) == 0
        assert torch.equal(offs, ref_offs)
        assert torch.equal(row_of, ref_row)
        total = int(ref_offs[-1].item())
        # integer and copy work: bit-exact
        assert torch.equal(A[:total].view(torch.int16), ref_A[:total].view(torch.int16))
        _check_against_oracle(ids_np, X, E, A, row_of, offs)


def _check_against_oracle(ids_np, X, E, A, row_of, offs):
    roffs, rrow, rA, _ = oracle.route(ids_np, X.cpu(), E)
    np.testing.assert_array_equal(offs.cpu().numpy(), roffs)
    np.testing.assert_array_equal(row_of.cpu().numpy(), rrow)
    np.testing.assert_array_equal(oracle.as_u16(A[: int(roffs[-1])]), rA)


def test_route_noalloc_rejects_problems_beyond_its_array():
    E, k = 1024, 4
    T = 16385  # ceil(T*k / 256) * E = 257 * 1024 > 2^18 entries
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    X = torch.zeros((T, 8), dtype=torch.bfloat16, device="cuda")
    A = torch.empty((T * k, 8), dtype=torch.bfloat16, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    offs = torch.empty(E, dtype=torch.int32, device="cuda")
    rc = _noalloc_fn()(ids.data_ptr(), T, k, E, X.data_ptr(), 8, A.data_ptr(), row_of.data_ptr(),
                       offs.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert rc == 4 and "TOO_LARGE" in gg.status_string(rc)


def test_route_noalloc_at_the_largest_size_of_its_array():
    """T=16384 tokens x top-4 over 1024 experts fills all GG_ROUTE_NOALLOC_MAX_COUNTS entries
    (256 blocks x 1024 experts): varied expert ids, so that a wrong bound or histogram index at
    the array's end would show in the offsets, the packed rows or the packed activations."""
    T, k, E, K = 16384, 4, 1024, 8
    ids_np, X = workloads.make_routing(T, k, E, K, seed=131, dropped=17)
    ids, X = torch.from_numpy(ids_np).cuda(), X.cuda()
    A, row_of, offs, st = _route_noalloc(ids, X, E)
    ref_A, ref_row, ref_offs = gg.route(ids, X, E)
    torch.cuda.synchronize()
    assert (int(st.item()) & gg.DEV_ERROR_MASK) == 0
    assert torch.equal(offs, ref_offs)
    assert torch.equal(row_of, ref_row)
    total = int(ref_offs[-1].item())
    assert torch.equal(A[:total].view(torch.int16), ref_A[:total].view(torch.int16))
    _check_against_oracle(ids_np, X, E, A, row_of, offs)
