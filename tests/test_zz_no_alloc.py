"""gg_route_noalloc: token routing for callers that cannot allocate device memory where they
route (a runtime whose device memory is all reserved by its own allocator, or code that must
not enter the CUDA allocator at that point). It takes no workspace: its histograms live in a
fixed array inside the library, shared by every call.

Checked through the C ABI against gg_route (which takes a caller-provided workspace): the
offsets, packed rows and packed activations must be identical, on two calls in a row with
different inputs (the shared array keeps the first call's contents). This file is collected
last so that a run stopping at its first failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest
import torch

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
    # the largest allowed size with 1024 experts is accepted
    T = 16384
    rc = _noalloc_fn()(ids.data_ptr(), T, k, E, X.data_ptr(), 8, A.data_ptr(), row_of.data_ptr(),
                       offs.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    assert int(offs[0].item()) == T * k
