"""gg_layer_step_host: forward, dgrad and wgrad on host tensors, streamed through the GPU by
chunks of consecutive experts with the copies overlapped with the GEMMs. The host results are
checked against the oracle on the same inputs (full on small cases, sampled rows and K rows on
the gate-up shape); host output rows past the last offset keep their sentinel."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import cuda_ok
from helpers import assert_close, is_sentinel, sample_k, sample_rows, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")


def run_host(r: workloads.RaggedInputs, chunks: int):
    rows, K, N, E = r.rows_alloc, r.K, r.N, r.E
    hA, hW, hdY = (t.cpu().pin_memory() for t in (r.A, r.W, r.dY))
    hoffs = torch.from_numpy(np.ascontiguousarray(r.offs, dtype=np.int32)).pin_memory()
    hout = workloads.sentinel_like((rows, N)).pin_memory()
    hdX = workloads.sentinel_like((rows, K)).pin_memory()
    hdW = workloads.sentinel_like((E, K, N)).pin_memory()
    staging = {"A": torch.empty_like(hA, device="cuda"), "W": torch.empty_like(hW, device="cuda"),
               "dY": torch.empty_like(hdY, device="cuda"),
               "offs": torch.empty(E, dtype=torch.int32, device="cuda"),
               "out": torch.empty((rows, N), dtype=torch.bfloat16, device="cuda"),
               "dX": torch.empty((rows, K), dtype=torch.bfloat16, device="cuda"),
               "dW": torch.empty((E, K, N), dtype=torch.bfloat16, device="cuda")}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.layer_step_host(hA, hW, hdY, hoffs, hout, hdX, hdW, staging, chunks=chunks, status=st)
    torch.cuda.current_stream().synchronize()
    return hout, hdX, hdW, int(st.item())


def check_host(r: workloads.RaggedInputs, chunks: int, sample: bool, seed: int = 0):
    out, dX, dW, st = run_host(r, chunks)
    assert st & gg.DEV_LAUNCHED, "the sm_100a kernels did not report completion"
    assert (st & gg.DEV_ERROR_MASK) == 0, hex(st)
    A, W, dY = oracle.as_u16(r.A), oracle.as_u16(r.W), oracle.as_u16(r.dY)
    rows = sample_rows(r.offs, r.rows_alloc, seed) if sample else None
    ref, grp = oracle.forward(A, W, r.offs, rows=rows)
    sel = grp >= 0
    ridx = torch.from_numpy((np.arange(r.rows_alloc) if rows is None else rows)[sel])
    assert_close(to_f64(out.index_select(0, ridx)), ref[sel], "forward")
    refd, _ = oracle.dgrad(dY, W, r.offs, rows=rows)
    assert_close(to_f64(dX.index_select(0, ridx)), refd[sel], "dgrad")
    untouched = torch.from_numpy(oracle.untouched_rows(r.offs, r.rows_alloc))
    assert bool(is_sentinel(out.index_select(0, untouched)).all())
    assert bool(is_sentinel(dX.index_select(0, untouched)).all())
    ks = sample_k(r.K, seed) if sample else None
    refw = oracle.wgrad(A, dY, r.offs, ks=ks)
    kidx = torch.from_numpy(np.arange(r.K) if ks is None else ks)
    assert_close(to_f64(dW.index_select(1, kidx)), refw, "wgrad")
    assert not bool(is_sentinel(dW).any())
    starts, ends, _ = oracle.group_bounds(r.offs, r.rows_alloc)
    for e in np.nonzero(ends == starts)[0]:
        assert bool((dW[e].view(torch.int16) == 0).all()), f"dW[{e}] of an empty expert"


@pytest.mark.parametrize("offs", [(8, 16, 32, 40), (8, 8, 32, 40), (0, 0, 0, 0),
                                  (48, 48, 48, 48)])
@pytest.mark.parametrize("chunks", [0, 1, 2, 4])
def test_host_step_tiny_repro(offs, chunks):
    check_host(workloads.make_tiny(offs), chunks, sample=False)


@pytest.mark.parametrize("chunks", [0, 3, 32])
def test_host_step_size_sweep(chunks):
    sizes = [0, 1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 255, 256, 257]
    r = workloads.make_ragged_custom(len(sizes), 200, 328, sizes, seed=300, tail=128)
    check_host(r, chunks, sample=False)


@pytest.mark.parametrize("chunks", [0, 5])
def test_host_step_gateup_shape(chunks):
    """E=64 Zipf-skewed gate-up shape (K=2048, N=1536) with empty experts, sampled."""
    r = workloads.make_ragged("gateup", tail=128, device="cpu")
    check_host(r, chunks, sample=True, seed=4)


def test_host_step_rejects_bad_offsets_before_enqueueing():
    r = workloads.make_tiny((8, 16, 32, 40))
    r.offs = np.array([8, 4, 32, 40], dtype=np.int32)
    with pytest.raises(gg.GGError):
        run_host(r, 0)
