"""Back-to-back calls in one stream, each reading what the call before it wrote.

The grouped GEMM kernels are launched with programmatic dependent launch: a kernel may be
scheduled while the previous kernel of its stream is still running, and it waits for that
kernel to complete before its first global read or write. Here the inputs of every call are
the outputs of the call before it (activations, gradients, and offsets rewritten by a torch
kernel in between), with no host synchronisation. The kernels are deterministic, so the
results must be bit-identical to the same calls separated by device synchronisations, and to
the same calls replayed from a CUDA graph. Output rows that no group covers keep their
sentinel in every run.
"""
import numpy as np
import pytest
import torch

import workloads
from conftest import cuda_ok

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")

D = 512                                   # K = N, so that outputs feed the next call
SIZES = [700, 0, 1300, 333, 64, 900]      # ragged, one empty expert
SIZES_ALT = [1000, 297, 0, 1200, 400, 400]
TAIL = 16
MMAX = 128


def _inputs():
    r = workloads.make_ragged_custom(len(SIZES), D, D, SIZES, seed=31, tail=TAIL,
                                     nan_tail=False, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(32)
    W2 = (torch.randn((len(SIZES), D, D), generator=gen, device="cuda") / np.sqrt(D)).to(
        torch.bfloat16)
    offs = torch.from_numpy(np.asarray(r.offs, dtype=np.int32)).cuda()
    offs_alt = torch.from_numpy(workloads.offsets_from_sizes(np.asarray(SIZES_ALT))).to(
        torch.int32).cuda()
    masked_m = torch.tensor([128, 5, 0, 77, 64, 128], dtype=torch.int32, device="cuda")
    return r, W2, offs, offs_alt, masked_m


def _buffers(rows, E):
    s = workloads.sentinel_like
    return {"y1": s((rows, D)).cuda(), "y2": s((rows, D)).cuda(), "g": s((rows, D)).cuda(),
            "dW": s((E, D, D)).cuda(), "offs2": torch.zeros(E, dtype=torch.int32, device="cuda"),
            "y3": s((rows, D)).cuda(), "y4": s((rows, D)).cuda(),
            "mout": s((E, MMAX, D)).cuda()}


def _chain(r, W2, offs, offs_alt, masked_m, b, sync: bool):
    E = r.E
    step = (lambda: torch.cuda.synchronize()) if sync else (lambda: None)
    gg.forward(r.A, r.W, offs, b["y1"]); step()
    gg.forward(b["y1"], W2, offs, b["y2"]); step()          # reads y1
    gg.dgrad(b["y2"], W2, offs, b["g"]); step()             # reads y2
    gg.wgrad(b["y1"], b["g"], offs, b["dW"]); step()        # reads g, written just before
    gg.forward(b["g"], b["dW"], offs, b["y4"]); step()      # reads dW (all of a split wgrad)
    b["offs2"].copy_(offs_alt); step()                      # offsets from a torch kernel
    gg.forward(b["g"], r.W, b["offs2"], b["y3"]); step()    # reads g and the new offsets
    mA = b["y3"][:E * MMAX].view(E, MMAX, D)
    gg.masked_forward(mA, W2, masked_m, b["mout"]); step()  # reads y3


def _same(x: torch.Tensor, y: torch.Tensor) -> bool:
    if x.dtype == torch.bfloat16:
        return torch.equal(x.view(torch.int16), y.view(torch.int16))  # NaN-safe, bitwise
    return torch.equal(x, y)


@pytest.mark.parametrize("variant", [0, 1, 2, 3], ids=["auto", "single_cta", "cta_pair",
                                                      "cta_pair_wide"])
def test_chained_calls_match_serialised_and_graph_replay(variant):
    gg.testing_force_variant(variant)
    try:
        r, W2, offs, offs_alt, masked_m = _inputs()
        rows, E = r.rows_alloc, r.E
        serial = _buffers(rows, E)
        _chain(r, W2, offs, offs_alt, masked_m, serial, sync=True)
        torch.cuda.synchronize()
        for rep in range(3):
            b = _buffers(rows, E)
            _chain(r, W2, offs, offs_alt, masked_m, b, sync=False)
            torch.cuda.synchronize()
            for k in serial:
                assert _same(b[k], serial[k]), (rep, k)
        g = _buffers(rows, E)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            _chain(r, W2, offs, offs_alt, masked_m, g, sync=False)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        for k in serial:
            assert _same(g[k], serial[k]), ("graph", k)
        del graph
        # the chain did real work: the rows of the groups hold finite products and the rows
        # past the last offset keep their sentinel
        T = int(sum(SIZES))
        assert bool(torch.isfinite(serial["y2"][:T].float()).all())
        assert _same(serial["y2"][T:], workloads.sentinel_like((TAIL, D)).cuda())
    finally:
        gg.testing_force_variant(0)
