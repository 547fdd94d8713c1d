"""W stored [E, N, K], zero-tail outputs and the autograd wrapper, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import cuda_ok
from helpers import assert_close, is_sentinel, sentinel, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")


@pytest.fixture(params=[1, 2, 3], ids=["single_cta", "cta_pair", "cta_pair_wide"])
def variant(request):
    prev = gg.testing_force_variant(request.param)
    yield request.param
    gg.testing_force_variant(prev)


SIZES = [0, 1, 127, 128, 129, 300, 17]


def _case(K=192, N=320, tail=40, seed=91):
    r = workloads.make_ragged_custom(len(SIZES), K, N, SIZES, seed=seed, tail=tail)
    Wt = r.W.transpose(1, 2).contiguous()  # [E, N, K]
    return r, Wt


def test_w_nk_forward_dgrad_wgrad(variant):
    r, Wt = _case()
    A, dY, offs = r.A.cuda(), r.dY.cuda(), torch.from_numpy(r.offs).cuda()
    out = sentinel((r.rows_alloc, r.N))
    dX = sentinel((r.rows_alloc, r.K))
    dWt = sentinel((r.E, r.N, r.K))
    gg.forward_ex(A, Wt.cuda(), offs, out, w_nk=True)
    gg.dgrad_ex(dY, Wt.cuda(), offs, dX, w_nk=True)
    gg.wgrad_ex(A, dY, offs, dWt, w_nk=True)
    torch.cuda.synchronize()
    T = r.T
    ref, _ = oracle.forward(r.A, r.W, r.offs)
    assert_close(to_f64(out[:T]), ref[:T], "forward W[E,N,K]")
    refd, _ = oracle.dgrad(r.dY, r.W, r.offs)
    assert_close(to_f64(dX[:T]), refd[:T], "dgrad W[E,N,K]")
    refw = oracle.wgrad(r.A, r.dY, r.offs)
    assert_close(to_f64(dWt), refw.transpose(0, 2, 1), "wgrad dW[E,N,K]")
    assert bool(is_sentinel(out[T:]).all()) and bool(is_sentinel(dX[T:]).all())


@pytest.mark.parametrize("w_nk", [False, True])
def test_zero_tail(w_nk, variant):
    r, Wt = _case(K=256, N=512)
    W = Wt if w_nk else r.W
    A, dY, offs = r.A.cuda(), r.dY.cuda(), torch.from_numpy(r.offs).cuda()
    out = sentinel((r.rows_alloc, r.N))
    half = sentinel((r.rows_alloc, r.N // 2))
    dX = sentinel((r.rows_alloc, r.K))
    gg.forward_ex(A, W.cuda(), offs, out, zero_tail=True, w_nk=w_nk)
    gg.forward_ex(A, W.cuda(), offs, half, act=gg.ACT_SILU_MUL, zero_tail=True, w_nk=w_nk)
    gg.dgrad_ex(dY, W.cuda(), offs, dX, zero_tail=True, w_nk=w_nk)
    torch.cuda.synchronize()
    T = r.T
    for t in (out, half, dX):
        assert bool((t[T:].view(torch.int16) == 0).all())  # +0.0 in the tail
    ref, _ = oracle.forward(r.A, r.W, r.offs)
    assert_close(to_f64(out[:T]), ref[:T], "forward zero tail")
    refh, _ = oracle.forward_ex(r.A, r.W, r.offs, act=1)
    assert_close(to_f64(half[:T]), refh[:T], "silu zero tail")
    refd, _ = oracle.dgrad(r.dY, r.W, r.offs)
    assert_close(to_f64(dX[:T]), refd[:T], "dgrad zero tail")


@pytest.mark.parametrize("w_nk", [False, True])
def test_autograd_grouped_mm(w_nk, variant):
    """torch._grouped_mm-style call with backward: out, dA (zero past the last offset) and
    dW against the oracle; the empty-expert backward of PyTorch issue 152668 completes."""
    r, Wt = _case(K=128, N=256, seed=93)
    A = r.A.clone()
    A[r.T:] = 0  # the unused rows hold finite values here: they must still get dA = 0
    A = A.cuda().requires_grad_(True)
    W = (Wt if w_nk else r.W).cuda().requires_grad_(True)
    offs = torch.from_numpy(r.offs).cuda()
    out = gg.grouped_mm(A, W, offs, w_nk=w_nk)
    dY = r.dY.clone()
    dY[r.T:] = 0
    out.backward(dY.cuda())
    torch.cuda.synchronize()
    T = r.T
    ref, _ = oracle.forward(r.A, r.W, r.offs)
    assert_close(to_f64(out.detach()[:T]), ref[:T], "autograd forward")
    assert bool((out.detach()[T:].float() == 0).all())
    refd, _ = oracle.dgrad(dY, r.W, r.offs)
    assert_close(to_f64(A.grad[:T]), refd[:T], "autograd dA")
    assert bool((A.grad[T:].float() == 0).all())
    refw = oracle.wgrad(r.A, dY, r.offs)
    got = to_f64(W.grad)
    assert_close(got.transpose(0, 2, 1) if w_nk else got, refw, "autograd dW")


def test_autograd_tiny_repro_with_empty_expert():
    """The repro of PyTorch issue 152668: forward and backward with offsets (8, 8, 32, 40)."""
    t = workloads.make_tiny((8, 8, 32, 40), nan_tail=False)
    x = t.A.cuda().requires_grad_(True)
    w = t.W.cuda().requires_grad_(True)
    offs = torch.tensor([8, 8, 32, 40], dtype=torch.int32, device="cuda")
    o = gg.grouped_mm(x, w, offs)
    o.backward(torch.ones_like(o))
    torch.cuda.synchronize()
    assert o.shape == (48, 16) and x.grad.shape == (48, 8) and w.grad.shape == (4, 8, 16)
    assert bool((w.grad[1] == 0).all())
