"""Robustness of the sm_100a kernels: invalid device data, host-side rejections, guard
regions around outputs, CUDA-graph capture with offsets changed between replays, a
concurrent copy stream, and the in-kernel watchdog (a wait that runs out returns a status;
no GPU fault, trap or hang is involved)."""
import ctypes

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


def _run3(A, W, dY, offs_np, rows, K, N, E):
    offs = torch.from_numpy(np.asarray(offs_np, np.int32)).cuda()
    out, dX, dW = sentinel((rows, N)), sentinel((rows, K)), sentinel((E, K, N))
    st = torch.zeros(3, dtype=torch.int32, device="cuda")
    gg.forward(A.cuda(), W.cuda(), offs, out, status=st[0:1])
    gg.dgrad(dY.cuda(), W.cuda(), offs, dX, status=st[1:2])
    gg.wgrad(A.cuda(), dY.cuda(), offs, dW, status=st[2:3])
    torch.cuda.synchronize()
    return out, dX, dW, st.cpu().numpy()


@pytest.mark.parametrize("offs", [(8, 4, 60, -1), (-5, 20, 300, 310), (100, 90, 80, 400),
                                  (0, 200, 150, 260)])
def test_invalid_offsets_are_clamped_and_flagged(offs, variant):
    """Decreasing, negative and too-large offsets: the kernels use t'_e = clamp(offs[e],
    t'_{e-1}, rows_alloc), compute every resulting group, and set GG_DEV_BAD_OFFSETS."""
    rows, K, N, E = 260, 128, 320, 4
    r = workloads.make_ragged_custom(E, K, N, [65, 65, 65, 65], seed=41, tail=0)
    out, dX, dW, st = _run3(r.A, r.W, r.dY, offs, rows, K, N, E)
    for s in st:
        assert s & gg.DEV_BAD_OFFSETS and s & gg.DEV_LAUNCHED
        assert not s & gg.DEV_TIMEOUT
    ref, grp = oracle.forward(r.A, r.W, offs)
    sel = grp >= 0
    idx = torch.from_numpy(np.nonzero(sel)[0]).cuda()
    assert_close(to_f64(out.index_select(0, idx)), ref[sel], "forward")
    refd, _ = oracle.dgrad(r.dY, r.W, offs)
    assert_close(to_f64(dX.index_select(0, idx)), refd[sel], "dgrad")
    assert_close(to_f64(dW), oracle.wgrad(r.A, r.dY, offs), "wgrad")
    un = torch.from_numpy(np.nonzero(~sel)[0]).cuda()
    assert bool(is_sentinel(out.index_select(0, un)).all())
    assert bool(is_sentinel(dX.index_select(0, un)).all())


def test_invalid_masked_m_is_clamped_and_flagged():
    m = workloads.make_masked(E=4, mmax=64, K=128, N=256, masked_m=[-3, 70, 17, 64], seed=43)
    out = sentinel((4, 64, 256))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.masked_forward(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                      status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_BAD_MASKED_M and s & gg.DEV_LAUNCHED
    ref, act, bad = oracle.masked_forward(m.A, m.W, m.masked_m)
    assert bad
    flat = out.view(-1, 256)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act], "masked")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())


def test_host_rejections_with_device_buffers():
    L = gg.lib()
    dev = "cuda"
    A = torch.zeros(64, 64, dtype=torch.bfloat16, device=dev)
    W = torch.zeros(2, 64, 64, dtype=torch.bfloat16, device=dev)
    out = torch.zeros(64, 64, dtype=torch.bfloat16, device=dev)
    offs = torch.tensor([32, 64], dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    f = L.gg_forward
    assert f(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr(), 64, 64, 64, 2,
             None, stream) == gg.GG_OK
    # misaligned A (2 bytes off) and out
    assert f(A.data_ptr() + 2, W.data_ptr(), offs.data_ptr(), out.data_ptr(), 63, 64, 64, 2,
             None, stream) == gg.GG_ERR_UNSUPPORTED
    assert f(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr() + 8, 63, 64, 64, 2,
             None, stream) == gg.GG_ERR_UNSUPPORTED
    # K or N not a multiple of 8
    assert f(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr(), 64, 60, 64, 2, None,
             stream) == gg.GG_ERR_UNSUPPORTED
    assert f(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr(), 64, 64, 36, 2, None,
             stream) == gg.GG_ERR_UNSUPPORTED
    # null pointers and empty expert lists
    assert f(0, W.data_ptr(), offs.data_ptr(), out.data_ptr(), 64, 64, 64, 2, None,
             stream) == gg.GG_ERR_INVALID_ARG
    assert f(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr(), 64, 64, 64, 0, None,
             stream) == gg.GG_ERR_INVALID_ARG
    assert L.gg_wgrad(A.data_ptr(), A.data_ptr(), offs.data_ptr(), 0, 64, 64, 64, 2, None,
                      stream) == gg.GG_ERR_INVALID_ARG
    with pytest.raises(gg.GGError):
        gg.forward(A[:, :60].contiguous(), W[:, :60].contiguous(), offs,
                   torch.zeros(64, 64, dtype=torch.bfloat16, device=dev))
    # the [gate | up] flag without the SiLU-and-mul epilogue, and a flag the masked call
    # does not take, are rejected before any launch
    with pytest.raises(gg.GGError) as ei:
        gg.forward_ex(A, W, offs, out, gate_up_concat=True)
    assert ei.value.code == gg.GG_ERR_INVALID_ARG
    with pytest.raises(gg.GGError) as ei:
        gg.masked_forward_ex(A.view(2, 32, 64), W, offs, out.view(2, 32, 64),
                             gate_up_concat=True)
    assert ei.value.code == gg.GG_ERR_INVALID_ARG
    epi = gg._Epilogue(None, None, gg.ACT_NONE, gg.FLAG_ZERO_TAIL)
    assert L.gg_masked_forward_ex(A.data_ptr(), W.data_ptr(), offs.data_ptr(), out.data_ptr(),
                                  32, 64, 64, 2, ctypes.byref(epi), None,
                                  stream) == gg.GG_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_guard_regions_around_outputs(variant):
    """Outputs are views into larger sentinel buffers: nothing before or after is written."""
    sizes = [0, 130, 1, 257, 77]
    E, K, N = len(sizes), 192, 264
    r = workloads.make_ragged_custom(E, K, N, sizes, seed=47, tail=33)
    g = 64
    big_out = sentinel((r.rows_alloc + 2 * g, N))
    big_dx = sentinel((r.rows_alloc + 2 * g, K))
    big_dw = sentinel((E + 2, K, N))
    out, dX, dW = big_out[g:g + r.rows_alloc], big_dx[g:g + r.rows_alloc], big_dw[1:1 + E]
    offs = torch.from_numpy(r.offs).cuda()
    A, W, dY = r.A.cuda(), r.W.cuda(), r.dY.cuda()
    gg.forward(A, W, offs, out)
    gg.dgrad(dY, W, offs, dX)
    gg.wgrad(A, dY, offs, dW)
    torch.cuda.synchronize()
    for big, inner_rows in ((big_out, r.rows_alloc), (big_dx, r.rows_alloc)):
        assert bool(is_sentinel(big[:g]).all()) and bool(is_sentinel(big[g + inner_rows:]).all())
    assert bool(is_sentinel(big_dw[0]).all()) and bool(is_sentinel(big_dw[-1]).all())
    T = r.T
    ref, _ = oracle.forward(r.A, r.W, r.offs)
    assert_close(to_f64(out[:T]), ref[:T], "forward")
    assert bool(is_sentinel(out[T:]).all())


def test_zero_rows_and_all_empty_groups():
    E, K, N = 3, 64, 128
    A = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    W = torch.randn(E, K, N, device="cuda").to(torch.bfloat16)
    offs = torch.zeros(E, dtype=torch.int32, device="cuda")
    out = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    dW = sentinel((E, K, N))
    gg.forward(A, W, offs, out)
    gg.wgrad(A, dY, offs, dW)
    torch.cuda.synchronize()
    assert bool((dW.view(torch.int16) == 0).all())
    # rows present but every group empty
    r = workloads.make_ragged_custom(E, K, N, [0, 0, 0], seed=3, tail=40)
    out, dX, dW, st = _run3(r.A, r.W, r.dY, [0, 0, 0], r.rows_alloc, K, N, E)
    assert bool(is_sentinel(out).all()) and bool(is_sentinel(dX).all())
    assert bool((dW.view(torch.int16) == 0).all())
    assert all((s & gg.DEV_ERROR_MASK) == 0 for s in st)


def test_many_experts(variant):
    """E spans several 32-wide scan chunks of the device schedule, most groups tiny."""
    rng = np.random.default_rng(5)
    E = 300
    sizes = rng.integers(0, 20, E)
    sizes[rng.choice(E, 60, replace=False)] = 0
    sizes[7] = 300
    r = workloads.make_ragged_custom(E, 64, 128, sizes, seed=51, tail=10)
    out, dX, dW, st = _run3(r.A, r.W, r.dY, r.offs, r.rows_alloc, 64, 128, E)
    assert all((s & gg.DEV_ERROR_MASK) == 0 for s in st)
    T = r.T
    ref, _ = oracle.forward(r.A, r.W, r.offs)
    assert_close(to_f64(out[:T]), ref[:T], "forward")
    refd, _ = oracle.dgrad(r.dY, r.W, r.offs)
    assert_close(to_f64(dX[:T]), refd[:T], "dgrad")
    assert_close(to_f64(dW), oracle.wgrad(r.A, r.dY, r.offs), "wgrad")


def test_cuda_graph_replay_with_offsets_changed_in_place(variant):
    """Capture forward+dgrad+wgrad once; change the device offsets between replays."""
    E, K, N, rows = 5, 128, 256, 700
    r = workloads.make_ragged_custom(E, K, N, [100, 0, 250, 50, 300], seed=53, tail=0)
    A, W, dY = r.A.cuda(), r.W.cuda(), r.dY.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    out, dX, dW = sentinel((rows, N)), sentinel((rows, K)), sentinel((E, K, N))
    st = torch.zeros(3, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (sets kernel attributes)
        gg.forward(A, W, offs, out, status=st[0:1])
        gg.dgrad(dY, W, offs, dX, status=st[1:2])
        gg.wgrad(A, dY, offs, dW, status=st[2:3])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gg.forward(A, W, offs, out, status=st[0:1])
        gg.dgrad(dY, W, offs, dX, status=st[1:2])
        gg.wgrad(A, dY, offs, dW, status=st[2:3])
    for new in ([100, 100, 350, 400, 700], [0, 0, 0, 10, 512], [700, 700, 700, 700, 700]):
        offs.copy_(torch.tensor(new, dtype=torch.int32))
        out.view(torch.int16).fill_(workloads.BF16_SENTINEL - (1 << 16))
        dX.view(torch.int16).fill_(workloads.BF16_SENTINEL - (1 << 16))
        st.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert all((int(x) & gg.DEV_ERROR_MASK) == 0 for x in st.cpu())
        ref, grp = oracle.forward(r.A, r.W, new)
        T = new[-1]
        assert_close(to_f64(out[:T]), ref[:T], f"graph forward {new}")
        assert bool(is_sentinel(out[T:]).all())
        refd, _ = oracle.dgrad(r.dY, r.W, new)
        assert_close(to_f64(dX[:T]), refd[:T], f"graph dgrad {new}")
        assert_close(to_f64(dW), oracle.wgrad(r.A, r.dY, new), f"graph wgrad {new}")
    del graph


def test_results_while_a_side_stream_copies(variant):
    """A concurrent stream streams large device copies while the grouped GEMM runs (the
    stale-output hazard of TransformerEngine PR 3542): every valid element is overwritten
    and no unused row is."""
    r = workloads.make_ragged_custom(6, 512, 1024, [900, 0, 1300, 17, 2000, 640], seed=55,
                                     tail=100)
    A, W, dY = r.A.cuda(), r.W.cuda(), r.dY.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    src = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    side = torch.cuda.Stream()
    for _ in range(3):
        out, dW = sentinel((r.rows_alloc, r.N)), sentinel((r.E, r.K, r.N))
        torch.cuda.synchronize()
        with torch.cuda.stream(side):
            for _ in range(8):
                dst.copy_(src, non_blocking=True)
        gg.forward(A, W, offs, out)
        gg.wgrad(A, dY, offs, dW)
        torch.cuda.synchronize()
        T = r.T
        ref, _ = oracle.forward(r.A, r.W, r.offs)
        assert_close(to_f64(out[:T]), ref[:T], "forward under concurrent copies")
        assert bool(is_sentinel(out[T:]).all())
        assert not bool(is_sentinel(dW).any())


@pytest.mark.parametrize("op", ["forward", "dgrad", "wgrad", "masked"])
def test_watchdog_reports_timeout_and_context_stays_usable(op, variant):
    """CTA 0's first stage is never loaded (test hook), so its consumer's wait runs out:
    the call ends with GG_DEV_TIMEOUT after about the watchdog bound; the next call works."""
    r = workloads.make_ragged_custom(3, 128, 256, [300, 5, 600], seed=57, tail=0)
    A, W, dY = r.A.cuda(), r.W.cuda(), r.dY.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    m = workloads.make_masked(E=2, mmax=128, K=128, N=256, masked_m=[100, 128], seed=59)
    mA, mW, mm = m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda()

    def call(status):
        if op == "forward":
            return gg.forward(A, W, offs, sentinel((r.rows_alloc, r.N)), status=status)
        if op == "dgrad":
            return gg.dgrad(dY, W, offs, sentinel((r.rows_alloc, r.K)), status=status)
        if op == "wgrad":
            return gg.wgrad(A, dY, offs, sentinel((r.E, r.K, r.N)), status=status)
        return gg.masked_forward(mA, mW, mm, sentinel((2, 128, 256)), status=status)

    prev_wd = gg.set_watchdog_ns(200_000_000)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        gg.testing_skip_first_load(True)
        call(st)
        torch.cuda.synchronize()
    finally:
        gg.testing_skip_first_load(False)
        gg.set_watchdog_ns(prev_wd)
    s = int(st.item())
    assert s & gg.DEV_TIMEOUT, hex(s)
    # the context is intact: a normal call right after is correct
    st.zero_()
    res = call(st)
    torch.cuda.synchronize()
    assert (int(st.item()) & gg.DEV_ERROR_MASK) == 0
    if op == "forward":
        ref, _ = oracle.forward(r.A, r.W, r.offs)
        assert_close(to_f64(res[:r.T]), ref[:r.T], "forward after timeout")
