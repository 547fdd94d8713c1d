"""Parity of the sm_100a kernels (through the C ABI) with the CPU oracle.

Every comparison is elementwise against the fp64 oracle on the same seeded inputs with
|gpu - ref| <= 1e-2*|ref| + 1e-2; group membership and untouched regions are bit-exact
(sentinel bit patterns), and so are the exact zeros of an empty expert's wgrad.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import cuda_ok
from helpers import assert_close, is_sentinel, sample_k, sample_rows, sentinel, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA device")]

gg = pytest.importorskip("moe_grouped_gemm_ragged_b200")


@pytest.fixture(params=[1, 2, 3], ids=["single_cta", "cta_pair", "cta_pair_wide"])
def variant(request):
    """Every pass with 128-row single-CTA tiles, 256-row CTA-pair tiles, and CTA pairs
    with 256 x 512 tiles (the automatic wgrad shape)."""
    prev = gg.testing_force_variant(request.param)
    yield request.param
    gg.testing_force_variant(prev)


def _dev(r: workloads.RaggedInputs):
    return (r.A.cuda(), r.W.cuda(), r.dY.cuda(),
            torch.from_numpy(np.ascontiguousarray(r.offs)).cuda())


def run_ragged(r: workloads.RaggedInputs):
    """All three passes on the GPU into sentinel-filled buffers; returns device tensors."""
    A, W, dY, offs = _dev(r) if r.A.device.type == "cpu" else (
        r.A, r.W, r.dY, torch.from_numpy(np.ascontiguousarray(r.offs)).cuda())
    rows, K, N, E = r.rows_alloc, r.K, r.N, r.E
    out = sentinel((rows, N))
    dX = sentinel((rows, K))
    dW = sentinel((E, K, N))
    st = torch.zeros(3, dtype=torch.int32, device="cuda")
    gg.forward(A, W, offs, out, status=st[0:1])
    gg.dgrad(dY, W, offs, dX, status=st[1:2])
    gg.wgrad(A, dY, offs, dW, status=st[2:3])
    torch.cuda.synchronize()
    return out, dX, dW, st.cpu().numpy()


def check_ragged(r: workloads.RaggedInputs, sample: bool, seed: int = 0,
                 expect_status: int = 0):
    out, dX, dW, st = run_ragged(r)
    for s in st:
        assert s & gg.DEV_LAUNCHED, "the sm_100a kernel did not report completion"
        assert (s & gg.DEV_ERROR_MASK) == expect_status, hex(s)
    A, W, dY = oracle.as_u16(r.A), oracle.as_u16(r.W), oracle.as_u16(r.dY)  # host copies
    rows = sample_rows(r.offs, r.rows_alloc, seed) if sample else None
    ref, grp = oracle.forward(A, W, r.offs, rows=rows)
    sel = grp >= 0
    ridx = np.arange(r.rows_alloc) if rows is None else rows
    ridx_t = torch.from_numpy(ridx[sel]).cuda()
    assert_close(to_f64(out.index_select(0, ridx_t)), ref[sel], "forward")
    refd, _ = oracle.dgrad(dY, W, r.offs, rows=rows)
    assert_close(to_f64(dX.index_select(0, ridx_t)), refd[sel], "dgrad")
    # rows outside every group: untouched, bit for bit
    untouched = torch.from_numpy(oracle.untouched_rows(r.offs, r.rows_alloc)).cuda()
    assert bool(is_sentinel(out.index_select(0, untouched)).all())
    assert bool(is_sentinel(dX.index_select(0, untouched)).all())
    ks = sample_k(r.K, seed) if sample else None
    refw = oracle.wgrad(A, dY, r.offs, ks=ks)
    kidx = torch.from_numpy(np.arange(r.K) if ks is None else ks).cuda()
    assert_close(to_f64(dW.index_select(1, kidx)), refw, "wgrad")
    # every dW element written; an empty expert's dW is exactly +0.0
    assert not bool(is_sentinel(dW).any())
    starts, ends, _ = oracle.group_bounds(r.offs, r.rows_alloc)
    for e in np.nonzero(ends == starts)[0]:
        assert bool((dW[e].view(torch.int16) == 0).all()), f"dW[{e}] of an empty expert"
    return out, dX, dW


@pytest.mark.parametrize("offs", [(8, 16, 32, 40), (8, 8, 32, 40), (0, 16, 32, 40),
                                  (8, 16, 32, 32), (0, 0, 0, 0), (40, 40, 40, 40),
                                  (48, 48, 48, 48), (0, 0, 0, 48)])
def test_tiny_repro_offsets(offs, variant):
    """The 4-expert M=48/K=8/N=16 repro with its two offset tuples and edge variants."""
    r = workloads.make_tiny(offs)
    out, dX, dW = check_ragged(r, sample=False)
    assert tuple(out.shape) == (48, 16) and tuple(dX.shape) == (48, 8)
    assert tuple(dW.shape) == (4, 8, 16)


SWEEP = [0, 1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 255, 256, 257]


@pytest.mark.parametrize("K,N", [(200, 328), (64, 256), (8, 16), (136, 520)])
def test_group_size_sweep(K, N, variant):
    """Group sizes around 0, 8, 16, 128 and 256 rows, K and N tails, NaN tail rows."""
    r = workloads.make_ragged_custom(len(SWEEP), K, N, SWEEP, seed=100 + K, tail=128)
    check_ragged(r, sample=False)


def test_shuffled_sizes_many_experts(variant):
    rng = np.random.default_rng(7)
    sizes = rng.permutation(np.array(SWEEP * 3))
    r = workloads.make_ragged_custom(len(sizes), 256, 384, sizes, seed=8, tail=200)
    check_ragged(r, sample=False)


def test_maximum_expert_count(variant):
    """GG_MAX_EXPERTS = 1024 experts (the largest group tables in shared memory), sizes 0-40
    rows with a fifth of the experts empty, sampled rows and K rows."""
    rng = np.random.default_rng(11)
    sizes = rng.integers(0, 41, 1024)
    sizes[rng.choice(1024, 205, replace=False)] = 0
    r = workloads.make_ragged_custom(1024, 128, 192, sizes, seed=12, tail=64)
    assert r.E == gg.MAX_EXPERTS
    check_ragged(r, sample=True, seed=5)


def test_group_id_probe_bit_exact(variant):
    """A[:,0]=1, W[e][0,:]=e+1: every output row equals its group id + 1 exactly."""
    sizes = [3, 0, 130, 1, 257, 0, 64]
    E, K, N = len(sizes), 64, 264
    offs = workloads.offsets_from_sizes(sizes)
    rows = int(offs[-1]) + 16
    A = torch.zeros(rows, K, dtype=torch.bfloat16)
    A[:, 0] = 1
    W = torch.zeros(E, K, N, dtype=torch.bfloat16)
    for e in range(E):
        W[e, 0] = e + 1
    out = sentinel((rows, N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.forward(A.cuda(), W.cuda(), torch.from_numpy(offs).cuda(), out, status=st)
    torch.cuda.synchronize()
    grp = np.concatenate([np.full(s, e) for e, s in enumerate(sizes)])
    expect = torch.from_numpy(grp + 1).float().cuda()[:, None].expand(-1, N)
    assert bool((out[: int(offs[-1])].float() == expect).all())
    assert bool(is_sentinel(out[int(offs[-1]):]).all())


# sizes around the 16-row MMA step, the 64-row wgrad stage and the 128/256-row tiles, an
# empty expert between live ones and at the end
PROBE_SIZES = [3, 0, 130, 1, 257, 16, 63, 64, 65, 15, 17, 300, 0]


def _probe_dy(sizes, N, tail):
    """dY[r, :] = e(r) + 1 for every row of group e (small integers, exact in bf16), NaN in the
    rows past the last offset; returns (dY, offs, rows)."""
    offs = workloads.offsets_from_sizes(sizes)
    rows = int(offs[-1]) + tail
    grp = np.concatenate([np.full(sz, e, np.float32) for e, sz in enumerate(sizes)])
    dY = torch.full((rows, N), float("nan"), dtype=torch.float32)
    dY[: int(offs[-1])] = torch.from_numpy(grp + 1)[:, None]
    return dY.to(torch.bfloat16), offs, rows


def test_wgrad_group_id_probe_bit_exact(variant):
    """A[:,0]=1 (other columns 0), dY rows of group e all equal to e+1: dW[e][0, n] is the
    integer m_e (e+1), summed exactly in fp32 and rounded once to bf16, and every other dW
    element is 0; a row counted in the wrong group, a row of the NaN tail read into a sum or
    a lost tail row of a 64-row stage changes the bits."""
    sizes = PROBE_SIZES
    E, K, N = len(sizes), 136, 264
    dY, offs, rows = _probe_dy(sizes, N, tail=40)
    A = torch.zeros(rows, K, dtype=torch.bfloat16)
    A[:, 0] = 1
    A[int(offs[-1]):] = float("nan")
    dW = sentinel((E, K, N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.wgrad(A.cuda(), dY.cuda(), torch.from_numpy(offs).cuda(), dW, status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    expect = torch.zeros(E, K, N, dtype=torch.float32)
    for e, m in enumerate(sizes):
        expect[e, 0, :] = float(m * (e + 1))
    expect = expect.to(torch.bfloat16).cuda()   # one rounding of the exact integer
    assert torch.equal(dW.view(torch.int16), expect.view(torch.int16))


def test_dgrad_group_id_probe_bit_exact(variant):
    """dY[:,0]=1 (other columns 0), W[e][:, 0]=e+1: dX[r, k] = e(r)+1 exactly for every row of
    every group; the rows past the last offset keep their sentinel."""
    sizes = PROBE_SIZES
    E, K, N = len(sizes), 264, 72
    offs = workloads.offsets_from_sizes(sizes)
    rows = int(offs[-1]) + 24
    dY = torch.zeros(rows, N, dtype=torch.bfloat16)
    dY[:, 0] = 1
    W = torch.zeros(E, K, N, dtype=torch.bfloat16)
    for e in range(E):
        W[e, :, 0] = e + 1
    dX = sentinel((rows, K))
    gg.dgrad(dY.cuda(), W.cuda(), torch.from_numpy(offs).cuda(), dX)
    torch.cuda.synchronize()
    grp = np.concatenate([np.full(sz, e) for e, sz in enumerate(sizes)])
    expect = torch.from_numpy(grp + 1).float().cuda()[:, None].expand(-1, K)
    assert bool((dX[: int(offs[-1])].float() == expect).all())
    assert bool(is_sentinel(dX[int(offs[-1]):]).all())


@pytest.mark.slow
@pytest.mark.parametrize("name", ["large", "large_unaligned"])
def test_large_group_id_probes_bit_exact(name):
    """Group-id probes at the full size of the large shape (E=16, 262144 rows, K=6144,
    N=4096), where the tolerance alone would not see one misassigned row: with A[:,0]=1 (other
    columns 0) and W[e][0,:]=e+1, every element of out is e(r)+1; with dY rows of group e all
    e+1, dW[e][0,n] is m_e (e+1), an exact fp32 sum rounded once to bf16, and every other dW
    element is 0. Compared in full on the GPU; the automatic launch shapes."""
    sizes = workloads.group_sizes(name)
    E, K, N = len(sizes), 6144, 4096
    offs = workloads.offsets_from_sizes(sizes)
    T = int(offs[-1])
    offs_d = torch.from_numpy(offs).cuda()
    grp = torch.repeat_interleave(torch.arange(E, device="cuda"),
                                  torch.from_numpy(np.asarray(sizes)).cuda())
    A = torch.zeros(T, K, dtype=torch.bfloat16, device="cuda")
    A[:, 0] = 1
    W = torch.zeros(E, K, N, dtype=torch.bfloat16, device="cuda")
    W[:, 0, :] = (torch.arange(E, device="cuda", dtype=torch.float32) + 1)[:, None].to(
        torch.bfloat16)
    out = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    gg.forward(A, W, offs_d, out, status=st[0:1])
    del W
    expect_row = (grp + 1).to(torch.bfloat16)
    assert bool((out == expect_row[:, None]).all()), "forward: a row left its group"
    del out
    dY = expect_row[:, None].expand(T, N).contiguous()
    dW = torch.empty(E, K, N, dtype=torch.bfloat16, device="cuda")
    gg.wgrad(A, dY, offs_d, dW, status=st[1:2])
    torch.cuda.synchronize()
    s = st.cpu().numpy()
    assert np.all(s & gg.DEV_LAUNCHED) and not np.any(s & gg.DEV_ERROR_MASK), s
    want = torch.tensor([float(m * (e + 1)) for e, m in enumerate(sizes)],
                        dtype=torch.float32).to(torch.bfloat16).cuda()
    assert bool((dW[:, 0, :] == want[:, None]).all()), "wgrad: probe row"
    assert bool((dW[:, 1:, :] == 0).all()), "wgrad: zero rows"


@pytest.mark.slow
def test_gateup_config_full_elementwise():
    """The E=64 Zipf gate-up config (K=2048, N=1536, 4 empty experts, unaligned sizes) in full:
    every element of out, dX (all rows of every group) and dW against the oracle, with NaN
    tail rows; the automatic launch shapes."""
    r = workloads.make_ragged("gateup", tail=128, device="cuda")
    check_ragged(r, sample=False)


def test_masked_config_full():
    """Masked layout E=8, mmax=128, K=768, N=2048; NaN in inactive rows."""
    m = workloads.make_masked()
    A, W = m.A.cuda(), m.W.cuda()
    mm = torch.from_numpy(m.masked_m).cuda()
    out = sentinel((m.E, m.mmax, m.N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.masked_forward(A, W, mm, out, status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, act, _ = oracle.masked_forward(m.A, m.W, m.masked_m)
    flat = out.view(-1, m.N)
    act_t = torch.from_numpy(np.nonzero(act)[0]).cuda()
    inact_t = torch.from_numpy(np.nonzero(~act)[0]).cuda()
    assert_close(to_f64(flat.index_select(0, act_t)), ref[act], "masked forward")
    assert bool(is_sentinel(flat.index_select(0, inact_t)).all())


@pytest.mark.parametrize("name", ["gateup", "downproj"])
def test_moe_projection_configs(name, variant):
    """E=64 Zipf gate-up (K=2048, N=1536) and E=32 down-proj (K=2048, N=7168): sampled rows
    {s, s+1, t-2, t-1} + 60 random per group and 32 K rows per expert, NaN tail rows."""
    r = workloads.make_ragged(name, tail=128, device="cuda")
    check_ragged(r, sample=True, seed=1)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["large", "large_unaligned"])
def test_large_configs(name, variant):
    """262144 x 6144 x 4096, E=16, aligned and +-1..127 perturbed sizes (sampled)."""
    r = workloads.make_ragged(name, tail=128, device="cuda")
    check_ragged(r, sample=True, seed=2)


def test_repeat_calls_bit_identical(variant):
    r = workloads.make_ragged_custom(5, 192, 512, [100, 0, 300, 7, 513], seed=3, tail=9)
    a = run_ragged(r)
    b = run_ragged(r)
    for x, y in zip(a[:3], b[:3]):
        assert bool((x.view(torch.int16) == y.view(torch.int16)).all())


@pytest.mark.parametrize("N", [2048, 264])
def test_masked_counts_across_box_and_tile_edges(N):
    """mmax=256 (two row tiles per expert), counts around the 32-row A boxes and the 128-row
    tiles, N with and without 64-wide chunks; inactive rows NaN and untouched."""
    counts = [0, 1, 31, 32, 33, 127, 128, 129, 255, 256]
    m = workloads.make_masked(E=len(counts), mmax=256, K=192, N=N, masked_m=counts, seed=61)
    out = sentinel((m.E, m.mmax, m.N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.masked_forward(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                      status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, act, _ = oracle.masked_forward(m.A, m.W, m.masked_m)
    flat = out.view(-1, m.N)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act], "masked")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())


@pytest.mark.parametrize("E,mmax,K,N,counts", [
    (5, 40, 200, 136, [40, 0, 17, 1, 33]),        # mmax and K off the 32-row box / 64 grid
    (3, 100, 776, 392, [100, 64, 99]),            # N without 64-wide chunks, 13 K blocks
    (4, 300, 64, 128, [300, 129, 0, 257]),        # three 128-row blocks per expert
    (70, 16, 128, 256, None),                     # many experts, 16-row capacity
])
def test_masked_forward_shapes(E, mmax, K, N, counts):
    """Masked forward over shapes around the kernel's blocks: the active rows of each expert
    in blocks of up to 128 (32-row boxes), 128-column weight tiles, 64-deep stages; inactive
    rows NaN in A and untouched in out."""
    if counts is None:
        counts = np.random.default_rng(7).integers(0, mmax + 1, E)
    m = workloads.make_masked(E=E, mmax=mmax, K=K, N=N, masked_m=counts, seed=63)
    out = sentinel((E, mmax, N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.masked_forward(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                      status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, act, _ = oracle.masked_forward(m.A, m.W, m.masked_m)
    flat = out.view(-1, N)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act], "masked")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())


@pytest.mark.parametrize("with_scale", [False, True])
def test_masked_forward_bias_scale(with_scale):
    """Masked forward with the fused bias (and per-row bias scale, NaN in inactive rows so a
    read of one would show): h = A W[e] + s[e*mmax + r] bias[e] for active rows only."""
    m = workloads.make_masked(E=6, mmax=72, K=256, N=384, masked_m=[72, 0, 5, 33, 64, 1],
                              seed=65)
    g = torch.Generator().manual_seed(9)
    bias = torch.randn(m.E, m.N, generator=g).to(torch.bfloat16)
    scale = None
    if with_scale:
        scale = torch.randn(m.E * m.mmax, generator=g, dtype=torch.float32)
        act_rows = np.zeros(m.E * m.mmax, bool)
        for e in range(m.E):
            act_rows[e * m.mmax: e * m.mmax + int(m.masked_m[e])] = True
        scale[torch.from_numpy(~act_rows)] = float("nan")
    out = sentinel((m.E, m.mmax, m.N))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.masked_forward_ex(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                         bias=bias.cuda(), bias_scale=None if scale is None else scale.cuda(),
                         status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, act, _ = oracle.masked_forward_ex(m.A, m.W, m.masked_m, bias,
                                           None if scale is None else scale.numpy(), 0)
    flat = out.view(-1, m.N)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act],
                 "masked bias")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())


@pytest.mark.parametrize("alpha,beta", [(1.0, 0.0), (0.5, 1.0), (-2.0, 0.25)])
def test_wgrad_f32_scaling_and_accumulation(alpha, beta, variant):
    """fp32 dW = alpha * A_e^T dY_e + beta * dW in place; beta == 0 never reads dW (NaN there
    stays out of the result); an empty expert gives beta * dW."""
    r = workloads.make_ragged_custom(len(SWEEP), 200, 328, SWEEP, seed=73, tail=64)
    A, dY = r.A.cuda(), r.dY.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    rng = np.random.default_rng(3)
    old = rng.standard_normal((r.E, r.K, r.N)).astype(np.float32) * 10
    if beta == 0.0:
        old[:] = np.nan
    dW = torch.from_numpy(old.copy()).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.wgrad_f32(A, dY, offs, dW, alpha=alpha, beta=beta, status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref = oracle.wgrad_accumulate(r.A, r.dY, r.offs, old, alpha, beta)
    assert_close(dW.double().cpu().numpy(), ref, "wgrad_f32")


def test_wgrad_f32_accumulates_over_two_calls():
    """Two accumulating calls into one main-grad buffer equal the sum of two products."""
    r = workloads.make_ragged("gateup", tail=128, device="cuda")
    offs = torch.from_numpy(r.offs).cuda()
    dW = torch.zeros(r.E, r.K, r.N, dtype=torch.float32, device="cuda")
    gg.wgrad_f32(r.A, r.dY, offs, dW, alpha=1.0, beta=1.0)
    gg.wgrad_f32(r.A, r.dY, offs, dW, alpha=1.0, beta=1.0)
    torch.cuda.synchronize()
    ks = sample_k(r.K, 5)
    ref = 2.0 * oracle.wgrad(oracle.as_u16(r.A), oracle.as_u16(r.dY), r.offs, ks=ks)
    got = dW[:, torch.from_numpy(ks).cuda(), :].double().cpu().numpy()
    assert_close(got, ref, "wgrad_f32 accumulated twice")


@pytest.mark.parametrize("act,with_bias,with_scale", [(0, True, False), (0, True, True),
                                                      (1, False, False), (1, True, True)])
def test_forward_epilogue_bias_scale_silu(act, with_bias, with_scale, variant):
    """Fused epilogue: h = A W[e] + s[r] bias[e]; SiLU-and-mul over gate/up blocks of 128.
    Rows past the last offset keep their sentinel and their NaN scale entries are not read."""
    sizes = [0, 1, 127, 128, 129, 300, 17]
    K, N = 192, 512
    r = workloads.make_ragged_custom(len(sizes), K, N, sizes, seed=81, tail=40)
    A, W = r.A.cuda(), r.W.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    g = torch.Generator().manual_seed(5)
    bias = torch.randn(r.E, N, generator=g).to(torch.bfloat16) if with_bias else None
    scale = None
    if with_scale:
        scale = torch.randn(r.rows_alloc, generator=g, dtype=torch.float32)
        scale[r.T:] = float("nan")  # capacity rows: never read
    ncols = N // 2 if act == 1 else N
    out = sentinel((r.rows_alloc, ncols))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.forward_ex(A, W, offs, out, bias=None if bias is None else bias.cuda(),
                  bias_scale=None if scale is None else scale.cuda(), act=act, status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, grp = oracle.forward_ex(r.A, r.W, r.offs, bias,
                                 None if scale is None else scale.numpy(), act)
    T = r.T
    assert_close(to_f64(out[:T]), ref[:T], "forward_ex")
    assert bool(is_sentinel(out[T:]).all())


@pytest.mark.parametrize("with_bias,w_nk", [(False, False), (True, False), (True, True)])
def test_forward_silu_mul_concatenated_gate_up(with_bias, w_nk, variant):
    """SiLU-and-mul with W's columns as [gate | up] (GG_FLAG_GATE_UP_CONCAT): out[r, j] =
    silu(h[r, j]) * h[r, N/2 + j] against the oracle's concatenated reading, on every launch
    shape and with W stored [E, N, K]; rows past the last offset keep their sentinel."""
    sizes = [0, 1, 127, 128, 129, 300, 17, 600]
    K, N = 192, 1024
    r = workloads.make_ragged_custom(len(sizes), K, N, sizes, seed=85, tail=40)
    A, W = r.A.cuda(), r.W.cuda()
    offs = torch.from_numpy(r.offs).cuda()
    g = torch.Generator().manual_seed(6)
    bias = torch.randn(r.E, N, generator=g).to(torch.bfloat16) if with_bias else None
    Wk = W.transpose(1, 2).contiguous() if w_nk else W
    out = sentinel((r.rows_alloc, N // 2))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gg.forward_ex(A, Wk, offs, out, bias=None if bias is None else bias.cuda(),
                  act=gg.ACT_SILU_MUL, gate_up_concat=True, w_nk=w_nk, status=st)
    torch.cuda.synchronize()
    s = int(st.item())
    assert s & gg.DEV_LAUNCHED and (s & gg.DEV_ERROR_MASK) == 0
    ref, _ = oracle.forward_ex(r.A, r.W, r.offs, bias, None, 1, concat=True)
    assert_close(to_f64(out[: r.T]), ref[: r.T], "forward silu concat")
    assert bool(is_sentinel(out[r.T:]).all())


def test_masked_forward_silu_mul_concatenated_gate_up():
    """The masked gate-up GEMM with fused SiLU-and-mul over [gate | up] weight halves."""
    m = workloads.make_masked(E=8, mmax=128, K=768, N=1536, seed=87)
    bias = torch.randn(8, 1536).to(torch.bfloat16)
    out = sentinel((8, 128, 768))
    gg.masked_forward_ex(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                         bias=bias.cuda(), act=gg.ACT_SILU_MUL, gate_up_concat=True)
    torch.cuda.synchronize()
    ref, act, _ = oracle.masked_forward_ex(m.A, m.W, m.masked_m, bias, None, 1, concat=True)
    flat = out.view(-1, 768)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act],
                 "masked silu concat")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())


def test_masked_forward_silu_mul_on_the_sglang_shape():
    """The masked down-GEMM input: gate-up GEMM of the masked layout with fused SiLU-and-mul,
    written only for the active rows (inactive rows NaN in A, sentinel in out)."""
    m = workloads.make_masked(E=8, mmax=128, K=768, N=1536, seed=83)
    bias = torch.randn(8, 1536).to(torch.bfloat16)
    out = sentinel((8, 128, 768))
    gg.masked_forward_ex(m.A.cuda(), m.W.cuda(), torch.from_numpy(m.masked_m).cuda(), out,
                         bias=bias.cuda(), act=gg.ACT_SILU_MUL)
    torch.cuda.synchronize()
    ref, act, _ = oracle.masked_forward_ex(m.A, m.W, m.masked_m, bias, None, 1)
    flat = out.view(-1, 768)
    assert_close(to_f64(flat[torch.from_numpy(np.nonzero(act)[0]).cuda()]), ref[act], "masked silu")
    assert bool(is_sentinel(flat[torch.from_numpy(np.nonzero(~act)[0]).cuda()]).all())
