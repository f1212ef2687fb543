"""GPU forward, input gradient and fused Q/K/V against the oracle.

Floating-point results: every element within 4e-3 * sum |a||w| of the fp64
oracle, and exactly 0 where that bound is 0.  Integer-exact inputs (all
products and partial sums exact in fp32): bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def run_fwd(inp, gs):
    blob = pack_on_gpu(inp, gs)
    N, K = inp.codes.shape
    y = q().q4gsw_linear_fwd(blob, N, K, gs, cuda(inp.x))
    route = q().q4gsw_last_route()
    q().q4gsw_device_error_check()   # a wait that ran out is reported as such, not as a wrong number
    return y.cpu().numpy(), route


def run_bwd(inp, gs):
    blob = pack_on_gpu(inp, gs)
    N, K = inp.codes.shape
    dx = q().q4gsw_linear_bwd_input(blob, N, K, gs, cuda(inp.d_out))
    route = q().q4gsw_last_route()
    q().q4gsw_device_error_check()
    return dx.cpu().numpy(), route


def check_fwd(inp, gs, rows=None):
    y, route = run_fwd(inp, gs)
    if rows is None:
        ref, bnd = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    else:
        ref, bnd = o.linear_fwd_rows(bits(inp.x), inp.codes, bits(inp.scales), gs, rows)
        y = y[rows]
    return assert_within_bound(y, ref, bnd, what=f"fwd {inp.shape.name} [{route}]")


def check_bwd(inp, gs, rows=None):
    dx, route = run_bwd(inp, gs)
    if rows is None:
        ref, bnd = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    else:
        ref, bnd = o.linear_bwd_input_rows(bits(inp.d_out), inp.codes, bits(inp.scales), gs, rows)
        dx = dx[rows]
    return assert_within_bound(dx, ref, bnd, what=f"bwd {inp.shape.name} [{route}]")


# ----------------------------------------------------------------------------- the five workloads
def test_tiny_config_fwd_bwd():
    sh = wl.tiny()[0]
    inp = wl.make_inputs(sh)
    check_fwd(inp, sh.group_size)
    check_bwd(inp, sh.group_size)


@pytest.mark.parametrize("sh", wl.decode(), ids=lambda s: s.name)
def test_decode_config_fwd(sh):
    check_fwd(wl.make_inputs(sh), sh.group_size)


@pytest.mark.parametrize("sh", wl.adapter(), ids=lambda s: s.name)
def test_adapter_config_fwd_bwd(sh):
    inp = wl.make_inputs(sh)
    check_fwd(inp, sh.group_size)
    check_bwd(inp, sh.group_size)


def _sample_rows(M, seed):
    if M <= 1024:
        return None
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.arange(8), np.arange(M - 8, M), rng.choice(M, 240, replace=False)]))


@pytest.mark.parametrize("sh", wl.sweep(), ids=lambda s: s.name)
def test_sweep_config_fwd_bwd(sh):
    inp = wl.make_inputs(sh)
    rows = _sample_rows(sh.M, sh.seed)
    check_fwd(inp, sh.group_size, rows)
    check_bwd(inp, sh.group_size, rows)


@pytest.mark.parametrize("sh", wl.qkv(), ids=lambda s: s.name)
def test_qkv_config(sh):
    inp = wl.make_inputs(sh)
    Nq, Nk, Nv = sh.splits
    blob = pack_on_gpu(inp, sh.group_size)
    yq, yk, yv = q().q4gsw_qkv_fwd(blob, Nq, Nk, Nv, sh.K, sh.group_size, cuda(inp.x))
    torch.cuda.synchronize()
    route = q().q4gsw_last_route()
    assert route.startswith("qkv")
    refs = o.qkv_fwd(bits(inp.x), inp.codes, bits(inp.scales), sh.group_size, Nq, Nk, Nv)
    for got, (ref, bnd), name in zip((yq, yk, yv), refs, "qkv"):
        assert_within_bound(got.cpu().numpy(), ref, bnd, what=f"qkv {name} M={sh.M} [{route}]")


# ----------------------------------------------------------------------------- exact cases
@pytest.mark.parametrize("M,N,K,gs", [(1, 64, 128, 32), (5, 136, 320, 64), (16, 64, 1024, 16),
                                      (17, 128, 256, 32), (130, 256, 512, 128), (508, 192, 384, 32)])
def test_integer_exact_inputs_are_bit_exact(M, N, K, gs):
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M * 31 + N)
    y, r1 = run_fwd(inp, gs)
    ref, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    assert np.array_equal(y.astype(np.float64), ref), r1
    dx, r2 = run_bwd(inp, gs)
    refb, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    assert np.array_equal(dx.astype(np.float64), refb), r2


@pytest.mark.parametrize("M", [1, 12, 200])
def test_one_hot_probes(M):
    N, K, gs = 64, 256, 32
    rng = np.random.default_rng(M)
    scales = rng.uniform(0.5, 2.0, (K // gs, N)).astype(np.float16)
    for n0, k0 in ((0, 0), (1, 31), (2, 32), (17, 63), (40, 64), (63, 255), (33, 130)):
        codes = np.full((N, K), 8, np.uint8)
        codes[n0, k0] = 9
        x = np.zeros((M, K), np.float16)
        x[:, k0] = 1.0
        d = np.zeros((M, N), np.float16)
        d[:, n0] = 1.0
        inp = wl.Inputs(x=x, codes=codes, scales=scales, d_out=d, shape=wl.Shape("probe", M, N, K, gs, 0))
        y, _ = run_fwd(inp, gs)
        want = np.zeros((M, N), np.float32)
        want[:, n0] = np.float32(scales[k0 // gs, n0])
        assert np.array_equal(y, want), (n0, k0)
        dx, _ = run_bwd(inp, gs)
        want = np.zeros((M, K), np.float32)
        want[:, k0] = np.float32(scales[k0 // gs, n0])
        assert np.array_equal(dx, want), (n0, k0)


def test_zero_point_codes_give_exact_zeros():
    inp = wl.random_inputs(24, 64, 256, 32, seed=3)
    inp.codes[:] = 8
    y, _ = run_fwd(inp, 32)
    dx, _ = run_bwd(inp, 32)
    assert not y.any() and not dx.any()


def test_scale_homogeneity_is_exact():
    inp = wl.random_inputs(6, 128, 512, 64, seed=4)
    y1, _ = run_fwd(inp, 64)
    inp.scales = (inp.scales * np.float16(2)).astype(np.float16)
    y2, _ = run_fwd(inp, 64)
    assert np.array_equal(y2, 2 * y1)


@pytest.mark.parametrize("M", [3, 64])
def test_adjoint_identity(M):
    inp = wl.random_inputs(M, 256, 512, 32, seed=M)
    y, _ = run_fwd(inp, 32)
    dx, _ = run_bwd(inp, 32)
    d = inp.d_out.astype(np.float64)
    x = inp.x.astype(np.float64)
    lhs = float(np.sum(d * y))
    rhs = float(np.sum(dx * x))
    w = np.abs(o.dequant_w32(inp.codes, bits(inp.scales), 32).astype(np.float64))
    scale = float(np.sum((np.abs(d) @ w) * np.abs(x)))
    assert abs(lhs - rhs) <= 4e-3 * scale


def test_qkv_equals_three_separate_forwards():
    Nq, Nk, Nv, K, gs, M = 128, 64, 64, 256, 32, 20
    inp = wl.integer_exact_inputs(M, Nq + Nk + Nv, K, gs, seed=11)
    blob = pack_on_gpu(inp, gs)
    yq, yk, yv = q().q4gsw_qkv_fwd(blob, Nq, Nk, Nv, K, gs, cuda(inp.x))
    for (lo, hi), got in zip(((0, Nq), (Nq, Nq + Nk), (Nq + Nk, Nq + Nk + Nv)), (yq, yk, yv)):
        part = wl.Inputs(x=inp.x, codes=inp.codes[lo:hi].copy(), scales=inp.scales[:, lo:hi].copy(),
                         d_out=inp.d_out, shape=inp.shape)
        ysep, _ = run_fwd(part, gs)
        assert np.array_equal(got.cpu().numpy(), ysep)


# ----------------------------------------------------------------------------- edges
def test_empty_batch_leaves_outputs_untouched():
    m = q()
    inp = wl.random_inputs(1, 64, 128, 32, seed=2)
    blob = pack_on_gpu(inp, 32)
    y = torch.full((0, 64), 1.0, device="cuda")
    m.q4gsw_linear_fwd(blob, 64, 128, 32, torch.empty((0, 128), dtype=torch.float16, device="cuda"), y)
    assert m.q4gsw_last_route() == "empty"


@pytest.mark.parametrize("M", [1, 2, 7, 8, 9, 15, 16, 17, 33, 127, 129, 511, 512, 513])
def test_ragged_token_counts(M):
    inp = wl.random_inputs(M, 72, 192, 64, seed=100 + M)
    check_fwd(inp, 64)
    check_bwd(inp, 64)


@pytest.mark.parametrize("N,K,gs", [(8, 64, 64), (24, 64, 16), (40, 448, 64), (1032, 576, 32)])
def test_odd_weight_shapes(N, K, gs):
    inp = wl.random_inputs(9, N, K, gs, seed=N + K)
    check_fwd(inp, gs)
    check_bwd(inp, gs)


@pytest.fixture(params=["tma", "tma_xs", "reg"])
def gemv_variant(request):
    """Pins the GEMV: TMA-ring weight stream (activations from global memory, or
    staged in the ring) or register-fed (q4gsw_debug_pin_routes)."""
    q().q4gsw_debug_pin_routes(gemv=request.param)
    yield request.param
    q().q4gsw_debug_pin_routes()


@pytest.mark.parametrize("M,N,K,gs", [(1, 64, 128, 32), (3, 136, 320, 16), (8, 1032, 576, 64), (9, 72, 256, 128),
                                      (16, 264, 1344, 32), (5, 8, 64, 64), (2, 4096, 2048, 256),
                                      (1, 128, 2048, 512), (12, 200, 4096, 1024), (7, 392, 3008, 64)])
def test_gemv_routes(M, N, K, gs, gemv_variant):
    inp = wl.random_inputs(M, N, K, gs, seed=3 * M + N + K)
    check_fwd(inp, gs)
    route = q().q4gsw_last_route()
    tma = gemv_variant != "reg"
    assert route.startswith("gemv_tma_fwd" if tma else "gemv_fwd"), route
    assert ("x=staged" in route) == (gemv_variant == "tma_xs"), route
    check_bwd(inp, gs)
    route = q().q4gsw_last_route()
    assert route.startswith("gemv_tma_bwd" if tma else "gemv_bwd"), route
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M + 1)
    y, _ = run_fwd(inp, gs)
    ref, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    assert np.array_equal(y.astype(np.float64), ref)
    dx, _ = run_bwd(inp, gs)
    ref, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    assert np.array_equal(dx.astype(np.float64), ref)


def test_non_default_stream():
    m = q()
    inp = wl.random_inputs(4, 128, 256, 32, seed=8)
    blob = pack_on_gpu(inp, 32)
    s = torch.cuda.Stream()
    x = cuda(inp.x)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y = m.q4gsw_linear_fwd(blob, 128, 256, 32, x)
    s.synchronize()
    ref, bnd = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    assert_within_bound(y.cpu().numpy(), ref, bnd)


# ----------------------------------------------------------------------------- tcgen05 GEMM routes
@pytest.fixture(params=["ts", "ss1", "ss2"])
def gemm_variant(request):
    """Pins the GEMM route: weight tile in tensor memory (ts, the default), or
    dequantised into shared memory with one or two 128-token accumulators."""
    q().q4gsw_debug_pin_routes(gemm=request.param)
    yield request.param
    q().q4gsw_debug_pin_routes()


def _route_ok(route, direction, variant):
    if variant == "ts":
        return route.startswith(f"tcgen05_ts_gemm_{direction}") and "tile=128x" in route
    return route.startswith(f"tcgen05_gemm_{direction}") and f"tile={128 * int(variant[2])}x" in route


@pytest.mark.parametrize("M,N,K,gs", [(17, 256, 256, 32), (40, 72, 192, 64), (130, 1032, 576, 32),
                                      (129, 264, 448, 16), (300, 520, 320, 64), (64, 256, 4096, 128),
                                      (520, 264, 192, 16), (33, 136, 128, 128)])
def test_gemm_route_tails(M, N, K, gs, gemm_variant):
    inp = wl.random_inputs(M, N, K, gs, seed=M + N + K)
    check_fwd(inp, gs)
    route = q().q4gsw_last_route()
    assert _route_ok(route, "fwd", gemm_variant), route
    check_bwd(inp, gs)
    route = q().q4gsw_last_route()
    assert _route_ok(route, "bwd", gemm_variant), route


@pytest.mark.parametrize("M,route", [(16, "gemv_tma"), (17, "tcgen05_ts_gemm"), (512, "tcgen05_ts_gemm"),
                                     (513, "tcgen05_gemm")])
def test_one_group_over_all_of_k_at_every_route_boundary(M, route):
    # gs == K: a single scale group per output feature; each side of the
    # GEMV / tensor-memory GEMM / shared-memory GEMM switches
    q().q4gsw_debug_pin_routes()
    inp = wl.random_inputs(M, 136, 512, 512, seed=M + 1)
    check_fwd(inp, 512)
    assert q().q4gsw_last_route().startswith(route + "_fwd"), q().q4gsw_last_route()
    check_bwd(inp, 512)
    assert q().q4gsw_last_route().startswith(route + "_bwd"), q().q4gsw_last_route()


def test_gemm_default_routes():
    q().q4gsw_debug_pin_routes()
    inp = wl.random_inputs(100, 256, 256, 32, seed=5)
    check_fwd(inp, 32)
    route = q().q4gsw_last_route()
    assert route.startswith("tcgen05_ts_gemm_fwd") and "tile=128x112x64" in route, route   # one 112-token tile
    inp = wl.random_inputs(600, 256, 256, 32, seed=6)
    check_bwd(inp, 32)
    route = q().q4gsw_last_route()
    assert route.startswith("tcgen05_gemm_bwd"), route   # above 512 tokens: shared-memory route


def test_ss_variant_choice_is_automatic():
    q().q4gsw_debug_pin_routes(gemm="ss")
    try:
        inp = wl.random_inputs(100, 256, 256, 32, seed=5)
        check_fwd(inp, 32)
        assert "tile=128x" in q().q4gsw_last_route()   # fewer than 129 tokens: one accumulator
    finally:
        q().q4gsw_debug_pin_routes()


def test_gemm_split_k_cluster_reduction(gemm_variant):
    # one output tile and a long contraction: the route splits K over a cluster
    inp = wl.integer_exact_inputs(100, 256, 4096, 64, seed=9)
    y, route = run_fwd(inp, 64)
    assert "x8" in route.split("grid=")[1], route
    ref, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 64)
    assert np.array_equal(y.astype(np.float64), ref)
    inp = wl.integer_exact_inputs(100, 4096, 256, 64, seed=10)
    dx, route = run_bwd(inp, 64)
    assert "x8" in route.split("grid=")[1], route
    ref, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), 64)
    assert np.array_equal(dx.astype(np.float64), ref)


@pytest.mark.parametrize("kind,M,N,K,gs", [("fwd", 512, 2048, 8192, 32), ("bwd", 512, 8192, 2048, 32),
                                            ("fwd", 400, 2048, 8192, 64)])
def test_split_k_wide_tiles_push_partials_bit_exact(kind, M, N, K, gs):
    # split-K with tiles of at least 192 tokens: each CTA stores its partial
    # rows into the owning rank's shared memory (the other split-K tests run
    # narrower tiles, whose owners read the partials remotely instead); the
    # 400-token case has a 208-token tile whose last rows lie past M
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M + N)
    if kind == "fwd":
        y, route = run_fwd(inp, gs)
        ref, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    else:
        y, route = run_bwd(inp, gs)
        ref, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    assert route.startswith("tcgen05_ts_gemm"), route
    bt = int(route.split("tile=128x")[1].split("x")[0])
    splits = int(route.split("grid=")[1].split()[0].split("x")[2])
    assert bt >= 192 and splits > 1, route
    assert np.array_equal(y.astype(np.float64), ref)


def test_no_kernel_wait_ran_out():
    q().q4gsw_device_error_check()


@pytest.mark.parametrize("M,N,K,gs,f32", [(1, 64, 64, 32, 0), (3, 264, 448, 16, 0), (8, 4096, 1024, 32, 0),
                                          (9, 1032, 2048, 128, 0), (16, 512, 4096, 256, 0), (16, 14336, 4096, 128, 0),
                                          (5, 520, 1088, 64, 1), (13, 2048, 2048, 16, 1)])
def test_staged_and_global_activations_agree_bit_for_bit(M, N, K, gs, f32):
    # the forward TMA ring takes its activation fragments from the stage (pin
    # "tma_xs") or from global memory (pin "tma"); the MMAs are the same, so
    # the outputs are identical
    inp = wl.random_inputs(M, N, K, gs, seed=M + N)
    scales = inp.scales.astype(np.float32) if f32 else inp.scales
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(scales), gs)
    outs = []
    try:
        for pin in ("tma", "tma_xs"):
            q().q4gsw_debug_pin_routes(gemv=pin)
            outs.append(q().q4gsw_linear_fwd(blob, N, K, gs, cuda(inp.x), f32s=bool(f32)).cpu())
            assert ("x=staged" in q().q4gsw_last_route()) == (pin == "tma_xs")
    finally:
        q().q4gsw_debug_pin_routes()
    q().q4gsw_device_error_check()
    assert torch.equal(outs[0], outs[1])
