"""Seeded random shapes through every operation and route, against the oracle.

The hand-picked cases of the other files pin the boundaries the kernels are
built around (route switches, ragged tails, group sizes, splits); this file
draws shapes at random from the accepted space (N % 8 == 0, K % 64 == 0, gs a
power of two in [16, K], M from 1 to 600) so that a tiling or indexing mistake
that only some shapes reach has many chances to show.  Every draw is seeded, so
a failure reproduces from its parameters.
"""
import numpy as np
import pytest
import torch

import oracle as o
from oracle import q4gsw_variants as v
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda

pytestmark = pytest.mark.gpu


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def draw(seed):
    rng = np.random.default_rng(seed)
    M = int(rng.choice([int(rng.integers(1, 17)), int(rng.integers(17, 300)), int(rng.integers(300, 600))]))
    K = 64 * int(rng.integers(1, 40))
    gs = int(rng.choice([g for g in (16, 32, 64, 128, 256, 512, 1024) if g <= K and K % g == 0]))
    N = 8 * int(rng.integers(1, 80))
    return M, N, K, gs


SEEDS = list(range(64))


@pytest.mark.parametrize("seed", SEEDS)
def test_random_shape_fwd_bwd(seed):
    M, N, K, gs = draw(seed)
    inp = wl.random_inputs(M, N, K, gs, seed=1000 + seed)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    y = q().q4gsw_linear_fwd(blob, N, K, gs, cuda(inp.x))
    r1 = q().q4gsw_last_route()
    dx = q().q4gsw_linear_bwd_input(blob, N, K, gs, cuda(inp.d_out))
    r2 = q().q4gsw_last_route()
    q().q4gsw_device_error_check()
    ref, bnd = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    assert_within_bound(y.cpu().numpy(), ref, bnd, what=f"fwd M={M} N={N} K={K} gs={gs} [{r1}]")
    ref, bnd = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    assert_within_bound(dx.cpu().numpy(), ref, bnd, what=f"bwd M={M} N={N} K={K} gs={gs} [{r2}]")


@pytest.mark.parametrize("seed", SEEDS[:32])
def test_random_shape_qkv_f32s_embedding(seed):
    M, N, K, gs = draw(100 + seed)
    rng = np.random.default_rng(200 + seed)
    # a Q/K/V split of N into three multiples of 8 (each output 16-byte aligned), each at least 8
    cuts = np.sort(rng.choice(np.arange(1, N // 8), size=2, replace=False)) * 8 if N >= 24 else None
    inp = wl.random_inputs(M, N, K, gs, seed=2000 + seed)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    if cuts is not None:
        Nq, Nk = int(cuts[0]), int(cuts[1] - cuts[0])
        Nv = N - Nq - Nk
        outs = q().q4gsw_qkv_fwd(blob, Nq, Nk, Nv, K, gs, cuda(inp.x))
        route = q().q4gsw_last_route()
        refs = o.qkv_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, Nq, Nk, Nv)
        for got, (ref, bnd), name in zip(outs, refs, "qkv"):
            assert_within_bound(got.cpu().numpy(), ref, bnd, what=f"qkv {name} {Nq}/{Nk}/{Nv} M={M} K={K} [{route}]")
    # the same weight with fp32 scales that fp16 cannot hold
    s32 = (inp.scales.astype(np.float32) * np.float32(1 + 2.0 ** -12)).astype(np.float32)
    blob32 = q().q4gsw_prepack(cuda(inp.codes), cuda(s32), gs)
    y = q().q4gsw_linear_fwd(blob32, N, K, gs, cuda(inp.x), f32s=True)
    route = q().q4gsw_last_route()
    ref, bnd = v.linear_fwd_f32s(bits(inp.x), inp.codes, s32.view(np.uint32), gs)
    assert_within_bound(y.cpu().numpy(), ref, bnd, what=f"f32s fwd M={M} N={N} K={K} gs={gs} [{route}]")
    # embedding rows of the fp16 blob: exact
    ids = rng.integers(0, N, int(rng.integers(1, 64))).astype(np.int32)
    rows = q().q4gsw_embedding(blob, N, K, gs, cuda(ids))
    q().q4gsw_device_error_check()
    assert np.array_equal(rows.cpu().numpy(), o.embedding(inp.codes, bits(inp.scales), gs, ids))


@pytest.mark.parametrize("seed", SEEDS[:32])
def test_random_shape_adapter_and_dq8ca(seed):
    M, N, K, gs = draw(300 + seed)
    rng = np.random.default_rng(400 + seed)
    inp = wl.random_inputs(M, N, K, gs, seed=3000 + seed)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    r = 8 * int(rng.integers(1, 9))
    A = (rng.standard_normal((r, K)) * 0.05).astype(np.float16)
    B = (rng.standard_normal((N, r)) * 0.05).astype(np.float16)
    y = q().q4gsw_adapter_fwd(blob, N, K, gs, cuda(A), cuda(B), cuda(inp.x))
    route = q().q4gsw_last_route()
    ref, bnd = v.adapter_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert_within_bound(y.cpu().numpy(), ref, bnd, what=f"adapter fwd r={r} M={M} N={N} K={K} [{route}]")
    dx = q().q4gsw_adapter_bwd_input(blob, N, K, gs, cuda(A), cuda(B), cuda(inp.d_out))
    route = q().q4gsw_last_route()
    ref, bnd = v.adapter_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert_within_bound(dx.cpu().numpy(), ref, bnd, what=f"adapter bwd r={r} M={M} N={N} K={K} [{route}]")
    if gs >= 32 and M <= 64:
        yq = q().q4gsw_linear_dq8ca_fwd(blob, N, K, gs, cuda(inp.x))
        route = q().q4gsw_last_route()
        ref, bnd = v.linear_dq8ca_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
        assert_within_bound(yq.cpu().numpy(), ref, bnd, what=f"dq8ca M={M} N={N} K={K} gs={gs} [{route}]")
    q().q4gsw_device_error_check()
