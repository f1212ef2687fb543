"""Fused Q/K/V forward on every kernel route, against the oracle.

"[ExecuTorch][WebGPU] Replace broad QKV fusion with BK64 kernel", description
of #21131: one packing of the Q/K/V weights and scales, three distinct
outputs.  The split points must land on the right buffer on every route: the
GEMV routes (M <= 16: register-fed and TMA-ring), the tensor-memory GEMM
(16 < M <= 512) and the shared-memory GEMM (M > 512, one or two 128-token
accumulators per CTA).  The 64/8/24 triple puts both split points inside one
16-row GEMV tile and inside one 128-feature GEMM tile.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu

SPLITS = {"config": (2048, 512, 512, 2048, 32),    # Hq32/Hkv8/D64 triple of the QKV prefill config
          "ragged": (64, 8, 24, 256, 32)}          # both split points inside one 16-row tile


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def run_qkv(inp, splits, gs):
    Nq, Nk, Nv = splits
    blob = pack_on_gpu(inp, gs)
    outs = q().q4gsw_qkv_fwd(blob, Nq, Nk, Nv, inp.codes.shape[1], gs, cuda(inp.x))
    route = q().q4gsw_last_route()
    q().q4gsw_device_error_check()
    return [t.cpu().numpy() for t in outs], route


def check_route(M, split_name, gemv="auto", gemm="auto", route_prefix=""):
    Nq, Nk, Nv, K, gs = SPLITS[split_name]
    q().q4gsw_debug_pin_routes(gemv=gemv, gemm=gemm)
    try:
        inp = wl.random_inputs(M, Nq + Nk + Nv, K, gs, seed=7 * M + Nk)
        outs, route = run_qkv(inp, (Nq, Nk, Nv), gs)
        assert route.startswith("qkv " + route_prefix), route
        refs = o.qkv_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, Nq, Nk, Nv)
        for got, (ref, bnd), name in zip(outs, refs, "qkv"):
            assert_within_bound(got, ref, bnd, what=f"qkv {name} M={M} {split_name} [{route}]")
        # integer-exact inputs: every route must agree with the oracle bit for bit
        inp = wl.integer_exact_inputs(M, Nq + Nk + Nv, K, gs, seed=M + 5)
        outs, route = run_qkv(inp, (Nq, Nk, Nv), gs)
        refs = o.qkv_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, Nq, Nk, Nv)
        for got, (ref, _), name in zip(outs, refs, "qkv"):
            assert np.array_equal(got.astype(np.float64), ref), f"qkv {name} M={M} {split_name} [{route}]"
    finally:
        q().q4gsw_debug_pin_routes()


@pytest.mark.parametrize("split_name", ["config", "ragged"])
@pytest.mark.parametrize("gemv", ["reg", "tma", "tma_xs"])
@pytest.mark.parametrize("M", [1, 4, 9, 16])
def test_qkv_gemv_routes(M, gemv, split_name):
    check_route(M, split_name, gemv=gemv, route_prefix="gemv_fwd" if gemv == "reg" else "gemv_tma_fwd")


@pytest.mark.parametrize("split_name", ["config", "ragged"])
@pytest.mark.parametrize("gemm", ["ss1", "ss2"])
@pytest.mark.parametrize("M", [600, 1024])
def test_qkv_shared_memory_gemm_routes(M, gemm, split_name):
    check_route(M, split_name, gemm=gemm, route_prefix="tcgen05_gemm_fwd")


@pytest.mark.parametrize("M", [40, 300])
def test_qkv_tensor_memory_gemm_ragged_split(M):
    check_route(M, "ragged", gemm="ts", route_prefix="tcgen05_ts_gemm_fwd")


def test_qkv_default_route_above_512_tokens():
    check_route(600, "ragged", route_prefix="tcgen05_gemm_fwd")
