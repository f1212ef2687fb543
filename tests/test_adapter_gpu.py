"""Frozen-base low-rank adapter step on the GPU against the oracle.

"[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
input-grad)", PR description: the input gradient of the frozen 4-bit base is
there for on-device adapter training.  Reading (as in the oracle):
    y   = x dequant(W)^T + (x A^T) B^T,     d_x = d_out dequant(W) + (d_out B) A.
Bound per element: 4e-3 * (sum |x||w| + sum_j (sum_k |x||A_jk|) |B_nj|).
"""
import numpy as np
import pytest
import torch

import oracle as o
from oracle import q4gsw_variants as v
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def adapter_mats(N, K, r, seed, scale=0.05):
    rng = np.random.default_rng(seed)
    A = (rng.standard_normal((r, K)) * scale).astype(np.float16)
    B = (rng.standard_normal((N, r)) * scale).astype(np.float16)
    return A, B


def run(kind, blob, N, K, gs, A, B, act, ws=None):
    m = q()
    f = m.q4gsw_adapter_fwd if kind == "fwd" else m.q4gsw_adapter_bwd_input
    out = f(blob, N, K, gs, cuda(A), cuda(B), cuda(act), workspace=ws)
    route = m.q4gsw_last_route()
    m.q4gsw_device_error_check()
    return out.cpu().numpy(), route


@pytest.mark.parametrize("M,N,K,gs,r", [(512, 8192, 2048, 32, 16), (512, 2048, 8192, 32, 64), (37, 264, 448, 16, 8),
                                        (1, 128, 256, 32, 24), (300, 1032, 576, 64, 40), (17, 136, 1024, 128, 64)])
def test_adapter_fwd_bwd_within_bound(M, N, K, gs, r):
    inp = wl.random_inputs(M, N, K, gs, seed=M + N + r, dout_sigma=1e-2 if M == 512 else 1.0)
    A, B = adapter_mats(N, K, r, seed=r)
    blob = pack_on_gpu(inp, gs)
    y, r1 = run("fwd", blob, N, K, gs, A, B, inp.x)
    assert r1.startswith("adapter_fwd") and "adapter_stage=1" in r1, r1
    ref, bnd = v.adapter_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert_within_bound(y, ref, bnd, what=f"adapter fwd [{r1}]")
    dx, r2 = run("bwd", blob, N, K, gs, A, B, inp.d_out)
    ref, bnd = v.adapter_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert_within_bound(dx, ref, bnd, what=f"adapter bwd [{r2}]")


@pytest.mark.parametrize("M,N,K,gs,r", [(40, 256, 256, 32, 16), (300, 264, 512, 64, 64), (5, 128, 4096, 64, 8)])
def test_adapter_integer_exact(M, N, K, gs, r):
    # integers everywhere: the intermediate and every partial sum are exact
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M + r)
    rng = np.random.default_rng(r)
    A = rng.integers(-1, 2, (r, K)).astype(np.float16)
    B = rng.integers(-1, 2, (N, r)).astype(np.float16)
    blob = pack_on_gpu(inp, gs)
    y, _ = run("fwd", blob, N, K, gs, A, B, inp.x)
    ref, _ = v.adapter_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert np.array_equal(y.astype(np.float64), ref)
    dx, _ = run("bwd", blob, N, K, gs, A, B, inp.d_out)
    ref, _ = v.adapter_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert np.array_equal(dx.astype(np.float64), ref)


def test_zero_adapter_adds_exactly_nothing_to_the_base_route():
    # a zero B (or A) adds +0 once: the base result, bit for bit (a contraction of
    # 4 stages runs unsplit, so the summation order is fixed)
    M, N, K, gs, r = 300, 256, 256, 32, 16
    inp = wl.random_inputs(M, N, K, gs, seed=3)
    A, B = adapter_mats(N, K, r, seed=4)
    blob = pack_on_gpu(inp, gs)
    q().q4gsw_debug_pin_routes(gemm="ts")
    try:
        base = q().q4gsw_linear_fwd(blob, N, K, gs, cuda(inp.x)).cpu().numpy()
        dbase = q().q4gsw_linear_bwd_input(blob, N, K, gs, cuda(inp.d_out)).cpu().numpy()
    finally:
        q().q4gsw_debug_pin_routes()
    y, _ = run("fwd", blob, N, K, gs, A, np.zeros_like(B), inp.x)
    assert np.array_equal(y, base)
    dx, _ = run("bwd", blob, N, K, gs, np.zeros_like(A), B, inp.d_out)
    assert np.array_equal(dx, dbase)


def test_adapter_adjoint_identity():
    M, N, K, gs, r = 64, 512, 1024, 32, 32
    inp = wl.random_inputs(M, N, K, gs, seed=5)
    A, B = adapter_mats(N, K, r, seed=6, scale=0.1)
    blob = pack_on_gpu(inp, gs)
    y, _ = run("fwd", blob, N, K, gs, A, B, inp.x)
    dx, _ = run("bwd", blob, N, K, gs, A, B, inp.d_out)
    d = inp.d_out.astype(np.float64)
    x = inp.x.astype(np.float64)
    lhs, rhs = float(np.sum(d * y)), float(np.sum(dx * x))
    _, bnd = v.adapter_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert abs(lhs - rhs) <= 4e-3 * float(np.sum(np.abs(d) * bnd))


def test_workspace_is_reused_and_overwritten():
    M, N, K, gs, r = 100, 256, 512, 32, 16
    inp = wl.random_inputs(M, N, K, gs, seed=7)
    A, B = adapter_mats(N, K, r, seed=8)
    blob = pack_on_gpu(inp, gs)
    ws = torch.full((q().library().q4gsw_adapter_workspace_bytes(M, r),), 0xFF, dtype=torch.uint8, device="cuda")
    y1, _ = run("fwd", blob, N, K, gs, A, B, inp.x, ws)
    dx, _ = run("bwd", blob, N, K, gs, A, B, inp.d_out, ws)
    y2, _ = run("fwd", blob, N, K, gs, A, B, inp.x, ws)
    assert np.array_equal(y1, y2)
    ref, bnd = v.adapter_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs, bits(A), bits(B))
    assert_within_bound(dx, ref, bnd)
