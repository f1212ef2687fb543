"""fp32-scale variant (packed layout version 2) on the GPU against the oracle.

"Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork", issue
#1361: the fp32-scale dequantise-and-accumulate helper of the fork's shader
list.  Reading (as in the oracle): w32 = fp32_RNE((code - 8) * s32), tensor-core
operand fp16_RNE(w32), fp32 accumulation.

* packing, dequantisation (w32 and w16) and embedding rows: bit-exact;
* forward, input gradient and fused Q/K/V on every route: within
  4e-3 * sum |a||w| of the exact result, and bit-exact on integer-exact inputs;
* fp32 scales that are fp16 values give bit for bit the fp16-scale results.
"""
import os

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


def bits32(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def scales32(G, N, seed, kind="wide"):
    rng = np.random.default_rng(seed)
    if kind == "wide":   # fp32 scales that are not fp16 values, log-uniform over [1e-3, 5e-2]
        return np.exp(rng.uniform(np.log(1e-3), np.log(5e-2), (G, N))).astype(np.float32)
    if kind == "pow2":   # integer-exact: powers of two in [2^-6, 2^-3]
        return np.ldexp(1.0, rng.integers(-6, -2, (G, N))).astype(np.float32)
    raise ValueError(kind)


def pack32(codes, s32, gs):
    return q().q4gsw_prepack_f32s(cuda(codes), cuda(s32), gs)


def run(kind, blob, N, K, gs, a, splits=None):
    m = q()
    if kind == "fwd":
        out = m.q4gsw_linear_fwd(blob, N, K, gs, cuda(a), f32s=True)
    elif kind == "bwd":
        out = m.q4gsw_linear_bwd_input(blob, N, K, gs, cuda(a), f32s=True)
    else:
        out = m.q4gsw_qkv_fwd(blob, *splits, K, gs, cuda(a), f32s=True)
    route = m.q4gsw_last_route()
    m.q4gsw_device_error_check()
    if kind == "qkv":
        return [t.cpu().numpy() for t in out], route
    return out.cpu().numpy(), route


# --------------------------------------------------------------------------- pack / dequant / embedding
@pytest.mark.parametrize("N,K,gs", [(64, 128, 32), (136, 320, 16), (1032, 576, 64), (24, 192, 64)])
def test_prepack_f32s_matches_oracle_bytes(N, K, gs):
    rng = np.random.default_rng(N + K)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s32 = scales32(K // gs, N, N)
    blob = pack32(codes, s32, gs)
    assert blob.numel() == q().library().q4gsw_packed_bytes_f32s(N, K, gs) == \
        v.packed_layout_f32s(N, K, gs)["total_bytes"]
    assert np.array_equal(blob.cpu().numpy(), v.pack_f32s(codes, bits32(s32), gs))
    assert np.array_equal(q().q4gsw_unpack(blob, N, K, gs).cpu().numpy(), codes)


def test_dequant_f32s_hand_values_and_every_code():
    # the hand-worked fixture's scales, and 4000 random fp32 scales of every exponent
    # range an fp32 product can reach, against all 16 codes
    path = os.path.join(os.path.dirname(__file__), "golden", "dequant_f32s_values.txt")
    fixture = [int(line.split()[1], 16) for line in open(path) if line.strip() and not line.startswith("#")]
    rng = np.random.default_rng(5)
    exps = rng.integers(1, 254, 4000, dtype=np.uint32)
    sb = np.concatenate([np.array(fixture, np.uint32), (exps << 23) | rng.integers(0, 1 << 23, 4000, dtype=np.uint32),
                         np.array([1, 0x7F7FFFFF, 0x80000001, 0x00800000], np.uint32)])
    sb = sb[:(sb.size // 8) * 8]
    N, K, gs = sb.size, 64, 64
    codes = np.tile(np.arange(16, dtype=np.uint8), (N, K // 16))
    s32 = sb.reshape(1, N).view(np.float32)
    blob = pack32(codes, s32, gs)
    w32, w16 = q().q4gsw_dequant(blob, N, K, gs, f32s=True)
    with np.errstate(over="ignore"):
        want32 = v.dequant_w32_f32s(codes, sb.reshape(1, N), gs)
        want16 = v.dequant_w16_bits_f32s_fast(codes, sb.reshape(1, N), gs)
    assert np.array_equal(w32.cpu().numpy().view(np.uint32), want32.view(np.uint32))
    assert np.array_equal(w16.cpu().numpy().view(np.uint16), want16)


def test_embedding_f32s_rows_are_exact():
    N, K, gs = 128, 256, 32
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s32 = scales32(K // gs, N, 9)
    blob = pack32(codes, s32, gs)
    idx = np.array([127, 0, 64, 5, 5, 77], np.int32)
    rows = q().q4gsw_embedding(blob, N, K, gs, cuda(idx), f32s=True)
    q().q4gsw_device_error_check()
    assert np.array_equal(rows.cpu().numpy().view(np.uint32),
                          v.embedding_f32s(codes, bits32(s32), gs, idx).view(np.uint32))


# --------------------------------------------------------------------------- products on every route
ROUTES = [("reg", "auto", 1), ("tma", "auto", 1), ("reg", "auto", 9), ("tma", "auto", 16), ("auto", "ts", 40),
          ("auto", "ts", 300), ("auto", "ss1", 600), ("auto", "ss2", 600)]


@pytest.fixture(params=ROUTES, ids=lambda r: f"{r[0]}-{r[1]}-M{r[2]}")
def route(request):
    gemv, gemm, M = request.param
    q().q4gsw_debug_pin_routes(gemv=gemv, gemm=gemm)
    yield M
    q().q4gsw_debug_pin_routes()


@pytest.mark.parametrize("N,K,gs", [(264, 448, 16), (1032, 576, 32), (256, 1024, 128)])
def test_f32s_fwd_bwd_within_bound(route, N, K, gs):
    M = route
    inp = wl.random_inputs(M, N, K, gs, seed=M + N + gs)
    s32 = scales32(K // gs, N, N + gs)
    blob = pack32(inp.codes, s32, gs)
    y, r1 = run("fwd", blob, N, K, gs, inp.x)
    ref, bnd = v.linear_fwd_f32s(bits(inp.x), inp.codes, bits32(s32), gs)
    assert_within_bound(y, ref, bnd, what=f"f32s fwd [{r1}]")
    dx, r2 = run("bwd", blob, N, K, gs, inp.d_out)
    ref, bnd = v.linear_bwd_input_f32s(bits(inp.d_out), inp.codes, bits32(s32), gs)
    assert_within_bound(dx, ref, bnd, what=f"f32s bwd [{r2}]")


def test_f32s_integer_exact_and_fp16_valued_scales(route):
    M = route
    N, K, gs = 200, 512, 32
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M)
    s32 = inp.scales.astype(np.float32)           # powers of two: fp16 values too
    blob32 = pack32(inp.codes, s32, gs)
    blob16 = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    y, _ = run("fwd", blob32, N, K, gs, inp.x)
    ref, _ = v.linear_fwd_f32s(bits(inp.x), inp.codes, bits32(s32), gs)
    assert np.array_equal(y.astype(np.float64), ref)
    dx, _ = run("bwd", blob32, N, K, gs, inp.d_out)
    ref, _ = v.linear_bwd_input_f32s(bits(inp.d_out), inp.codes, bits32(s32), gs)
    assert np.array_equal(dx.astype(np.float64), ref)
    # random inputs, fp16-valued fp32 scales: the same bits as the fp16-scale path
    inp = wl.random_inputs(M, N, K, gs, seed=M + 3)
    blob32 = pack32(inp.codes, inp.scales.astype(np.float32), gs)
    blob16 = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    y32, _ = run("fwd", blob32, N, K, gs, inp.x)
    y16 = q().q4gsw_linear_fwd(blob16, N, K, gs, cuda(inp.x)).cpu().numpy()
    assert np.array_equal(y32, y16)
    d32, _ = run("bwd", blob32, N, K, gs, inp.d_out)
    d16 = q().q4gsw_linear_bwd_input(blob16, N, K, gs, cuda(inp.d_out)).cpu().numpy()
    assert np.array_equal(d32, d16)


@pytest.mark.parametrize("split", [(2048, 512, 512), (64, 8, 24)])
def test_f32s_qkv(route, split):
    M = route
    Nq, Nk, Nv = split
    K, gs = (2048, 32) if Nq == 2048 else (256, 32)
    inp = wl.random_inputs(M, Nq + Nk + Nv, K, gs, seed=M + Nk)
    s32 = scales32(K // gs, Nq + Nk + Nv, Nk)
    blob = pack32(inp.codes, s32, gs)
    outs, r = run("qkv", blob, Nq + Nk + Nv, K, gs, inp.x, splits=split)
    refs = v.qkv_fwd_f32s(bits(inp.x), inp.codes, bits32(s32), gs, Nq, Nk, Nv)
    for got, (ref, bnd), name in zip(outs, refs, "qkv"):
        assert_within_bound(got, ref, bnd, what=f"f32s qkv {name} [{r}]")


def test_f32s_sweep_shape_sampled_rows():
    # the large sweep matrix at M=1024 with fp32 scales: sampled rows against the oracle
    sh = wl.by_name("sweep_M1024_N14336_K4096")
    inp = wl.make_inputs(sh)
    s32 = scales32(sh.K // sh.group_size, sh.N, 77)
    blob = pack32(inp.codes, s32, sh.group_size)
    rows = np.array([0, 1, 511, 512, 1000, 1023])
    y, r = run("fwd", blob, sh.N, sh.K, sh.group_size, inp.x)
    ref, bnd = v.linear_fwd_f32s(bits(inp.x[rows]), inp.codes, bits32(s32), sh.group_size)
    assert_within_bound(y[rows], ref, bnd, what=f"f32s fwd M1024 [{r}]")
