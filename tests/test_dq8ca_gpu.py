"""linear_dq8ca_q4gsw on the GPU against the oracle.

The shader list in "Upstream the Gemma 4 Vulkan support we carry on our
ExecuTorch fork" (issue #1361) carries linear_dq8ca_q4gsw beside linear_q4gsw:
int8 dynamically quantised activations times the 4-bit weight.  Reading (as in
the oracle): per token lo = min(0, min x), hi = max(0, max x),
a_s = (hi - lo) / 255, a_z = rint(-128 - lo / a_s),
q = clamp(rint(x / a_s) + a_z, -128, 127), all in IEEE fp32; then
y = a_s * sum_g s * sum (q - a_z)(code - 8).

The quantised activations are integers decided in fp32 on both sides, so they
are compared bit for bit; y within 4e-3 of the oracle's bound
a_s * sum_g |s| sum |q - a_z| |code - 8|, and bit for bit where every partial
sum is exact in fp32.
"""
import os

import numpy as np
import pytest
import torch

from oracle import q4gsw_variants as v
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def read_workspace(ws, M, K):
    """(q [M, K] int8 in column order, a_s fp32 [M], a_z int32 [M]) from the workspace."""
    lib = q().library()
    raw = ws.cpu().numpy()
    # byte 16 t + 4 i + slot of a 64-column block holds column 16 i + 4 t + (0, 2, 1, 3)[slot]
    qs = raw[:M * K].view(np.int8).reshape(M, K // 64, 4, 4, 4)[..., [0, 2, 1, 3]]
    qs = qs.transpose(0, 1, 3, 2, 4).reshape(M, K)
    o_s = lib.q4gsw_dq8ca_workspace_bytes(M, K) - 2 * (((4 * M) + 255) // 256 * 256)
    o_z = o_s + ((4 * M) + 255) // 256 * 256
    a_s = raw[o_s:o_s + 4 * M].view(np.float32)
    a_z = raw[o_z:o_z + 4 * M].view(np.int32)
    return qs, a_s, a_z


def quantise_rows(x):
    ws = q().q4gsw_dq8ca_quantize(cuda(x))
    q().q4gsw_device_error_check()
    return read_workspace(ws, *x.shape)


def activation_rows(M, K, seed):
    """Rows of every kind the quantiser meets: wide and narrow ranges, one-signed, zero, ties."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 4, (M, 1)))).astype(np.float16)
    if M > 4:
        x[1] = np.abs(x[1])
        x[2] = -np.abs(x[2])
        x[3] = 0
        x[4] = np.round(rng.uniform(-100, 155, K) * 2) / 2   # halves: ties of rint
        x[4, :2] = (-100, 155)
    return x


@pytest.mark.parametrize("M,K", [(1, 64), (7, 192), (64, 4096), (300, 14336)])
def test_quantised_activations_bit_exact(M, K):
    x = activation_rows(M, K, seed=M + K)
    got_q, got_s, got_z = quantise_rows(x)
    ref_q, ref_s, ref_z = v.dq8ca_quantize(bits(x))
    assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(got_z, ref_z)
    assert np.array_equal(got_q, ref_q)


def test_quantiser_reproduces_the_hand_worked_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "dq8ca_rows.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            name, sb, z, *pairs = line.split()
            rows.append((name, int(sb, 16), int(z), [float(p.split(":")[0]) for p in pairs],
                         [int(p.split(":")[1]) for p in pairs]))
    K = 64
    x = np.zeros((len(rows), K), np.float16)   # zero padding: the range holds 0 already
    for i, (_, _, _, xs, _) in enumerate(rows):
        x[i, :len(xs)] = xs
    got_q, got_s, got_z = quantise_rows(x)
    for i, (name, sb, z, xs, qs) in enumerate(rows):
        assert int(got_s[i:i + 1].view(np.uint32)[0]) == sb, name
        assert int(got_z[i]) == z, name
        assert list(got_q[i, :len(xs)].astype(int)) == qs, name
        assert (got_q[i, len(xs):] == z).all(), name       # q of 0 is the zero point


@pytest.mark.parametrize("M,N,K,gs", [(1, 64, 64, 32), (3, 264, 448, 64), (8, 4096, 1024, 32), (9, 1032, 2048, 128),
                                      (16, 512, 4096, 256), (37, 136, 640, 32), (1, 4096, 14336, 32),
                                      (16, 14336, 4096, 32)])
def test_linear_dq8ca_within_bound(M, N, K, gs):
    inp = wl.random_inputs(M, N, K, gs, seed=M * 7 + K)
    x = activation_rows(M, K, seed=N)
    blob = pack_on_gpu(inp, gs)
    y = q().q4gsw_linear_dq8ca_fwd(blob, N, K, gs, cuda(x))
    route = q().q4gsw_last_route()
    q().q4gsw_device_error_check()
    assert route.startswith("dq8ca"), route
    ref, bnd = v.linear_dq8ca_fwd(bits(x), inp.codes, bits(inp.scales), gs)
    assert_within_bound(y.cpu().numpy(), ref, bnd, what=f"dq8ca [{route}]")


@pytest.mark.parametrize("M,N,K,gs", [(5, 256, 512, 32), (16, 200, 1024, 64)])
def test_linear_dq8ca_integer_exact(M, N, K, gs):
    # every row spans exactly [-100, 155]: a_s = 1, a_z = -28, q = x - 28; the
    # power-of-two scales keep every partial sum exact in fp32
    inp = wl.integer_exact_inputs(M, N, K, gs, seed=M + N)
    rng = np.random.default_rng(K)
    x = rng.integers(-100, 156, (M, K)).astype(np.float16)
    x[:, 0], x[:, 1] = -100, 155
    blob = pack_on_gpu(inp, gs)
    y = q().q4gsw_linear_dq8ca_fwd(blob, N, K, gs, cuda(x)).cpu().numpy()
    ref, _ = v.linear_dq8ca_fwd(bits(x), inp.codes, bits(inp.scales), gs)
    assert np.array_equal(y.astype(np.float64), ref)


def test_workspace_reuse_and_group_size_limit():
    M, N, K, gs = 12, 256, 512, 32
    inp = wl.random_inputs(M, N, K, gs, seed=1)
    x = activation_rows(M, K, seed=2)
    blob = pack_on_gpu(inp, gs)
    ws = torch.full((q().library().q4gsw_dq8ca_workspace_bytes(M, K),), 0x5A, dtype=torch.uint8, device="cuda")
    y1 = q().q4gsw_linear_dq8ca_fwd(blob, N, K, gs, cuda(x), workspace=ws).cpu().numpy()
    y2 = q().q4gsw_linear_dq8ca_fwd(blob, N, K, gs, cuda(x), workspace=ws).cpu().numpy()
    assert np.array_equal(y1, y2)
    blob16 = pack_on_gpu(wl.random_inputs(M, N, K, 16, seed=1), 16)
    with pytest.raises(q().Q4gswError, match="unsupported"):
        q().q4gsw_linear_dq8ca_fwd(blob16, N, K, 16, cuda(x))
