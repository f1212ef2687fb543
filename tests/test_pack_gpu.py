"""GPU packing, unpacking and dequantisation: bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import bits, cuda

pytestmark = pytest.mark.gpu


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


SHAPES = [(64, 128, 32), (8, 64, 64), (24, 192, 16), (200, 640, 128), (2048, 2048, 32), (3072, 2048, 32)]


@pytest.mark.parametrize("N,K,gs", SHAPES)
def test_prepack_bytes_equal_oracle(N, K, gs):
    inp = wl.random_inputs(1, N, K, gs, seed=N + K + gs, scales="loguniform")
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    want = o.pack_fast(inp.codes, bits(inp.scales), gs)
    got = blob.cpu().numpy()
    assert got.size == want.size
    assert np.array_equal(got, want)
    assert q().q4gsw_last_route() == "prepack"


def test_prepack_small_blob_equals_loop_oracle():
    inp = wl.random_inputs(1, 16, 128, 32, seed=1)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), 32)
    assert np.array_equal(blob.cpu().numpy(), o.pack(inp.codes, bits(inp.scales), 32))


@pytest.mark.parametrize("N,K,gs", SHAPES)
def test_unpack_round_trip(N, K, gs):
    inp = wl.random_inputs(1, N, K, gs, seed=7 * N + K)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    assert np.array_equal(q().q4gsw_unpack(blob, N, K, gs).cpu().numpy(), inp.codes)


@pytest.mark.parametrize("N,K,gs,dist", [(64, 128, 32, "uniform"), (512, 1024, 128, "loguniform"),
                                         (96, 256, 16, "loguniform")])
def test_dequant_bit_exact(N, K, gs, dist):
    inp = wl.random_inputs(1, N, K, gs, seed=N * 3 + gs, scales=dist)
    blob = q().q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)
    w32, w16 = q().q4gsw_dequant(blob, N, K, gs)
    want32 = o.dequant_w32(inp.codes, bits(inp.scales), gs)
    want16 = o.dequant_w16_bits_fast(inp.codes, bits(inp.scales), gs)
    assert np.array_equal(w32.cpu().numpy().view(np.uint32), want32.view(np.uint32))
    assert np.array_equal(w16.cpu().numpy().view(np.uint16), want16)


def test_dequant_every_code_and_scale_pattern():
    # all 16 codes x all finite fp16 scale bit patterns of both signs, zero and
    # subnormals included: every product the tensor cores can be fed.
    scales_bits = np.concatenate([np.arange(0, 0x7C00), np.arange(0x8000, 0xFC00)]).astype(np.uint16)
    N = 2 * ((scales_bits.size + 1) // 2)
    N = (N + 7) // 8 * 8
    sb = np.zeros(N, np.uint16)
    sb[:scales_bits.size] = scales_bits
    K, gs = 64, 64
    codes = np.tile((np.arange(K) % 16).astype(np.uint8), (N, 1))
    s16 = sb.view(np.float16)[None, :]
    blob = q().q4gsw_prepack(cuda(codes), cuda(s16), gs)
    w32, w16 = q().q4gsw_dequant(blob, N, K, gs)
    want16 = o.dequant_w16_bits_fast(codes, sb[None, :], gs)
    want32 = o.dequant_w32(codes, sb[None, :], gs)
    assert np.array_equal(w16.cpu().numpy().view(np.uint16), want16)
    assert np.array_equal(w32.cpu().numpy().view(np.uint32), want32.view(np.uint32))


def test_prepack_rejects_out_of_range_codes():
    m = q()
    codes = np.full((16, 64), 3, np.uint8)
    codes[5, 17] = 16
    with pytest.raises(m.Q4gswError) as ei:
        m.q4gsw_prepack(cuda(codes), cuda(np.ones((1, 16), np.float16)), 64)
    assert ei.value.status_name == "Q4GSW_ERR_CODE_RANGE"


def test_prepack_into_larger_buffer_and_trailer():
    m = q()
    inp = wl.random_inputs(1, 64, 128, 32, seed=5)
    nbytes = m.q4gsw_packed_bytes(64, 128, 32)
    buf = torch.full((nbytes + 512,), 0xAB, dtype=torch.uint8, device="cuda")
    m.q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), 32, packed=buf)
    got = buf.cpu().numpy()
    assert np.array_equal(got[:nbytes], o.pack(inp.codes, bits(inp.scales), 32))
    assert (got[nbytes:] == 0xAB).all()   # nothing written past the blob
    tw = o.trailer_words(got[:nbytes], 64, 128, 32)
    assert list(tw[:6]) == [0x53473451, 1, 64, 128, 32, 0]
