"""GPU embedding gather against the oracle: every element is an exact fp32
product, so the rows must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def gather(inp, gs, idx):
    blob = pack_on_gpu(inp, gs)
    N, K = inp.codes.shape
    out = q().q4gsw_embedding(blob, N, K, gs, torch.from_numpy(np.asarray(idx, np.int32)).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy(), blob


@pytest.mark.parametrize("N,K,gs,T", [(64, 128, 32, 4), (1032, 576, 16, 300), (24, 2048, 128, 17),
                                      (8, 64, 64, 1), (200, 4096, 1024, 65)])
def test_embedding_rows_are_bit_exact(N, K, gs, T):
    inp = wl.random_inputs(2, N, K, gs, seed=N + K + T)
    rng = np.random.default_rng(T)
    idx = rng.integers(0, N, T).astype(np.int32)
    idx[0], idx[-1] = 0, N - 1                    # first and last rows, even and odd
    got, blob = gather(inp, gs, idx)
    ref = o.embedding(inp.codes, bits(inp.scales), gs, idx)
    assert got.shape == ref.shape
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))   # signed zeros included
    assert q().q4gsw_last_route().startswith("embedding_gather")
    w32, _ = q().q4gsw_dequant(blob, N, K, gs, want_w16=False)
    assert np.array_equal(got, w32.cpu().numpy()[idx])
    q().q4gsw_device_error_check()


def test_embedding_index_out_of_range_is_reported_and_zeroed():
    N, K, gs = 64, 128, 32
    inp = wl.random_inputs(2, N, K, gs, seed=5)
    idx = np.array([3, N, -1, 5], np.int32)
    got, _ = gather(inp, gs, idx)
    ref = o.embedding(inp.codes, bits(inp.scales), gs, idx[[0, 3]])
    assert np.array_equal(got[[0, 3]], ref)
    assert (got[1] == 0).all() and (got[2] == 0).all()
    with pytest.raises(q().Q4gswError) as e:
        q().q4gsw_device_error_check()
    assert e.value.status_name == "Q4GSW_ERR_INDEX"
    q().q4gsw_device_error_check()                # the check cleared the word


def test_embedding_of_no_tokens_enqueues_nothing():
    inp = wl.random_inputs(2, 64, 128, 32, seed=6)
    blob = pack_on_gpu(inp, 32)
    out = q().q4gsw_embedding(blob, 64, 128, 32, torch.empty(0, dtype=torch.int32, device="cuda"))
    assert out.shape == (0, 128)
    assert q().q4gsw_last_route() == "empty"


def test_embedding_on_a_non_default_stream():
    inp = wl.random_inputs(2, 136, 320, 16, seed=7)
    blob = pack_on_gpu(inp, 16)
    idx = np.arange(136, dtype=np.int32)[::-1].copy()
    ids = cuda(idx)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out = q().q4gsw_embedding(blob, 136, 320, 16, ids)
    s.synchronize()
    assert np.array_equal(out.cpu().numpy(), o.embedding(inp.codes, bits(inp.scales), 16, idx))


@pytest.mark.parametrize("sh", wl.embedding(), ids=lambda s: s.name)
def test_embedding_configs_sampled_rows(sh):
    inp = wl.make_inputs(sh, M=1)
    idx = wl.embedding_indices(sh)
    got, _ = gather(inp, sh.group_size, idx)
    rows = np.unique(np.linspace(0, len(idx) - 1, min(len(idx), 64)).astype(int))
    ref = o.embedding(inp.codes, bits(inp.scales), sh.group_size, idx[rows])
    assert np.array_equal(got[rows], ref)
