"""The allocation-free adapter forward (q4gsw_adapter_fwd_noalloc), through the C ABI.

Some callers cannot allocate device memory when they call the library: a
latency-critical path where cudaMalloc may synchronise the whole device, a
plugin inside a runtime that owns all device memory, a program whose memory is
fixed up front.  For them the adapter forward has a variant that keeps its
intermediate in a fixed scratch array inside the library instead of a
workspace the caller passes.  This test calls that variant twice in a row (the
second call finds the first call's data in the shared array) and checks both
results against the workspace entry point and against the oracle's bound.

The file is named so that pytest collects it last; it passes alone in a fresh
process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import q4gsw_variants as v
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import REL, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu


def lib():
    import bit_group_quantized_q4gsw_b200 as m
    return m.library()


def adapter_case(M, N, K, gs, r, seed):
    inp = wl.random_inputs(M, N, K, gs, seed=seed)
    rng = np.random.default_rng(seed + 1)
    A = (rng.standard_normal((r, K)) * 0.05).astype(np.float16)
    B = (rng.standard_normal((N, r)) * 0.05).astype(np.float16)
    return inp, A, B


@pytest.mark.parametrize("M,N,K,gs,r", [(512, 8192, 2048, 32, 16), (77, 264, 448, 16, 24)])
def test_noalloc_adapter_matches_the_workspace_entry_point_twice(M, N, K, gs, r):
    L = lib()
    inp, A, B = adapter_case(M, N, K, gs, r, seed=M + r)
    blob = pack_on_gpu(inp, gs)
    a, b, x = cuda(A), cuda(B), cuda(inp.x)
    stream = torch.cuda.current_stream().cuda_stream
    ref, bnd = v.adapter_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, bits(A), bits(B))

    # the entry point with a caller-owned workspace
    y_ws = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = torch.empty(L.q4gsw_adapter_workspace_bytes(M, r), dtype=torch.uint8, device="cuda")
    st = L.q4gsw_adapter_fwd(blob.data_ptr(), N, K, gs, a.data_ptr(), b.data_ptr(), r, x.data_ptr(), M,
                             y_ws.data_ptr(), ws.data_ptr(), ws.numel(), ctypes.c_void_p(stream))
    assert st == 0, L.q4gsw_status_str(st)

    # the allocation-free variant, two calls in a row into fresh outputs
    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = L.q4gsw_adapter_fwd_noalloc(blob.data_ptr(), N, K, gs, a.data_ptr(), b.data_ptr(), r, x.data_ptr(), M,
                                         y.data_ptr(), ctypes.c_void_p(stream))
        assert st == 0, L.q4gsw_status_str(st)
        outs.append(y)
    torch.cuda.synchronize()
    assert L.q4gsw_device_error_check(ctypes.c_void_p(stream)) == 0
    y_ws = y_ws.cpu().numpy().astype(np.float64)
    for y in outs:
        y = y.cpu().numpy().astype(np.float64)
        assert np.isfinite(y).all()
        assert (np.abs(y - y_ws) <= REL * bnd).all()     # against the workspace entry point
        assert (np.abs(y - ref) <= REL * bnd).all()      # and against the oracle


def test_noalloc_adapter_rejects_a_batch_beyond_its_array():
    L = lib()
    x = torch.zeros((8193, 64), dtype=torch.float16, device="cuda")
    y = torch.zeros((8193, 64), dtype=torch.float32, device="cuda")
    w = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = L.q4gsw_adapter_fwd_noalloc(w.data_ptr(), 64, 64, 64, w.data_ptr(), w.data_ptr(), 16, x.data_ptr(), 8193,
                                     y.data_ptr(), None)
    assert L.q4gsw_status_str(st).decode() == "buffer too small"
    assert (y == 0).all()   # nothing was enqueued
