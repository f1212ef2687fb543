"""Shared test helpers: move seeded inputs to the GPU and compare the CUDA
results with the oracle under the per-element bound."""
import numpy as np
import torch

import oracle as o

REL = 4e-3   # |gpu - oracle| <= REL * sum |a| |w|  per element; exact zero where the bound is 0


def bits(a16):
    return np.asarray(a16, dtype=np.float16).view(np.uint16)


def cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def pack_on_gpu(inp, gs):
    import bit_group_quantized_q4gsw_b200 as q
    return q.q4gsw_prepack(cuda(inp.codes), cuda(inp.scales), gs)


def assert_within_bound(got, ref, bound, rel=REL, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    lim = rel * bound
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside bound; worst at {i}: "
                             f"got {got[i]!r} want {ref[i]!r} bound {bound[i]!r}")
    zero = bound == 0
    assert (got[zero] == 0).all(), f"{what}: nonzero output where the bound is 0"
    return float((err / np.where(lim > 0, lim, 1)).max())
