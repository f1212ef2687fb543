"""Failure detection on the GPU without a fault, and concurrent first calls.

A kernel wait that runs out must not hang or fault the GPU: the waiting kernel
records a time-out in the device status word and returns, the context stays
usable, and q4gsw_device_error_check reports Q4GSW_ERR_TIMEOUT once (the check
clears the word).  The probe waits on a barrier that nothing completes, under
a short limit, through the same bounded wait every compute kernel uses.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import assert_within_bound, bits, cuda, pack_on_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


@pytest.mark.parametrize("limit_us", [20, 2000])
def test_wait_that_runs_out_is_reported_once(limit_us):
    m = q()
    m.q4gsw_device_error_check()            # start from a clear word
    m.q4gsw_debug_wait_timeout(limit_us)
    with pytest.raises(m.Q4gswError) as err:
        m.q4gsw_device_error_check()
    assert err.value.status_name == "Q4GSW_ERR_TIMEOUT"
    m.q4gsw_device_error_check()            # cleared by the first check
    # the context is still usable: a compute call right after gives correct results
    inp = wl.random_inputs(3, 64, 256, 32, seed=12)
    blob = pack_on_gpu(inp, 32)
    y = m.q4gsw_linear_fwd(blob, 64, 256, 32, cuda(inp.x))
    ref, bnd = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    assert_within_bound(y.cpu().numpy(), ref, bnd)
    m.q4gsw_device_error_check()


def test_time_out_recorded_on_another_stream_is_kept_for_the_next_check():
    m = q()
    m.q4gsw_device_error_check()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        m.q4gsw_debug_wait_timeout(50)
    side.synchronize()
    with pytest.raises(m.Q4gswError):
        m.q4gsw_device_error_check()
    m.q4gsw_device_error_check()


CONCURRENT = r"""
import sys, threading
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import bit_group_quantized_q4gsw_b200 as q
import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl
torch.cuda.init()
bits = lambda a: np.asarray(a, np.float16).view(np.uint16)
jobs = [(1, 128, 512), (12, 128, 512), (40, 256, 512), (700, 256, 512)]   # one job per kernel route
packed, xs, results, errors = [], [], [None] * len(jobs), []
for i, (M, N, K) in enumerate(jobs):
    inp = wl.random_inputs(M, N, K, 32, seed=40 + i)
    packed.append((inp, q.q4gsw_prepack(torch.from_numpy(inp.codes).cuda(), torch.from_numpy(inp.scales).cuda(), 32)))
torch.cuda.synchronize()
barrier = threading.Barrier(len(jobs))
def work(i):
    try:
        inp, blob = packed[i]
        M, N, K = jobs[i]
        s = torch.cuda.Stream()
        x = torch.from_numpy(inp.x).cuda()
        d = torch.from_numpy(inp.d_out).cuda()
        torch.cuda.synchronize()
        barrier.wait()
        with torch.cuda.stream(s):
            y = q.q4gsw_linear_fwd(blob, N, K, 32, x)
            dx = q.q4gsw_linear_bwd_input(blob, N, K, 32, d)
        s.synchronize()
        results[i] = (y.cpu().numpy(), dx.cpu().numpy())
    except Exception as e:
        errors.append(repr(e))
ts = [threading.Thread(target=work, args=(i,)) for i in range(len(jobs))]
[t.start() for t in ts]
[t.join() for t in ts]
assert not errors, errors
for i, (M, N, K) in enumerate(jobs):
    inp, _ = packed[i]
    ref, bnd = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    assert (np.abs(results[i][0] - ref) <= 4e-3 * bnd).all(), i
    ref, bnd = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), 32)
    assert (np.abs(results[i][1] - ref) <= 4e-3 * bnd).all(), i
q.q4gsw_device_error_check()
print("concurrent first calls ok")
"""


def test_first_calls_from_several_threads_at_once():
    # a fresh process, so that every first-use cache is filled by racing threads
    r = subprocess.run([sys.executable, "-c", CONCURRENT, ROOT], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "concurrent first calls ok" in r.stdout
