"""The adapter-training step launched back to back, as the benchmark times it.

Consecutive launches of the tensor-memory GEMM overlap (programmatic dependent
launch), and with the packed weights rotating through more copies than L2 holds
the stages' loads land in any order.  Under exactly those conditions a barrier
protocol that lets a warp fall two phases behind a barrier deadlocks now and
then; the bounded wait then gives up after a second and raises the device error
word instead of hanging.  So this runs the five operations of the step (fused
Q/K/V forward, MLP up and down forward, down and up input gradients, M = 512) a
few hundred times without synchronising, then checks that no wait ran out and
that the last outputs equal those of one launch bit for bit.
"""
import numpy as np
import pytest
import torch

from bit_group_quantized_q4gsw_b200 import workloads as wl
from helpers import cuda, pack_on_gpu

pytestmark = pytest.mark.gpu

COPIES = 8    # 8 x (3 + 8.4 + 8.4 MB) of packed weights: more than the 126 MB L2
ROUNDS = 300


def q():
    import bit_group_quantized_q4gsw_b200 as m
    return m


def test_step_back_to_back_completes_and_repeats():
    m = q()
    qkv, up, down = wl.by_name("qkv_M512"), wl.by_name("adapter_up_M512"), wl.by_name("adapter_down_M512")
    ops = []
    for sh, kinds in ((qkv, ("qkv",)), (up, ("fwd", "bwd")), (down, ("fwd", "bwd"))):
        inp = wl.random_inputs(sh.M, sh.N, sh.K, sh.group_size, seed=sh.seed)
        blob = pack_on_gpu(inp, sh.group_size)
        blobs = [blob] + [blob.clone() for _ in range(COPIES - 1)]
        x, d = cuda(inp.x), cuda(inp.d_out)
        for kind in kinds:
            ops.append((sh, kind, blobs, x, d))

    def run(sh, kind, blob, x, d):
        if kind == "qkv":
            nq, nk, nv = sh.splits
            return m.q4gsw_qkv_fwd(blob, nq, nk, nv, sh.K, sh.group_size, x)
        if kind == "fwd":
            return (m.q4gsw_linear_fwd(blob, sh.N, sh.K, sh.group_size, x),)
        return (m.q4gsw_linear_bwd_input(blob, sh.N, sh.K, sh.group_size, d),)

    ref = []
    for sh, kind, blobs, x, d in ops:
        ref.append([t.cpu() for t in run(sh, kind, blobs[0], x, d)])
        torch.cuda.synchronize()
    m.q4gsw_device_error_check()

    last = [None] * len(ops)
    for i in range(ROUNDS):
        for j, (sh, kind, blobs, x, d) in enumerate(ops):
            last[j] = run(sh, kind, blobs[i % COPIES], x, d)
    torch.cuda.synchronize()
    m.q4gsw_device_error_check()   # raises if any bounded wait ran out
    for j, (sh, kind, _, _, _) in enumerate(ops):
        for got, want in zip(last[j], ref[j]):
            assert torch.equal(got.cpu(), want), f"{sh.name} {kind}: last of {ROUNDS} back-to-back launches differs"
            assert np.isfinite(want.numpy()).all()
