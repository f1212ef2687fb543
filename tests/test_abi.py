"""Host-side checks of the C ABI: the library loads without a GPU, exports
every function that include/q4gsw.h declares, sizes blobs like the layout
definition, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import oracle as o
from bit_group_quantized_q4gsw_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "q4gsw.h")).read()
    return re.findall(r"Q4GSW_API\s+[\w\s\*]*?\b(q4gsw_\w+)\s*\(", text)


def test_library_exports_every_declared_function():
    lib = b.library()
    names = declared_functions()
    assert len(names) == 28
    assert sorted(names) == sorted(n for n, _, _ in b.SIGNATURES)
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_the_in_tree_build():
    lib = b.library()
    assert os.path.samefile(lib._name, b.LIB_PATH)


@pytest.mark.parametrize("N,K,gs", [(64, 128, 32), (2048, 2048, 32), (14336, 4096, 128), (8, 64, 64), (24, 192, 16)])
def test_packed_bytes_matches_layout_definition(N, K, gs):
    assert b.q4gsw_packed_bytes(N, K, gs) == o.packed_layout(N, K, gs)["total_bytes"]


@pytest.mark.parametrize("N,K,gs,status", [
    (0, 128, 32, 2), (64, 0, 32, 2), (62, 128, 32, 2), (64, 130, 32, 2), (64, 128, 30, 2),
    (68, 128, 32, 3), (64, 96, 32, 3), (64, 128, 48, 4), (64, 128, 8, 4), (64, 128, 256, 4),
])
def test_bad_shapes_are_rejected_on_the_host(N, K, gs, status):
    lib = b.library()
    assert lib.q4gsw_packed_bytes(N, K, gs) == 0
    fake = 0x100000  # never dereferenced: the shape check fails first
    assert lib.q4gsw_linear_fwd(fake, N, K, gs, fake, 4, fake, None) == status
    assert lib.q4gsw_linear_bwd_input(fake, N, K, gs, fake, 4, fake, None) == status


def test_null_alignment_size_and_empty_batch():
    lib = b.library()
    fake = 0x100000
    assert lib.q4gsw_linear_fwd(None, 64, 128, 32, fake, 4, fake, None) == 1
    assert lib.q4gsw_linear_fwd(fake, 64, 128, 32, fake + 8, 4, fake, None) == 3
    assert lib.q4gsw_linear_fwd(fake, 64, 128, 32, fake, -1, fake, None) == 2
    assert lib.q4gsw_linear_fwd(None, 64, 128, 32, None, 0, None, None) == 0       # empty batch
    assert b.q4gsw_last_route() == "empty"
    assert lib.q4gsw_linear_bwd_input(fake, 64, 128, 32, None, 4, fake, None) == 1
    assert lib.q4gsw_prepack(fake, fake, 64, 128, 32, fake, 100, None) == 7         # blob too small
    assert lib.q4gsw_prepack(fake, None, 64, 128, 32, fake, 1 << 20, None) == 1
    assert lib.q4gsw_prepack(fake + 4, fake, 64, 128, 32, fake, 1 << 20, None) == 3
    assert lib.q4gsw_unpack(fake, 64, 128, 32, None, None) == 1
    assert lib.q4gsw_dequant(fake, 64, 128, 32, None, None, None) == 1
    assert lib.q4gsw_dequant(fake, 64, 128, 32, fake + 4, None, None) == 3


def test_qkv_split_rules():
    lib = b.library()
    fake = 0x100000
    q = lambda Nq, Nk, Nv, M=4: lib.q4gsw_qkv_fwd(fake, Nq, Nk, Nv, 128, 32, fake, M, fake, fake, fake, None)
    assert q(0, 16, 16) == 2
    assert q(64, 12, 16) == 2 or q(64, 12, 16) == 3
    assert q(64, 20, 20) == 3          # multiples of 4 but not of 8
    assert q(64, 16, 16, M=0) == 0
    assert lib.q4gsw_qkv_fwd(fake, 64, 16, 16, 128, 32, fake, 4, fake, None, fake, None) == 1


def test_status_strings_and_version():
    assert b.q4gsw_layout_version() == o.LAYOUT_VERSION == 1
    for s in range(9):
        assert b.q4gsw_status_str(s)
    assert b.q4gsw_status_str(99) == "unknown status"


def test_embedding_arguments_are_checked_on_the_host():
    lib = b.library()
    fake = 0x100000
    assert lib.q4gsw_embedding(fake, 62, 128, 32, fake, 4, fake, None) == 2        # N % 4
    assert lib.q4gsw_embedding(fake, 64, 96, 32, fake, 4, fake, None) == 3         # K % 64
    assert lib.q4gsw_embedding(fake, 64, 128, 48, fake, 4, fake, None) == 4        # group size
    assert lib.q4gsw_embedding(fake, 64, 128, 32, fake, -1, fake, None) == 2       # T < 0
    assert lib.q4gsw_embedding(None, 64, 128, 32, None, 0, None, None) == 0        # T = 0: nothing to do
    assert b.q4gsw_last_route() == "empty"
    assert lib.q4gsw_embedding(None, 64, 128, 32, fake, 4, fake, None) == 1
    assert lib.q4gsw_embedding(fake, 64, 128, 32, None, 4, fake, None) == 1
    assert lib.q4gsw_embedding(fake, 64, 128, 32, fake + 2, 4, fake, None) == 3    # indices 4-byte aligned
    assert lib.q4gsw_embedding(fake, 64, 128, 32, fake, 4, fake + 4, None) == 3    # out 16-byte aligned
    assert b.q4gsw_status_str(9).startswith("an embedding index")


def test_every_workload_shape_is_accepted_by_the_library():
    from bit_group_quantized_q4gsw_b200 import workloads as wl
    for sh in wl.all_shapes():
        assert b.q4gsw_packed_bytes(sh.N, sh.K, sh.group_size) == \
            o.packed_layout(sh.N, sh.K, sh.group_size)["total_bytes"] > 0, sh.name
        if sh.splits:
            assert sum(sh.splits) == sh.N and all(s % 8 == 0 for s in sh.splits), sh.name


def test_embedding_token_ids_are_seeded_and_in_range():
    import numpy as np
    from bit_group_quantized_q4gsw_b200 import workloads as wl
    for sh in wl.embedding():
        ids = wl.embedding_indices(sh)
        assert ids.dtype == np.int32 and ids.shape == (sh.M,)
        assert ids.min() >= 0 and ids.max() < sh.N
        assert np.array_equal(ids, wl.embedding_indices(sh))


def test_debug_route_pins_are_checked_and_thread_local():
    import threading
    lib = b.library()
    assert lib.q4gsw_debug_pin_routes(4, 0) == 2          # gemv pin out of range
    assert lib.q4gsw_debug_pin_routes(0, 5) == 2          # gemm pin out of range
    assert lib.q4gsw_debug_pin_routes(-1, 0) == 2
    for gemv in range(4):
        for gemm in range(5):
            assert lib.q4gsw_debug_pin_routes(gemv, gemm) == 0
    seen = []
    # a pin set on another thread does not leak into this one, nor the reverse:
    # the other thread's status on a valid pin is OK whatever this thread pinned
    t = threading.Thread(target=lambda: seen.append(lib.q4gsw_debug_pin_routes(1, 1)))
    t.start()
    t.join()
    assert seen == [0]
    assert lib.q4gsw_debug_pin_routes(0, 0) == 0


def test_wait_probe_limit_is_checked_on_the_host():
    lib = b.library()
    assert lib.q4gsw_debug_wait_timeout(0, None) == 2
    assert lib.q4gsw_debug_wait_timeout(1000001, None) == 2


def test_f32s_entry_points_check_arguments_on_the_host():
    import oracle.q4gsw_variants as v
    lib = b.library()
    fake = 0x100000
    assert lib.q4gsw_packed_bytes_f32s(64, 128, 32) == v.packed_layout_f32s(64, 128, 32)["total_bytes"]
    assert lib.q4gsw_packed_bytes_f32s(62, 128, 32) == 0
    need = lib.q4gsw_packed_bytes_f32s(64, 128, 32)
    assert lib.q4gsw_prepack_f32s(fake, fake, 64, 128, 32, fake, need - 1, None) == 7
    assert lib.q4gsw_prepack_f32s(fake, None, 64, 128, 32, fake, need, None) == 1
    assert lib.q4gsw_linear_fwd_f32s(fake, 64, 96, 32, fake, 4, fake, None) == 3
    assert lib.q4gsw_linear_bwd_input_f32s(None, 64, 128, 32, fake, 4, fake, None) == 1
    assert lib.q4gsw_qkv_fwd_f32s(fake, 64, 20, 20, 128, 32, fake, 4, fake, fake, fake, None) == 3
    assert lib.q4gsw_embedding_f32s(fake, 64, 128, 32, fake, -1, fake, None) == 2
    assert lib.q4gsw_dequant_f32s(fake, 64, 128, 32, None, None, None) == 1
    assert lib.q4gsw_linear_fwd_f32s(None, 64, 128, 32, None, 0, None, None) == 0


def test_adapter_entry_points_check_arguments_on_the_host():
    lib = b.library()
    fake = 0x100000
    assert lib.q4gsw_adapter_workspace_bytes(512, 16) == 512 * 128
    assert lib.q4gsw_adapter_workspace_bytes(512, 12) == 0
    assert lib.q4gsw_adapter_workspace_bytes(512, 72) == 0
    f = lib.q4gsw_adapter_fwd
    assert f(fake, 64, 128, 32, fake, fake, 12, fake, 4, fake, fake, 4 * 128, None) == 2    # rank rule
    assert f(fake, 64, 128, 32, fake, fake, 16, fake, 4, fake, fake, 4 * 128 - 1, None) == 7   # workspace
    assert f(fake, 64, 128, 32, None, fake, 16, fake, 4, fake, fake, 4 * 128, None) == 1
    assert f(fake, 64, 128, 32, fake, fake, 16, fake, 4, fake, fake + 8, 4 * 128, None) == 3
    assert f(None, 64, 128, 32, None, None, 16, None, 0, None, None, 0, None) == 0            # empty batch
    g = lib.q4gsw_adapter_bwd_input
    assert g(fake, 62, 128, 32, fake, fake, 16, fake, 4, fake, fake, 4 * 128, None) == 2
    assert g(fake, 64, 128, 32, fake, fake, 16, fake, -1, fake, fake, 4 * 128, None) == 2


def test_noalloc_adapter_rejects_sizes_beyond_its_array_on_the_host():
    lib = b.library()
    fake = 0x100000
    # 8193 tokens need more than the 1 MiB array: rejected before any set-up or launch
    assert lib.q4gsw_adapter_fwd_noalloc(fake, 64, 128, 32, fake, fake, 16, fake, 8193, fake, None) == 7
    assert lib.q4gsw_adapter_fwd_noalloc(fake, 64, 128, 32, fake, fake, 16, fake, -1, fake, None) == 2


def test_dq8ca_entry_points_check_arguments_on_the_host():
    lib = b.library()
    fake = 0x100000
    need = lib.q4gsw_dq8ca_workspace_bytes(4, 128)
    assert need == 512 + 256 + 256 and lib.q4gsw_dq8ca_workspace_bytes(4, 100) == 0
    f = lib.q4gsw_linear_dq8ca_fwd
    assert f(fake, 64, 128, 16, fake, 4, fake, fake, need, None) == 4          # gs 16: unsupported
    assert f(fake, 64, 128, 32, fake, 4, fake, fake, need - 1, None) == 7      # workspace too small
    assert f(fake, 64, 128, 32, fake, 4, fake, None, need, None) == 1
    assert f(fake, 64, 96, 32, fake, 4, fake, fake, need, None) == 3
    assert f(None, 64, 128, 32, None, 0, None, None, 0, None) == 0             # empty batch
    g = lib.q4gsw_dq8ca_quantize
    assert g(fake, 4, 100, fake, need, None) == 3 and g(fake, 4, -64, fake, need, None) == 2
    assert g(fake, 4, 128, fake, need - 1, None) == 7
