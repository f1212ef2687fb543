"""Pins for the CPU oracle: it is checked against things other than itself.

* fp16 decode and encode against numpy's binary16 type (an independent
  implementation), exhaustively;
* the packing against hand-worked bytes and an exhaustive byte round trip;
* dequantisation against hand-worked values (zero point, ties, subnormals, inf);
* the products against exact rational arithmetic (``fractions.Fraction``) and
  exact integer arithmetic, and against closed-form probes (one-hot codes,
  all-zero-point codes, scale homogeneity, the adjoint identity);
* a mutation check: plausible mistakes planted in a copy of the oracle fail at
  least one pin.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as o
from bit_group_quantized_q4gsw_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    rows = {}
    lines = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lines.append(line.split())
        key, *vals = line.split()
        rows[key] = vals
    return rows, lines


def bits(a16):
    return np.asarray(a16, dtype=np.float16).view(np.uint16)


# --------------------------------------------------------------------------- fp16
def test_fp16_decode_exhaustive():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = o.fp16_bits_to_float(allbits)
    ref = allbits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(mine[0x8000]) and not np.signbit(mine[0])


def test_fp16_encode_exhaustive_on_every_dequant_product():
    # all 16 codes x all finite positive fp16 scales (subnormals included)
    sb = np.arange(1, 0x7C00, dtype=np.uint16)
    s = sb.view(np.float16).astype(np.float64)
    prod = (np.arange(16)[:, None] - 8.0) * s[None, :]
    mine = o.float_to_fp16_bits_rne(prod)
    with np.errstate(over="ignore"):
        ref = prod.astype(np.float16).view(np.uint16)
    assert np.array_equal(mine, ref)


def test_fp16_encode_halfway_and_overflow_cases():
    v = np.array([2.0 ** -25, 3 * 2.0 ** -25, 65504.0, 65519.0, 65520.0, -0.0, 1 + 2.0 ** -11,
                  1 + 3 * 2.0 ** -11, 2.0 ** -14 - 2.0 ** -25])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(o.float_to_fp16_bits_rne(v), ref)


# --------------------------------------------------------------------------- packing
def test_pack_hand_example():
    _, lines = _read_fixture("nibble_pairs.txt")
    codes = np.full((2, 64), 8, np.uint8)
    want = np.full(64, 0x88, np.uint8)
    for _, col, lo, hi, byte, off in (ln[:6] for ln in lines):
        codes[0, int(col)], codes[1, int(col)] = int(lo), int(hi)
        want[int(off)] = int(byte, 16)
    blob = o.pack(codes, np.zeros((2, 2), np.uint16), 32)
    assert np.array_equal(blob[:64], want)
    assert np.array_equal(o.unpack_codes(blob, 2, 64, 32), codes)


def test_codes_offsets_are_a_permutation_of_each_block():
    K = 256
    offs = [o.codes_byte_offset(0, k, K) for k in range(K)]
    assert sorted(offs) == list(range(K))
    for k in range(K):
        assert offs[k] // 64 == k // 64          # a column never leaves its 64-byte block
    assert o.codes_byte_offset(3, 5, K) == 3 * K + offs[5]


def test_pack_every_byte_value_round_trips():
    # N = 2, K = 256: column k carries lo = k & 15, hi = k >> 4, i.e. byte value k
    K = 256
    codes = np.stack([np.arange(K) & 15, np.arange(K) >> 4]).astype(np.uint8)
    blob = o.pack(codes, np.zeros((K // 32, 2), np.uint16), 32)
    for k in range(K):
        assert blob[o.codes_byte_offset(0, k, K)] == k
    assert sorted(blob[:K].tolist()) == list(range(256))
    assert np.array_equal(o.unpack_codes(blob, 2, K, 32), codes)


def test_pack_layout_sizes_and_trailer():
    lay = o.packed_layout(14336, 4096, 128)
    assert lay["codes_bytes"] == 14336 // 2 * 4096
    assert lay["scales_offset"] % 256 == 0 and lay["scales_offset"] >= lay["codes_bytes"]
    assert lay["trailer_offset"] % 256 == 0
    assert lay["trailer_offset"] >= lay["scales_offset"] + 2 * 32 * 14336
    assert lay["total_bytes"] == lay["trailer_offset"] + 64
    lay = o.packed_layout(6, 64, 16)     # codes 192 B -> scales at 256, 48 B -> trailer at 512
    assert (lay["scales_offset"], lay["trailer_offset"], lay["total_bytes"]) == (256, 512, 576)
    codes = np.zeros((6, 64), np.uint8)
    blob = o.pack(codes, np.ones((4, 6), np.uint16), 16)
    tw = o.trailer_words(blob, 6, 64, 16)
    assert bytes(blob[512:516]) == b"Q4GS"
    assert list(tw[:6]) == [0x53473451, 1, 6, 64, 16, 0] and not tw[6:].any()


@pytest.mark.parametrize("N,K,gs", [(2, 64, 64), (8, 64, 32), (64, 128, 32), (24, 192, 16)])
def test_pack_fast_matches_loop(N, K, gs):
    rng = np.random.default_rng(N * K)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sb = rng.integers(0, 0x7C00, (K // gs, N)).astype(np.uint16)
    blob = o.pack(codes, sb, gs)
    assert np.array_equal(o.pack_fast(codes, sb, gs), blob)
    assert np.array_equal(o.unpack_codes_fast(blob, N, K, gs), codes)
    assert np.array_equal(o.unpack_scale_bits(blob, N, K, gs), sb)


def test_pack_rejects_out_of_range_codes():
    with pytest.raises(ValueError):
        o.pack(np.full((2, 64), 16, np.uint8), np.zeros((1, 2), np.uint16), 64)


# --------------------------------------------------------------------------- dequant
def test_dequant_hand_values():
    _, lines = _read_fixture("dequant_values.txt")
    for code, sbits, val, wbits in lines:
        c = np.array([[int(code)], [8]], np.uint8)          # N = 2, K = 1 ... gs = 1
        sb = np.array([[int(sbits, 16), 0x3C00]], np.uint16)
        w32 = o.dequant_w32(c, sb, 1)
        assert w32[0, 0] == np.float32(float(val)), (code, sbits)
        assert o.dequant_w16_bits(c, sb, 1)[0, 0] == int(wbits, 16), (code, sbits)
        assert o.dequant_w16_bits_fast(c, sb, 1)[0, 0] == int(wbits, 16)
    # the zero point gives a zero with the sign of the IEEE product (+0 * s)
    c = np.full((2, 1), 8, np.uint8)
    w = o.dequant_w32(c, np.array([[0xBC00, 0x3C00]], np.uint16), 1)
    assert w[0, 0] == 0 and np.signbit(w[0, 0]) and not np.signbit(w[1, 0])
    assert list(o.dequant_w16_bits(c, np.array([[0xBC00, 0x3C00]], np.uint16), 1)[:, 0]) == [0x8000, 0]


def test_dequant_group_index_runs_along_k():
    # scale g applies to columns [g*gs, (g+1)*gs) of every row, with its own n
    N, K, gs = 4, 64, 16
    codes = np.full((N, K), 9, np.uint8)                  # (9 - 8) * s = s
    s = (np.arange(K // gs)[:, None] * 16 + np.arange(N)[None, :] + 1).astype(np.float16)
    w = o.dequant_w32(codes, bits(s), gs)
    for n in range(N):
        for k in range(K):
            assert w[n, k] == float(s[k // gs, n])


def test_dequant_fast_matches_direct():
    inp = wl.random_inputs(2, 16, 64, 16, seed=3, scales="loguniform")
    a = o.dequant_w16_bits(inp.codes, bits(inp.scales), 16)
    b = o.dequant_w16_bits_fast(inp.codes, bits(inp.scales), 16)
    assert np.array_equal(a, b)


# --------------------------------------------------------------------------- products
def test_tiny_linear_hand_example():
    rows, _ = _read_fixture("tiny_linear.txt")
    x = np.array([[float(v) for v in rows["x"]]], np.float16)
    codes = np.array([[int(v) for v in rows["codes0"]], [int(v) for v in rows["codes1"]]], np.uint8)
    s = np.array([[float(v) for v in rows["scales"]]], np.float16)
    d = np.array([[float(v) for v in rows["d_out"]]], np.float16)
    y, _ = o.linear_fwd(bits(x), codes, bits(s), 4)
    dx, _ = o.linear_bwd_input(bits(d), codes, bits(s), 4)
    assert np.array_equal(y[0], [float(v) for v in rows["y"]])
    assert np.array_equal(dx[0], [float(v) for v in rows["d_x"]])


def _frac_fp16(a16):
    return [[Fraction(float(v)) for v in row] for row in np.asarray(a16, np.float16)]


def _frac_weights(codes, s16, gs):
    N, K = codes.shape
    s = np.asarray(s16, np.float16)
    return [[(int(codes[n, k]) - 8) * Fraction(float(s[k // gs, n])) for k in range(K)] for n in range(N)]


@pytest.mark.parametrize("shape", [(1, 4, 4, 4), (4, 64, 128, 32)])
def test_products_against_exact_rationals(shape):
    M, N, K, gs = shape
    inp = wl.random_inputs(M, N, K, gs, seed=11)
    xf = _frac_fp16(inp.x)
    df = _frac_fp16(inp.d_out)
    wf = _frac_weights(inp.codes, inp.scales, gs)
    y, by = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs)
    dx, bdx = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), gs)
    for m in range(M):
        for n in range(N):
            exact = sum(xf[m][k] * wf[n][k] for k in range(K))
            babs = sum(abs(xf[m][k] * wf[n][k]) for k in range(K))
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(1, 10 ** 12) * babs
            assert abs(Fraction(float(by[m, n])) - babs) <= Fraction(1, 10 ** 12) * babs
        for k in range(K):
            exact = sum(df[m][n] * wf[n][k] for n in range(N))
            babs = sum(abs(df[m][n] * wf[n][k]) for n in range(N))
            assert abs(Fraction(float(dx[m, k])) - exact) <= Fraction(1, 10 ** 12) * babs
            assert abs(Fraction(float(bdx[m, k])) - babs) <= Fraction(1, 10 ** 12) * babs


def test_tiny_config_against_exact_rationals():
    sh = wl.tiny()[0]
    inp = wl.make_inputs(sh)
    wf = _frac_weights(inp.codes, inp.scales, sh.group_size)
    xf = _frac_fp16(inp.x)
    y, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), sh.group_size)
    for m in range(sh.M):
        for n in range(0, sh.N, 7):
            exact = sum(xf[m][k] * wf[n][k] for k in range(sh.K))
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(1, 10 ** 12) * abs(exact) + Fraction(1, 10 ** 300)


def test_integer_exact_inputs_give_exact_integers():
    inp = wl.integer_exact_inputs(3, 16, 256, 32, seed=5)
    y, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    dx, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), 32)
    # in units of 2^-6 every weight is an integer: w * 64 = (c - 8) * (s * 64)
    s64 = (inp.scales.astype(np.float64) * 64).astype(np.int64)
    x = inp.x.astype(np.int64)
    d = inp.d_out.astype(np.int64)
    c = inp.codes.astype(np.int64) - 8
    for m in range(3):
        for n in range(16):
            acc = sum(int(x[m, k]) * int(c[n, k]) * int(s64[k // 32, n]) for k in range(256))
            assert y[m, n] * 64 == acc
        for k in range(0, 256, 5):
            acc = sum(int(d[m, n]) * int(c[n, k]) * int(s64[k // 32, n]) for n in range(16))
            assert dx[m, k] * 64 == acc


def test_zero_point_codes_give_zero_outputs():
    inp = wl.random_inputs(3, 32, 64, 32, seed=7)
    codes = np.full_like(inp.codes, 8)
    y, b = o.linear_fwd(bits(inp.x), codes, bits(inp.scales), 32)
    dx, bd = o.linear_bwd_input(bits(inp.d_out), codes, bits(inp.scales), 32)
    assert not y.any() and not b.any() and not dx.any() and not bd.any()


@pytest.mark.parametrize("n0,k0", [(0, 0), (1, 31), (2, 32), (5, 63), (6, 64), (31, 127), (17, 95)])
def test_one_hot_probe_hits_one_scale(n0, k0):
    N, K, gs, M = 32, 128, 32, 2
    rng = np.random.default_rng(n0 * 1000 + k0)
    s = rng.uniform(0.5, 2.0, (K // gs, N)).astype(np.float16)
    codes = np.full((N, K), 8, np.uint8)
    codes[n0, k0] = 9
    x = np.zeros((M, K), np.float16)
    x[:, k0] = 1.0
    y, _ = o.linear_fwd(bits(x), codes, bits(s), gs)
    want = np.zeros((M, N))
    want[:, n0] = float(s[k0 // gs, n0])
    assert np.array_equal(y, want)
    d = np.zeros((M, N), np.float16)
    d[:, n0] = 1.0
    dx, _ = o.linear_bwd_input(bits(d), codes, bits(s), gs)
    want = np.zeros((M, K))
    want[:, k0] = float(s[k0 // gs, n0])
    assert np.array_equal(dx, want)


def test_scale_homogeneity_is_exact():
    inp = wl.random_inputs(4, 32, 128, 32, seed=9)
    y, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    y2, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales * np.float16(2)), 32)
    assert np.array_equal(y2, 2 * y)


def test_adjoint_identity():
    inp = wl.random_inputs(5, 48, 96, 32, seed=13)
    y, _ = o.linear_fwd(bits(inp.x), inp.codes, bits(inp.scales), 32)
    dx, _ = o.linear_bwd_input(bits(inp.d_out), inp.codes, bits(inp.scales), 32)
    lhs = float(np.sum(inp.d_out.astype(np.float64) * y))
    rhs = float(np.sum(dx * inp.x.astype(np.float64)))
    scale = float(np.sum(np.abs(inp.d_out.astype(np.float64)) @ np.abs(o.dequant_w32(inp.codes, bits(inp.scales), 32)) * np.abs(inp.x.astype(np.float64))))
    assert abs(lhs - rhs) <= 1e-12 * scale


def test_qkv_matches_column_split_of_one_product():
    Nq, Nk, Nv, K, gs = 64, 16, 16, 128, 32
    inp = wl.random_inputs(3, Nq + Nk + Nv, K, gs, seed=21)
    (yq, _), (yk, _), (yv, _) = o.qkv_fwd(bits(inp.x), inp.codes, bits(inp.scales), gs, Nq, Nk, Nv)
    # independent route: the full product over all rows, then split its columns
    x = inp.x.astype(np.float64)
    w = ((inp.codes.astype(np.float64) - 8) * np.repeat(inp.scales.astype(np.float64), gs, axis=0).T)
    y = x @ w.T
    assert np.allclose(yq, y[:, :Nq], rtol=0, atol=1e-12)
    assert np.allclose(yk, y[:, Nq:Nq + Nk], rtol=0, atol=1e-12)
    assert np.allclose(yv, y[:, Nq + Nk:], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- mutations
def _pins_pass(dq):
    """Re-run three pins against a candidate dequant function; False if any fails."""
    # hand-worked tiny example
    rows, _ = _read_fixture("tiny_linear.txt")
    x = np.array([[float(v) for v in rows["x"]]], np.float64)
    codes = np.array([[int(v) for v in rows["codes0"]], [int(v) for v in rows["codes1"]]], np.uint8)
    s = np.array([[float(v) for v in rows["scales"]]], np.float16)
    y = x @ dq(codes, bits(s), 4).astype(np.float64).T
    if not np.array_equal(y[0], [float(v) for v in rows["y"]]):
        return False
    # one-hot probes
    N, K, gs = 8, 64, 16
    s = (np.arange(K // gs)[:, None] * 8 + np.arange(N)[None, :] + 1).astype(np.float16)
    for n0, k0 in ((1, 17), (6, 40), (3, 63)):
        codes = np.full((N, K), 8, np.uint8)
        codes[n0, k0] = 9
        w = dq(codes, bits(s), gs)
        want = np.zeros((N, K), np.float32)
        want[n0, k0] = float(s[k0 // gs, n0])
        if not np.array_equal(w, want):
            return False
    # hand dequant values
    _, lines = _read_fixture("dequant_values.txt")
    for code, sbits, val, _ in lines[:3]:
        c = np.array([[int(code)], [8]], np.uint8)
        sb = np.array([[int(sbits, 16), 0x3C00]], np.uint16)
        if dq(c, sb, 1)[0, 0] != np.float32(float(val)):
            return False
    return True


def test_pins_catch_planted_mistakes():
    assert _pins_pass(o.dequant_w32)

    def wrong_zero_point(c, sb, gs):
        return o.dequant_w32(c, sb, gs) - o.fp16_bits_to_float(sb)[np.arange(c.shape[1]) // gs, :].T.astype(np.float32)

    def wrong_group_index(c, sb, gs):  # k % G instead of k // gs
        G = sb.shape[0]
        s = o.fp16_bits_to_float(sb)[np.arange(c.shape[1]) % G, :].T
        return ((c.astype(np.float64) - 8) * s).astype(np.float32)

    def transposed_scale(c, sb, gs):   # scale read as [N, G]
        flat = o.fp16_bits_to_float(sb).reshape(-1)
        N, K = c.shape
        G = K // gs
        s = np.array([[flat[(n * G + k // gs) % flat.size] for k in range(K)] for n in range(N)])
        return ((c.astype(np.float64) - 8) * s).astype(np.float32)

    def sign_flip(c, sb, gs):
        return -o.dequant_w32(c, sb, gs)

    def swapped_nibbles(c, sb, gs):    # even/odd rows exchanged
        c2 = c.copy()
        c2[0::2], c2[1::2] = c[1::2], c[0::2]
        return o.dequant_w32(c2, sb, gs)

    for bad in (wrong_zero_point, wrong_group_index, transposed_scale, sign_flip, swapped_nibbles):
        assert not _pins_pass(bad), bad.__name__


# ----------------------------------------------------------------------------- embedding rows
def _embedding_fixture():
    """N=4 rows (2 nibble pairs), K=64, gs=32: hand-chosen codes and scales."""
    codes = np.full((4, 64), 8, dtype=np.uint8)
    codes[0, :4] = [15, 0, 8, 7]
    codes[1, :4] = [1, 2, 3, 4]
    codes[2, :] = 0
    codes[3, :] = 15
    scales = np.array([[0.5, -0.25, 2.0, 1.0], [0.125, 4.0, -1.0, 0.0625]], dtype=np.float16)
    return codes, scales.view(np.uint16)


def test_embedding_hand_worked_rows():
    codes, sb = _embedding_fixture()
    out = o.embedding(codes, sb, 32, [3, 0, 2, 3, 1])
    assert out.shape == (5, 64) and out.dtype == np.float32
    # row 3: code 15 -> 7 x 1.0 in group 0, 7 x 0.0625 in group 1
    assert (out[0, :32] == 7.0).all() and (out[0, 32:] == 0.4375).all()
    assert np.array_equal(out[3], out[0])
    # row 0: (15-8) 0.5, (0-8) 0.5, (8-8) 0.5, (7-8) 0.5, then zero point
    assert out[1, :4].tolist() == [3.5, -4.0, 0.0, -0.5]
    assert (out[1, 4:] == 0.0).all()
    # row 2: code 0 -> -8 x 2.0, -8 x -1.0
    assert (out[2, :32] == -16.0).all() and (out[2, 32:] == 8.0).all()
    # row 1: (1..4 - 8) x -0.25, then 0 x -0.25 = -0.0 (IEEE) and 0 x 4.0 = +0.0
    assert out[4, :4].tolist() == [1.75, 1.5, 1.25, 1.0]
    assert np.signbit(out[4, 4:32]).all() and not np.signbit(out[4, 32:]).any()


def test_embedding_rejects_indices_out_of_range_and_allows_empty():
    codes, sb = _embedding_fixture()
    with pytest.raises(IndexError):
        o.embedding(codes, sb, 32, [4])
    with pytest.raises(IndexError):
        o.embedding(codes, sb, 32, [-1])
    assert o.embedding(codes, sb, 32, []).shape == (0, 64)


def test_embedding_is_a_row_selection_of_the_dequantised_weight():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, size=(24, 192), dtype=np.uint8)
    sb = rng.uniform(-2, 2, size=(12, 24)).astype(np.float16).view(np.uint16)
    idx = rng.integers(0, 24, size=40)
    assert np.array_equal(o.embedding(codes, sb, 16, idx), o.dequant_w32(codes, sb, 16)[idx])


def test_embedding_planted_mistakes_fail_the_fixture():
    codes, sb = _embedding_fixture()
    idx = np.array([3, 0, 2, 3, 1])
    good = o.embedding(codes, sb, 32, idx)
    s = o.fp16_bits_to_float(sb)
    g = np.arange(64) // 32
    # scale taken from the token position instead of the gathered row
    wrong_col = ((codes[idx].astype(np.int64) - 8) * s[g][:, np.arange(5) % 4].T).astype(np.float32)
    assert not np.array_equal(wrong_col, good)
    # odd rows read from the low nibble of the pair (rows 2p and 2p+1 swapped)
    swapped = o.embedding(codes, sb, 32, idx ^ 1)
    assert not np.array_equal(swapped, good)
