"""Pins for the oracle of the two variants (fp32 scales, frozen-base adapter).

Each is checked against something other than itself:
* binary32 decode and the definition-based binary32 encoder against numpy's
  float32 type, on every exponent and on constructed ties;
* the fp32-scale dequantisation against hand-worked values
  (tests/golden/dequant_f32s_values.txt: ties, overflow, subnormals, a double
  rounding) and against the definition-based encoder;
* layout version 2 against hand-computed offsets and bytes;
* the products against exact rational arithmetic, exact integers and closed
  forms (zero adapter, rank-1 adapter, adjoint identity);
* planted mistakes fail at least one pin.
"""
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle as o
from oracle import q4gsw_variants as v
from bit_group_quantized_q4gsw_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits16(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def bits32(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def f32_of_bits(b):
    return struct.unpack("<f", struct.pack("<I", int(b)))[0]


# --------------------------------------------------------------------------- binary32
def test_fp32_decode_matches_numpy_on_every_exponent():
    rng = np.random.default_rng(1)
    exps = np.repeat(np.arange(256, dtype=np.uint32), 64)
    fracs = rng.integers(0, 1 << 23, exps.size, dtype=np.uint32)
    fracs[::64] = 0
    fracs[1::64] = 1
    fracs[2::64] = (1 << 23) - 1
    b = np.concatenate([(exps << 23) | fracs, ((exps << 23) | fracs) | np.uint32(0x80000000)])
    mine = v.fp32_bits_to_float(b)
    with np.errstate(invalid="ignore"):
        ref = b.view(np.float32).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.signbit(v.fp32_bits_to_float(np.uint32(0x80000000)))


def test_fp32_encoder_matches_numpy_on_dequant_products():
    # (code - 8) * s32 for random fp32 scales of every exponent, subnormals included
    rng = np.random.default_rng(2)
    exps = rng.integers(0, 255, 20000, dtype=np.uint32)
    sb = (exps << 23) | rng.integers(0, 1 << 23, exps.size, dtype=np.uint32)
    s = sb.view(np.float32).astype(np.float64)
    for c in range(16):
        prod = (c - 8) * s
        mine = np.array([v.encode_fp32_rne(float(p)) for p in prod], dtype=np.uint32)
        with np.errstate(over="ignore"):
            ref = prod.astype(np.float32).view(np.uint32)
        assert np.array_equal(mine, ref), c


def test_fp32_encoder_ties_go_to_even():
    ulp = 2.0 ** -23
    assert v.encode_fp32_rne(1 + 0.5 * ulp) == 0x3F800000          # tie, even below
    assert v.encode_fp32_rne(1 + 1.5 * ulp) == 0x3F800002          # tie, even above
    assert v.encode_fp32_rne(1 + 0.5 * ulp + 2.0 ** -50) == 0x3F800001   # just above the tie
    assert v.encode_fp32_rne(2.0 ** -150) == 0                     # half the smallest subnormal: to even (0)
    assert v.encode_fp32_rne(3 * 2.0 ** -150) == 2                 # 1.5 quanta: to even (2)
    assert v.encode_fp32_rne(-(2.0 ** 128)) == 0xFF800000
    assert v.encode_fp32_rne((2 - ulp / 2) * 2.0 ** 127) == 0x7F800000   # rounds up past FLT_MAX
    assert v.encode_fp32_rne(-0.0) == 0x80000000


# --------------------------------------------------------------------------- dequant with fp32 scales
def _f32s_fixture():
    rows = []
    for line in open(os.path.join(GOLDEN, "dequant_f32s_values.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            c, sb, exact, w32, w16 = line.split()
            rows.append((int(c), int(sb, 16), float.fromhex(exact) if "p+130" not in exact else None,
                         int(w32, 16), int(w16, 16)))
    return rows


def test_f32s_dequant_hand_values():
    for c, sb, _, w32, w16 in _f32s_fixture():
        codes = np.array([[c], [8]], np.uint8)
        s = np.array([[sb, 0x3F800000]], np.uint32)
        got32 = v.dequant_w32_f32s(codes, s, 1)[0, 0]
        assert int(np.float32(got32).view(np.uint32)) == w32, (c, hex(sb))
        got16 = v.dequant_w16_bits_f32s(codes, s, 1)[0, 0]
        assert int(got16) == w16, (c, hex(sb))
        # the encoder written from the definition gives the same w32 from the exact product
        # (an integer times a 24-bit significand is exact in a double, signed zeros included)
        exact = (c - 8) * f32_of_bits(sb)
        assert v.encode_fp32_rne(exact) == w32


def test_f32s_double_rounding_case_takes_the_fp32_product():
    # exact product lies just above an fp16 tie; fp32 rounding lands on the tie
    codes = np.array([[11], [8]], np.uint8)
    s = np.array([[0x3EAB6AAB, 0x3F800000]], np.uint32)
    exact = 3 * Fraction(f32_of_bits(0x3EAB6AAB))
    assert exact == 1 + Fraction(9, 2 ** 11) + Fraction(1, 2 ** 25)
    assert int(v.dequant_w16_bits_f32s(codes, s, 1)[0, 0]) == 0x3C04
    assert int(o.float_to_fp16_bits_rne(np.array([float(exact)]))[0]) == 0x3C05


def test_f32s_dequant_matches_definition_encoder_and_fast_form():
    rng = np.random.default_rng(3)
    N, K, gs = 8, 128, 32
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s = bits32(rng.uniform(-2, 2, (K // gs, N)) * np.exp(rng.uniform(-30, 30, (K // gs, N))))
    w = v.dequant_w32_f32s(codes, s, gs)
    sf = v.fp32_bits_to_float(s)
    for n in range(N):
        for k in range(K):
            want = v.encode_fp32_rne((int(codes[n, k]) - 8) * float(sf[k // gs, n]))
            assert int(np.float32(w[n, k]).view(np.uint32)) == want
    assert np.array_equal(v.dequant_w16_bits_f32s(codes, s, gs), v.dequant_w16_bits_f32s_fast(codes, s, gs))


def test_f32s_group_index_runs_along_k():
    N, K, gs = 4, 64, 16
    codes = np.full((N, K), 9, np.uint8)
    s = bits32((np.arange(K // gs)[:, None] * 10 + np.arange(N)[None, :] + 1).astype(np.float32))
    w = v.dequant_w32_f32s(codes, s, gs)
    for n in range(N):
        for k in range(K):
            assert w[n, k] == (k // gs) * 10 + n + 1


# --------------------------------------------------------------------------- layout version 2
def test_layout_v2_offsets_by_hand():
    # N=8, K=64, gs=16: codes 4*64 = 256 B; scales at 256, 4 groups x 8 x 4 B = 128 B;
    # trailer at round_up(384, 256) = 512; total 576
    lay = v.packed_layout_f32s(8, 64, 16)
    assert (lay["codes_bytes"], lay["scales_offset"], lay["scales_bytes"], lay["trailer_offset"],
            lay["total_bytes"]) == (256, 256, 128, 512, 576)
    codes = np.full((8, 64), 8, np.uint8)
    codes[2, 1] = 3          # pair 1, column 1 -> byte slot 2 of word slot 0 (k % 64 = 1: i=0, t=0, e=1)
    codes[3, 1] = 12
    s = np.zeros((4, 8), np.uint32)
    s[2, 5] = 0x3F800001     # group 2, column 5 -> bytes at 256 + 4 * (2 * 8 + 5) = 340
    blob = v.pack_f32s(codes, s, 16)
    assert blob[64 + 2] == 3 | (12 << 4)
    assert list(blob[340:344]) == [0x01, 0x00, 0x80, 0x3F]
    words = blob[512:].view("<u4")
    assert list(words[:6]) == [0x53473451, 2, 8, 64, 16, 0] and not words[6:].any()
    assert np.array_equal(v.unpack_scale_bits_f32s(blob, 8, 64, 16), s)
    assert np.array_equal(o.unpack_codes_fast(blob, 8, 64, 16), codes)


# --------------------------------------------------------------------------- fp32-scale products
def _frac32(sb):
    return np.vectorize(lambda b: Fraction(f32_of_bits(b)), otypes=[object])(sb)


def test_f32s_products_against_exact_rationals():
    M, N, K, gs = 2, 8, 64, 16
    rng = np.random.default_rng(4)
    x = rng.standard_normal((M, K)).astype(np.float16)
    d = rng.standard_normal((M, N)).astype(np.float16)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s = bits32(rng.uniform(0.001, 0.05, (K // gs, N)))
    sf = _frac32(s)
    # w32 formed from the exact product and rounded by the definition-based encoder
    wf = [[Fraction(f32_of_bits(v.encode_fp32_rne(float((int(codes[n, k]) - 8) * sf[k // gs, n]))))
           for k in range(K)] for n in range(N)]
    xf = [[Fraction(float(a)) for a in row] for row in x]
    df = [[Fraction(float(a)) for a in row] for row in d]
    y, by = v.linear_fwd_f32s(bits16(x), codes, s, gs)
    dx, bdx = v.linear_bwd_input_f32s(bits16(d), codes, s, gs)
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


def test_f32s_with_fp16_representable_scales_equals_fp16_path():
    # an fp32 scale that is exactly an fp16 value gives the version-1 weight exactly
    inp = wl.random_inputs(3, 16, 128, 32, seed=5)
    s32 = bits32(inp.scales.astype(np.float32))
    assert np.array_equal(v.dequant_w32_f32s(inp.codes, s32, 32), o.dequant_w32(inp.codes, bits16(inp.scales), 32))
    y1, _ = o.linear_fwd(bits16(inp.x), inp.codes, bits16(inp.scales), 32)
    y2, _ = v.linear_fwd_f32s(bits16(inp.x), inp.codes, s32, 32)
    assert np.array_equal(y1, y2)


def test_f32s_adjoint_identity_and_qkv_split():
    inp = wl.random_inputs(4, 48, 128, 32, seed=6)
    s32 = bits32(np.random.default_rng(6).uniform(0.005, 0.02, (4, 48)))
    y, _ = v.linear_fwd_f32s(bits16(inp.x), inp.codes, s32, 32)
    dx, _ = v.linear_bwd_input_f32s(bits16(inp.d_out), inp.codes, s32, 32)
    lhs = float(np.sum(inp.d_out.astype(np.float64) * y))
    rhs = float(np.sum(dx * inp.x.astype(np.float64)))
    w = np.abs(v.dequant_w32_f32s(inp.codes, s32, 32).astype(np.float64))
    assert abs(lhs - rhs) <= 1e-12 * float(np.sum((np.abs(inp.d_out.astype(np.float64)) @ w) * np.abs(inp.x)))
    parts = v.qkv_fwd_f32s(bits16(inp.x), inp.codes, s32, 32, 32, 8, 8)
    assert np.allclose(np.concatenate([p[0] for p in parts], axis=1), y, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- adapter
def _adapter_inputs(M, N, K, r, seed):
    rng = np.random.default_rng(seed)
    inp = wl.random_inputs(M, N, K, 32, seed=seed)
    A = (rng.standard_normal((r, K)) * 0.05).astype(np.float16)
    B = (rng.standard_normal((N, r)) * 0.05).astype(np.float16)
    return inp, A, B


def test_adapter_against_exact_rationals():
    M, N, K, r = 2, 8, 64, 3
    inp, A, B = _adapter_inputs(M, N, K, r, 7)
    fr = lambda a: [[Fraction(float(t)) for t in row] for row in a]
    xf, Af, Bf, df = fr(inp.x), fr(A), fr(B), fr(inp.d_out)
    s = inp.scales
    wf = [[(int(inp.codes[n, k]) - 8) * Fraction(float(s[k // 32, n])) for k in range(K)] for n in range(N)]
    y, by = v.adapter_fwd(bits16(inp.x), inp.codes, bits16(s), 32, bits16(A), bits16(B))
    dx, bdx = v.adapter_bwd_input(bits16(inp.d_out), inp.codes, bits16(s), 32, bits16(A), bits16(B))
    for m in range(M):
        u = [sum(xf[m][k] * Af[j][k] for k in range(K)) for j in range(r)]
        ua = [sum(abs(xf[m][k] * Af[j][k]) for k in range(K)) for j in range(r)]
        for n in range(N):
            exact = sum(xf[m][k] * wf[n][k] for k in range(K)) + sum(u[j] * Bf[n][j] for j in range(r))
            babs = sum(abs(xf[m][k] * wf[n][k]) for k in range(K)) + sum(ua[j] * abs(Bf[n][j]) for j in range(r))
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(1, 10 ** 12) * babs
            assert abs(Fraction(float(by[m, n])) - babs) <= Fraction(1, 10 ** 12) * babs
        vv = [sum(df[m][n] * Bf[n][j] for n in range(N)) for j in range(r)]
        for k in range(K):
            exact = sum(df[m][n] * wf[n][k] for n in range(N)) + sum(vv[j] * Af[j][k] for j in range(r))
            babs = sum(abs(df[m][n] * wf[n][k]) for n in range(N)) + \
                sum(sum(abs(df[m][n] * Bf[n][j]) for n in range(N)) * abs(Af[j][k]) for j in range(r))
            assert abs(Fraction(float(dx[m, k])) - exact) <= Fraction(1, 10 ** 12) * babs
            assert abs(Fraction(float(bdx[m, k])) - babs) <= Fraction(1, 10 ** 12) * babs


def test_zero_adapter_is_the_base_layer():
    inp, A, B = _adapter_inputs(3, 16, 128, 4, 8)
    y0, b0 = o.linear_fwd(bits16(inp.x), inp.codes, bits16(inp.scales), 32)
    for a, b in ((np.zeros_like(A), B), (A, np.zeros_like(B))):
        y, by = v.adapter_fwd(bits16(inp.x), inp.codes, bits16(inp.scales), 32, bits16(a), bits16(b))
        assert np.array_equal(y, y0)
    d0, _ = o.linear_bwd_input(bits16(inp.d_out), inp.codes, bits16(inp.scales), 32)
    dx, _ = v.adapter_bwd_input(bits16(inp.d_out), inp.codes, bits16(inp.scales), 32, bits16(A), bits16(np.zeros_like(B)))
    assert np.array_equal(dx, d0)


def test_rank_one_adapter_with_integers_is_an_exact_outer_product():
    # codes all 8 (zero base); x, a, b small integers: y[m, n] = (x[m] . a) b[n] exactly
    M, N, K = 3, 8, 64
    rng = np.random.default_rng(9)
    x = rng.integers(-2, 3, (M, K)).astype(np.float16)
    a = rng.integers(-2, 3, (1, K)).astype(np.float16)
    b = rng.integers(-2, 3, (N, 1)).astype(np.float16)
    codes = np.full((N, K), 8, np.uint8)
    s = np.ones((K // 32, N), np.float16)
    y, _ = v.adapter_fwd(bits16(x), codes, bits16(s), 32, bits16(a), bits16(b))
    xi, ai, bi = x.astype(np.int64), a.astype(np.int64), b.astype(np.int64)
    for m in range(M):
        dot = int(sum(int(xi[m, k]) * int(ai[0, k]) for k in range(K)))
        for n in range(N):
            assert y[m, n] == dot * int(bi[n, 0])
    d = rng.integers(-2, 3, (M, N)).astype(np.float16)
    dx, _ = v.adapter_bwd_input(bits16(d), codes, bits16(s), 32, bits16(a), bits16(b))
    di = d.astype(np.int64)
    for m in range(M):
        dot = int(sum(int(di[m, n]) * int(bi[n, 0]) for n in range(N)))
        for k in range(K):
            assert dx[m, k] == dot * int(ai[0, k])


def test_adapter_adjoint_identity():
    inp, A, B = _adapter_inputs(4, 32, 128, 8, 10)
    y, _ = v.adapter_fwd(bits16(inp.x), inp.codes, bits16(inp.scales), 32, bits16(A), bits16(B))
    dx, _ = v.adapter_bwd_input(bits16(inp.d_out), inp.codes, bits16(inp.scales), 32, bits16(A), bits16(B))
    lhs = float(np.sum(inp.d_out.astype(np.float64) * y))
    rhs = float(np.sum(dx * inp.x.astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + float(np.sum(np.abs(y))) + 1.0)


def test_adapter_planted_mistakes_fail_a_pin():
    inp, A, B = _adapter_inputs(2, 8, 64, 3, 11)

    def transposed_product(xb, c, sb, gs, ab, bb):      # (x B) A instead of (x A^T) B^T, shapes forced square
        y0, b0 = o.linear_fwd(xb, c, sb, gs)
        x = o.fp16_bits_to_float(xb)
        Af = o.fp16_bits_to_float(ab)
        Bf = o.fp16_bits_to_float(bb)
        return y0 + (x @ Af.T) @ Bf[::-1].T, b0

    def dropped_adapter(xb, c, sb, gs, ab, bb):
        return o.linear_fwd(xb, c, sb, gs)

    def sign_flip(xb, c, sb, gs, ab, bb):
        y, b = v.adapter_fwd(xb, c, sb, gs, ab, bb)
        y0, _ = o.linear_fwd(xb, c, sb, gs)
        return 2 * y0 - y, b

    def pin_ok(fn):
        # the exact-rational pin on one element per output row
        M, N, K, r = 2, 8, 64, 3
        xf = [[Fraction(float(t)) for t in row] for row in inp.x]
        Af = [[Fraction(float(t)) for t in row] for row in A]
        Bf = [[Fraction(float(t)) for t in row] for row in B]
        s = inp.scales
        y, _ = fn(bits16(inp.x), inp.codes, bits16(s), 32, bits16(A), bits16(B))
        for m in range(M):
            for n in (0, 5):
                base = sum(xf[m][k] * (int(inp.codes[n, k]) - 8) * Fraction(float(s[k // 32, n])) for k in range(K))
                ad = sum(sum(xf[m][k] * Af[j][k] for k in range(K)) * Bf[n][j] for j in range(r))
                if abs(Fraction(float(y[m, n])) - (base + ad)) > Fraction(1, 10 ** 9) * (abs(base) + abs(ad) + 1):
                    return False
        return True

    assert pin_ok(v.adapter_fwd)
    for bad in (transposed_product, dropped_adapter, sign_flip):
        assert not pin_ok(bad), bad.__name__


# --------------------------------------------------------------------------- dq8ca
def _dq8ca_fixture():
    rows = []
    for line in open(os.path.join(GOLDEN, "dq8ca_rows.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            name, sb, z, *pairs = line.split()
            xs = [float(p.split(":")[0]) for p in pairs]
            qs = [int(p.split(":")[1]) for p in pairs]
            rows.append((name, int(sb, 16), int(z), xs, qs))
    return rows


def test_dq8ca_quantisation_hand_rows():
    for name, sb, z, xs, qs in _dq8ca_fixture():
        x = np.array([xs], np.float16)
        q, a_s, a_z = v.dq8ca_quantize(bits16(x))
        assert int(np.float32(a_s[0]).view(np.uint32)) == sb, name
        assert int(a_z[0]) == z, name
        assert list(q[0].astype(int)) == qs, name


def test_dq8ca_quantisation_properties():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float16)
    x[3] = np.abs(x[3])          # one-signed rows: the range still holds 0
    x[4] = -np.abs(x[4])
    q, a_s, a_z = v.dq8ca_quantize(bits16(x))
    xf = x.astype(np.float64)
    assert q.min() >= -128 and q.max() <= 127
    back = (q.astype(np.float64) - a_z[:, None]) * a_s[:, None].astype(np.float64)
    # every value within half a step (plus the float32 rounding of x / a_s)
    assert (np.abs(back - xf) <= a_s[:, None] * (0.5 + 1e-5)).all()
    # zero is represented exactly: (q - a_z) == 0 where x == 0
    x0 = x.copy()
    x0[:, :8] = 0
    q0, _, z0 = v.dq8ca_quantize(bits16(x0))
    assert (q0[:, :8].astype(int) == z0[:, None]).all()


def test_dq8ca_equals_the_base_product_when_quantisation_is_exact():
    # integer activations spanning exactly [-100, 155]: a_s = 1, q - a_z = x
    rng = np.random.default_rng(13)
    M, N, K, gs = 4, 16, 128, 32
    x = rng.integers(-100, 156, (M, K)).astype(np.float16)
    x[:, 0], x[:, 1] = -100, 155
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    s = np.ldexp(1.0, rng.integers(-6, -2, (K // gs, N))).astype(np.float16)
    y8, _ = v.linear_dq8ca_fwd(bits16(x), codes, bits16(s), gs)
    y, _ = o.linear_fwd(bits16(x), codes, bits16(s), gs)
    assert np.array_equal(y8, y)


def test_dq8ca_product_against_exact_rationals():
    M, N, K, gs = 2, 8, 64, 32
    inp = wl.random_inputs(M, N, K, gs, seed=14)
    q, a_s, a_z = v.dq8ca_quantize(bits16(inp.x))
    y, b = v.linear_dq8ca_fwd(bits16(inp.x), inp.codes, bits16(inp.scales), gs)
    for m in range(M):
        for n in range(N):
            exact = Fraction(0)
            babs = Fraction(0)
            for g in range(K // gs):
                t = sum((int(q[m, k]) - int(a_z[m])) * (int(inp.codes[n, k]) - 8) for k in range(g * gs, (g + 1) * gs))
                ta = sum(abs((int(q[m, k]) - int(a_z[m])) * (int(inp.codes[n, k]) - 8))
                         for k in range(g * gs, (g + 1) * gs))
                exact += t * Fraction(float(inp.scales[g, n]))
                babs += ta * abs(Fraction(float(inp.scales[g, n])))
            exact *= Fraction(float(a_s[m]))
            babs *= Fraction(float(a_s[m]))
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(1, 10 ** 12) * babs
            assert abs(Fraction(float(b[m, n])) - babs) <= Fraction(1, 10 ** 12) * babs


def test_dq8ca_planted_mistakes_fail_the_fixture():
    def run(fn):
        for name, sb, z, xs, qs in _dq8ca_fixture():
            q, a_s, a_z = fn(bits16(np.array([xs], np.float16)))
            if list(q[0].astype(int)) != qs or int(a_z[0]) != z:
                return False
        return True

    def wrong_zero_point_sign(xb):
        q, s, z = v.dq8ca_quantize(xb)
        return np.clip(q.astype(int) - 2 * z[:, None], -128, 127).astype(np.int8), s, -z

    def rounds_half_away(xb):   # round-half-away-from-zero instead of to even
        x = o.fp16_bits_to_float(xb).astype(np.float32)
        q, s, z = v.dq8ca_quantize(xb)
        r = np.sign(x / s[:, None]) * np.floor(np.abs(x / s[:, None]) + 0.5)
        return np.clip(r + z[:, None], -128, 127).astype(np.int8), s, z

    def symmetric_range(xb):    # max |x| / 127, no zero point
        x = o.fp16_bits_to_float(xb).astype(np.float32)
        s = np.abs(x).max(axis=1) / np.float32(127)
        s = np.where(s == 0, np.float32(1), s).astype(np.float32)
        return np.clip(np.rint(x / s[:, None]), -128, 127).astype(np.int8), s, np.zeros(x.shape[0], np.int32)

    assert run(v.dq8ca_quantize)
    for bad in (wrong_zero_point_sign, rounds_half_away, symmetric_range):
        assert not run(bad), bad.__name__
