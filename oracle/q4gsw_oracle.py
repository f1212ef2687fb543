"""Plain CPU oracle for the q4gsw 4-bit group-symmetric weight-quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
this module.  The CUDA library never imports it and it never imports the CUDA
library: the two share no code, no tables and no helpers.

What it computes, and where each definition comes from
------------------------------------------------------
Sources are three web pages:

* [P2] "[ExecuTorch][Vulkan] Add et_vk.linear_q4gsw_backward kernel (4-bit
  input-grad)" (pytorch/executorch pull request #20943), PR description:
  - the input gradient  d_x[M, K] = d_out[M, N] @ dequant(W)[N, K], a sum over N;
  - the dequantisation  dequant(W[n, k]) = (code - 8) * scale;
  - "Key changes": codes are nibbles with the even-N element in the low nibble
    and the odd-N element in the high nibble, and the scales are a
    [num_groups, N] tensor; "Constraints": N, K and group_size are multiples
    of 4; the kernel works in fp32.
* [P3] "[ExecuTorch][WebGPU] Replace broad QKV fusion with BK64 kernel"
  (pytorch/executorch pull request #21650), description of the stacked #21131:
  the Q/K/V projection triple is fused, the constant weights and scales are
  packed once, and the result goes to three distinct outputs.
* [P1] "Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork"
  (software-mansion/react-native-executorch issue #1361), comment of
  Oct 20, 2026: weight scales are kept in fp16.

Readings taken where the pages are silent (each is listed with its reason in
the design notes of the repository):

* groups run along K: scale index g = floor(k / group_size), K % group_size == 0;
* the forward is y[M, N] = x[M, K] @ dequant(W)[N, K]^T (the per-projection GEMM
  that the backward mirrors);
* the order of the bytes inside a pair row, the position of the scales and
  the trailer of the packed blob (``packed_layout``) are this library's own
  layout, not the Vulkan W_4X8 block order, which the pages do not spell out;
  it needs K % 64 == 0;
* a GPU tensor-core operand is the fp16 value fp16_RNE((code - 8) * scale): one
  correctly rounded product.  ``dequant_w16_bits`` gives it;
* all outputs are fp32 on the GPU; here they are fp64 sums of exact fp32
  weights (``dequant_w32``), with the per-element bound sum |a| |w| beside them.

Every function below is a direct restatement of its definition: loops or one
library primitive (a numpy matmul, ``round``, ``math.frexp``), no blocking and
no reordering.
"""
from __future__ import annotations

import math

import numpy as np

ZERO_POINT = 8          # [P2] dequant(W[n, k]) = (code - 8) * scale
CODE_MAX = 15           # 4-bit codes
LAYOUT_VERSION = 1
REGION_ALIGN = 256      # byte alignment of the scales region and the trailer
TRAILER_BYTES = 64
TRAILER_MAGIC = 0x53473451   # bytes "Q4GS"

# Own-layout choices for the codes region (version 1), see ``packed_layout``:
# inside each 64-byte block of a pair row, word slot w (4 bytes) holds the
# columns 16*(w % 4) + 4*(w // 4) + 0..3, and inside a word the byte slots
# 0, 1, 2, 3 hold the columns +0, +2, +1, +3.
_SLOT_OF_K_MOD4 = (0, 2, 1, 3)


# ----------------------------------------------------------------------------
# fp16 <-> real, written from the IEEE 754 binary16 definition
# (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits).
# ----------------------------------------------------------------------------
def fp16_bits_to_float(bits) -> np.ndarray:
    """Decode binary16 bit patterns (uint16) to float64 exactly.

    normal:    (-1)^s * 2^(e-15) * (1 + f/1024)   for 1 <= e <= 30
    subnormal: (-1)^s * 2^(-14)  * (f/1024)       for e == 0
    e == 31:   +-inf (f == 0) or NaN.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    e = (b >> 10) & 0x1F
    f = (b & 0x3FF).astype(np.float64)
    normal = sign * np.ldexp(1.0 + f / 1024.0, (e - 15).astype(np.int64))
    sub = sign * np.ldexp(f / 1024.0, -14)
    out = np.where(e == 0, sub, normal)
    out = np.where((e == 31) & (f == 0), sign * np.inf, out)
    out = np.where((e == 31) & (f != 0), np.nan, out)
    return out


def float_to_fp16_bits_rne(v) -> np.ndarray:
    """Round real values (float64, exact inputs) to binary16, ties to even.

    For |v| in [2^e, 2^(e+1)) with e >= -14 the spacing of binary16 values is
    2^(e-10); below 2^-14 the spacing is the subnormal quantum 2^-24.  The value
    is divided by its spacing (exact, a power of two), rounded half-to-even with
    Python's ``round`` and re-assembled; a significand that rounds up to 2048 carries
    into the exponent, and magnitudes that round to 2^16 or more become inf.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.uint16)
    flat_v = v.reshape(-1)
    flat_o = out.reshape(-1)
    for i in range(flat_v.size):
        flat_o[i] = _encode_one(float(flat_v[i]))
    return out


def _encode_one(x: float) -> int:
    if x != x:
        return 0x7E00
    s = 0x8000 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a == 0:
        return s
    if a == math.inf:
        return s | 0x7C00
    _, e2 = math.frexp(a)        # a = m * 2^e2, m in [0.5, 1)  ->  floor(log2 a) = e2 - 1
    e = e2 - 1
    if e < -14:                  # subnormal range: quantum 2^-24
        q = round(math.ldexp(a, 24))          # Python round(): half to even
        if q >= 1024:            # rounded up into the smallest normal
            return s | (1 << 10)
        return s | q
    q = round(math.ldexp(a, 10 - e))          # in [1024, 2048]
    if q == 2048:
        q = 1024
        e += 1
    if e > 15:
        return s | 0x7C00
    return s | ((e + 15) << 10) | (q - 1024)


# ----------------------------------------------------------------------------
# The packed blob (layout version 1)
# ----------------------------------------------------------------------------
def packed_layout(N: int, K: int, group_size: int) -> dict:
    """Byte map of one packed weight (layout version 1).

    codes region, offset 0, N/2 * K bytes.  The byte of (pair p, column k) holds
      code[2p, k] in bits 0..3 and code[2p+1, k] in bits 4..7   ([P2] nibble rule)
    and sits at ``codescodes_byte_offset(p, k, K)``: row p of K bytes, cut into
    64-byte blocks (K % 64 == 0); in a block, column r = 16 i + 4 t + e
    (i, t, e in 0..3) is in word slot 4 t + i, byte slot (0, 2, 1, 3)[e].
    scales region, offset round_up(N/2*K, 256): fp16 [G][N] row-major, G = K/gs
    ([P2] "[num_groups, N] scales"; fp16 per [P1]).
    trailer, offset round_up(scales end, 256), 64 bytes of little-endian u32:
    magic "Q4GS", layout version, N, K, group_size, range flag (1 if a code
    exceeded 15 at packing time, else 0), then zeros.
    """
    G = K // group_size
    codes_bytes = (N // 2) * K
    scales_offset = -(-codes_bytes // REGION_ALIGN) * REGION_ALIGN
    scales_bytes = 2 * G * N
    trailer_offset = -(-(scales_offset + scales_bytes) // REGION_ALIGN) * REGION_ALIGN
    return {
        "G": G,
        "codes_offset": 0,
        "codes_bytes": codes_bytes,
        "scales_offset": scales_offset,
        "scales_bytes": scales_bytes,
        "trailer_offset": trailer_offset,
        "total_bytes": trailer_offset + TRAILER_BYTES,
    }


def codes_byte_offset(p: int, k: int, K: int) -> int:
    r = k % 64
    i, t, e = r // 16, (r % 16) // 4, r % 4
    return p * K + 64 * (k // 64) + 4 * (4 * t + i) + _SLOT_OF_K_MOD4[e]


def _trailer(N: int, K: int, group_size: int, range_flag: int) -> np.ndarray:
    words = np.zeros(TRAILER_BYTES // 4, dtype="<u4")
    words[:6] = (TRAILER_MAGIC, LAYOUT_VERSION, N, K, group_size, range_flag)
    return words.view(np.uint8)


def pack(codes: np.ndarray, scale_bits: np.ndarray, group_size: int) -> np.ndarray:
    """codes uint8 [N, K] in 0..15 and fp16 scale bits uint16 [G, N] -> uint8 blob."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    lay = packed_layout(N, K, group_size)
    if codes.max(initial=0) > CODE_MAX:
        raise ValueError("code out of range")
    blob = np.zeros(lay["total_bytes"], dtype=np.uint8)
    for p in range(N // 2):
        for k in range(K):
            lo = int(codes[2 * p, k])
            hi = int(codes[2 * p + 1, k])
            blob[codes_byte_offset(p, k, K)] = lo | (hi << 4)
    sb = np.ascontiguousarray(np.asarray(scale_bits, dtype=np.uint16))
    assert sb.shape == (lay["G"], N)
    blob[lay["scales_offset"]:lay["scales_offset"] + lay["scales_bytes"]] = sb.view(np.uint8).reshape(-1)
    blob[lay["trailer_offset"]:] = _trailer(N, K, group_size, 0)
    return blob


def unpack_codes(blob: np.ndarray, N: int, K: int, group_size: int) -> np.ndarray:
    """Inverse of ``pack`` on the codes region: uint8 [N, K]."""
    blob = np.asarray(blob, dtype=np.uint8)
    codes = np.zeros((N, K), dtype=np.uint8)
    for p in range(N // 2):
        for k in range(K):
            b = int(blob[codes_byte_offset(p, k, K)])
            codes[2 * p, k] = b & 0xF
            codes[2 * p + 1, k] = b >> 4
    return codes


def unpack_scale_bits(blob: np.ndarray, N: int, K: int, group_size: int) -> np.ndarray:
    lay = packed_layout(N, K, group_size)
    raw = np.ascontiguousarray(np.asarray(blob, dtype=np.uint8)[lay["scales_offset"]:lay["scales_offset"] + lay["scales_bytes"]])
    return raw.view(np.uint16).reshape(lay["G"], N).copy()


# Vectorised versions of the two loops above, for the large configurations.
# They compute the same byte map; the tests check them against the loops.
def _codes_offset_table(K: int) -> np.ndarray:
    """offset of column k inside its pair row, for k in [0, K)."""
    return np.array([codes_byte_offset(0, k, K) for k in range(K)], dtype=np.int64)


def pack_fast(codes: np.ndarray, scale_bits: np.ndarray, group_size: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    lay = packed_layout(N, K, group_size)
    if codes.max(initial=0) > CODE_MAX:
        raise ValueError("code out of range")
    byte_pk = (codes[0::2, :] | (codes[1::2, :] << 4)).astype(np.uint8)   # [N/2, K]
    rows = np.zeros((N // 2, K), dtype=np.uint8)
    rows[:, _codes_offset_table(K)] = byte_pk
    blob = np.zeros(lay["total_bytes"], dtype=np.uint8)
    blob[:lay["codes_bytes"]] = rows.reshape(-1)
    sb = np.ascontiguousarray(np.asarray(scale_bits, dtype=np.uint16))
    assert sb.shape == (lay["G"], N)
    blob[lay["scales_offset"]:lay["scales_offset"] + lay["scales_bytes"]] = sb.view(np.uint8).reshape(-1)
    blob[lay["trailer_offset"]:] = _trailer(N, K, group_size, 0)
    return blob


def unpack_codes_fast(blob: np.ndarray, N: int, K: int, group_size: int) -> np.ndarray:
    lay = packed_layout(N, K, group_size)
    rows = np.asarray(blob, dtype=np.uint8)[:lay["codes_bytes"]].reshape(N // 2, K)
    byte_pk = rows[:, _codes_offset_table(K)]
    codes = np.empty((N, K), dtype=np.uint8)
    codes[0::2] = byte_pk & 0xF
    codes[1::2] = byte_pk >> 4
    return codes


def trailer_words(blob: np.ndarray, N: int, K: int, group_size: int) -> np.ndarray:
    lay = packed_layout(N, K, group_size)
    return np.ascontiguousarray(np.asarray(blob, np.uint8)[lay["trailer_offset"]:]).view("<u4").copy()


# ----------------------------------------------------------------------------
# Dequantisation  [P2]: dequant(W[n, k]) = (code[n, k] - 8) * scale[k // gs, n]
# ----------------------------------------------------------------------------
def dequant_w32(codes: np.ndarray, scale_bits: np.ndarray, group_size: int) -> np.ndarray:
    """Exact dequantised weight as float32 [N, K].

    (code - 8) is an integer of magnitude <= 8 and the fp16 scale has an 11-bit
    significand, so the product has at most 15 significant bits and is exact in
    float32 (barring overflow beyond float32, impossible for fp16 scales).
    """
    codes = np.asarray(codes, dtype=np.int64)
    N, K = codes.shape
    s = fp16_bits_to_float(scale_bits)                  # [G, N] float64
    g_of_k = np.arange(K) // group_size                 # group index along K
    s_nk = s[g_of_k, :].T                               # s[k // gs, n] -> [N, K]
    w = (codes - ZERO_POINT).astype(np.float64) * s_nk  # exact in float64
    return w.astype(np.float32)                         # exact in float32


def dequant_w16_bits(codes: np.ndarray, scale_bits: np.ndarray, group_size: int) -> np.ndarray:
    """fp16 operand bits: binary16 round-to-nearest-even of the exact product."""
    w = dequant_w32(codes, scale_bits, group_size).astype(np.float64)
    return float_to_fp16_bits_rne(w)


def dequant_w16_bits_fast(codes: np.ndarray, scale_bits: np.ndarray, group_size: int) -> np.ndarray:
    """Same values as ``dequant_w16_bits`` through a 16 x 65536 table.

    Each entry of the table is ``_encode_one((c - 8) * s)`` for one code c and
    one scale bit pattern s, so only the lookup differs from the direct form.
    """
    codes = np.asarray(codes, dtype=np.int64)
    N, K = codes.shape
    sb = np.asarray(scale_bits, dtype=np.uint16)
    used = np.unique(sb)
    table = {}
    for s_bits in used.tolist():
        s = float(fp16_bits_to_float(np.uint16(s_bits)))
        table[s_bits] = np.array([_encode_one((c - ZERO_POINT) * s) for c in range(16)], dtype=np.uint16)
    lut = np.zeros((65536, 16), dtype=np.uint16)
    for s_bits, row in table.items():
        lut[s_bits] = row
    g_of_k = np.arange(K) // group_size
    s_nk = sb[g_of_k, :].T.astype(np.int64)
    return lut[s_nk, codes]


# ----------------------------------------------------------------------------
# The three products.  Accumulation is in float64 on exact float32 weights.
# ----------------------------------------------------------------------------
def embedding(codes: np.ndarray, scale_bits: np.ndarray, group_size: int, indices) -> np.ndarray:
    """Rows of the dequantised weight gathered by index, exact float32 [T, K].

    The Q4 embedding reads the linear weight's nibble layout ("[ExecuTorch][WebGPU]
    Replace broad QKV fusion with BK64 kernel", description of #21483:
    is_linear_weight); each element is the dequantisation of "[ExecuTorch][Vulkan]
    Add et_vk.linear_q4gsw_backward kernel (4-bit input-grad)", PR description:
        out[t, k] = (code[idx[t], k] - 8) * s[k // gs, idx[t]].
    An index outside [0, N) raises IndexError.
    """
    codes = np.asarray(codes)
    idx = np.asarray(indices, dtype=np.int64).reshape(-1)
    N, K = codes.shape
    if idx.size and (idx.min() < 0 or idx.max() >= N):
        raise IndexError("embedding index outside [0, N)")
    c = codes[idx, :].astype(np.int64)                    # [T, K]
    s = fp16_bits_to_float(scale_bits)                    # [G, N]
    g_of_k = np.arange(K) // group_size
    s_tk = s[g_of_k, :][:, idx].T                         # s[k // gs, idx[t]] -> [T, K]
    return ((c - ZERO_POINT).astype(np.float64) * s_tk).astype(np.float32)


def linear_fwd(x_bits: np.ndarray, codes: np.ndarray, scale_bits: np.ndarray, group_size: int):
    """y[m, n] = sum_k x[m, k] * w[n, k]; returns (y, bound) with bound = sum_k |x||w|.

    x_bits: fp16 bits uint16 [M, K].  The forward is the per-projection GEMM
    that [P2]'s backward mirrors and [P3] fuses three times.
    """
    x = fp16_bits_to_float(x_bits)
    w = dequant_w32(codes, scale_bits, group_size).astype(np.float64)
    y = x @ w.T
    bound = np.abs(x) @ np.abs(w).T
    return y, bound


def linear_bwd_input(dout_bits: np.ndarray, codes: np.ndarray, scale_bits: np.ndarray, group_size: int):
    """d_x[m, k] = sum_n d_out[m, n] * w[n, k]  ([P2], contraction over N).

    Returns (d_x, bound) with bound = sum_n |d_out||w|.
    """
    d = fp16_bits_to_float(dout_bits)
    w = dequant_w32(codes, scale_bits, group_size).astype(np.float64)
    dx = d @ w
    bound = np.abs(d) @ np.abs(w)
    return dx, bound


def qkv_fwd(x_bits, codes, scale_bits, group_size, Nq: int, Nk: int, Nv: int):
    """[P3]: three projections of one x from one row-concatenated weight.

    Rows [0, Nq) are Q, [Nq, Nq+Nk) are K, [Nq+Nk, Nq+Nk+Nv) are V, and the scales
    are split the same way along their N axis.  Returns ((y_q, b_q), (y_k, b_k),
    (y_v, b_v)).
    """
    codes = np.asarray(codes)
    sb = np.asarray(scale_bits)
    assert codes.shape[0] == Nq + Nk + Nv
    out = []
    for lo, hi in ((0, Nq), (Nq, Nq + Nk), (Nq + Nk, Nq + Nk + Nv)):
        out.append(linear_fwd(x_bits, codes[lo:hi], sb[:, lo:hi], group_size))
    return tuple(out)


def linear_fwd_rows(x_bits, codes, scale_bits, group_size, rows):
    """The forward on a subset of token rows (rows are independent)."""
    return linear_fwd(np.asarray(x_bits)[rows], codes, scale_bits, group_size)


def linear_bwd_input_rows(dout_bits, codes, scale_bits, group_size, rows):
    return linear_bwd_input(np.asarray(dout_bits)[rows], codes, scale_bits, group_size)
