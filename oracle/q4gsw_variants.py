"""Plain CPU oracle for the variants of the q4gsw layer beside the fp16-scale path.

TEST INFRASTRUCTURE ONLY, under the same rule as ``q4gsw_oracle``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import
it; it shares no code with the CUDA library.

1. fp32 scales ("Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch
   fork", issue #1361: the fork's shader list has an fp32-scale
   dequantise-and-accumulate helper, ``linear_fp32_scale_dq_acc``; the Oct 20
   comment says it brought no measurable accuracy gain and that fp16 scales
   are kept).  The pages give only the name.  Reading taken here:
     - packed layout version 2: the version 1 codes region unchanged, the
       scales as fp32 [G][N] (4 bytes each) at the same 256-byte-aligned offset,
       the trailer after them with version word 2;
     - the dequantised weight is w32[n, k] = fp32_RNE((code - 8) * s32[k // gs, n]):
       one rounding, because (code - 8) * s32 can need up to 27 significant bits;
     - accumulation in fp32 (fp64 here), outputs fp32;
     - a tensor-core operand is fp16_RNE(w32).
2. The frozen-base adapter step ("[ExecuTorch][Vulkan] Add
   et_vk.linear_q4gsw_backward kernel (4-bit input-grad)", PR description: the
   input gradient of the frozen 4-bit base exists for on-device adapter
   training).  The pages do not define the adapter.  Reading taken here: a
   rank-r low-rank adapter beside the frozen base,
       y   = x dequant(W)^T + (x A^T) B^T          A fp16 [r, K], B fp16 [N, r]
       d_x = d_out dequant(W) + (d_out B) A        (the adjoint of the forward)
   with no scaling factor (a caller folds one into B).
3. linear_dq8ca_q4gsw (the same fork's shader list): 8-bit dynamically
   quantised activations times the q4gsw weight; the reading is stated above
   ``dq8ca_quantize``.

Each function returns the exact value (fp64 sums of exact terms) and the
per-element bound of the absolute products, as ``q4gsw_oracle`` does.
"""
from __future__ import annotations

import math

import numpy as np

from .q4gsw_oracle import (CODE_MAX, REGION_ALIGN, TRAILER_BYTES, TRAILER_MAGIC, ZERO_POINT, _codes_offset_table,
                           dequant_w32, float_to_fp16_bits_rne, fp16_bits_to_float, linear_bwd_input, linear_fwd)

LAYOUT_VERSION_F32S = 2


# ----------------------------------------------------------------------------
# binary32 <-> real, written from the IEEE 754 definition
# (1 sign bit, 8 exponent bits with bias 127, 23 fraction bits).
# ----------------------------------------------------------------------------
def fp32_bits_to_float(bits) -> np.ndarray:
    """Decode binary32 bit patterns (uint32) to float64 exactly.

    normal:    (-1)^s * 2^(e-127) * (1 + f/2^23)   for 1 <= e <= 254
    subnormal: (-1)^s * 2^(-126)  * (f/2^23)       for e == 0
    e == 255:  +-inf (f == 0) or NaN.
    """
    b = np.asarray(bits, dtype=np.uint32).astype(np.int64)
    sign = np.where((b >> 31) & 1, -1.0, 1.0)
    e = (b >> 23) & 0xFF
    f = (b & 0x7FFFFF).astype(np.float64)
    normal = sign * np.ldexp(1.0 + f / 8388608.0, (e - 127).astype(np.int64))
    sub = sign * np.ldexp(f / 8388608.0, -126)
    out = np.where(e == 0, sub, normal)
    out = np.where((e == 255) & (f == 0), sign * np.inf, out)
    out = np.where((e == 255) & (f != 0), np.nan, out)
    return out


def encode_fp32_rne(x: float) -> int:
    """Round one real (a float64 holding it exactly) to binary32, ties to even.

    For |x| in [2^e, 2^(e+1)) with e >= -126 the spacing of binary32 values is
    2^(e-23); below 2^-126 it is the subnormal quantum 2^-149.  The value is
    divided by its spacing (exact), rounded half-to-even by Python's ``round``
    and re-assembled; a significand rounding up to 2^24 carries into the
    exponent and magnitudes rounding to 2^128 or more become inf.
    """
    if x != x:
        return 0x7FC00000
    s = 0x80000000 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a == 0:
        return s
    if a == math.inf:
        return s | 0x7F800000
    _, e2 = math.frexp(a)
    e = e2 - 1
    if e < -126:
        q = round(math.ldexp(a, 149))
        if q >= (1 << 23):
            return s | (1 << 23)
        return s | q
    q = round(math.ldexp(a, 23 - e))          # in [2^23, 2^24]
    if q == (1 << 24):
        q = 1 << 23
        e += 1
    if e > 127:
        return s | 0x7F800000
    return s | ((e + 127) << 23) | (q - (1 << 23))


# ----------------------------------------------------------------------------
# Packed layout version 2 (fp32 scales)
# ----------------------------------------------------------------------------
def packed_layout_f32s(N: int, K: int, group_size: int) -> dict:
    """Byte map of one packed weight with fp32 scales (layout version 2).

    codes region as version 1 (offset 0, N/2 * K bytes); scales fp32 [G][N]
    row-major at round_up(N/2*K, 256); trailer (64 bytes: magic, version 2, N,
    K, group_size, range flag, zeros) at round_up(scales end, 256).
    """
    G = K // group_size
    codes_bytes = (N // 2) * K
    scales_offset = -(-codes_bytes // REGION_ALIGN) * REGION_ALIGN
    scales_bytes = 4 * G * N
    trailer_offset = -(-(scales_offset + scales_bytes) // REGION_ALIGN) * REGION_ALIGN
    return {"G": G, "codes_offset": 0, "codes_bytes": codes_bytes, "scales_offset": scales_offset,
            "scales_bytes": scales_bytes, "trailer_offset": trailer_offset,
            "total_bytes": trailer_offset + TRAILER_BYTES}


def pack_f32s(codes: np.ndarray, scale_bits32: np.ndarray, group_size: int) -> np.ndarray:
    """codes uint8 [N, K] in 0..15 and fp32 scale bits uint32 [G, N] -> uint8 blob (version 2)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    lay = packed_layout_f32s(N, K, group_size)
    if codes.max(initial=0) > CODE_MAX:
        raise ValueError("code out of range")
    byte_pk = (codes[0::2, :] | (codes[1::2, :] << 4)).astype(np.uint8)
    rows = np.zeros((N // 2, K), dtype=np.uint8)
    rows[:, _codes_offset_table(K)] = byte_pk
    blob = np.zeros(lay["total_bytes"], dtype=np.uint8)
    blob[:lay["codes_bytes"]] = rows.reshape(-1)
    sb = np.ascontiguousarray(np.asarray(scale_bits32, dtype="<u4"))
    assert sb.shape == (lay["G"], N)
    blob[lay["scales_offset"]:lay["scales_offset"] + lay["scales_bytes"]] = sb.view(np.uint8).reshape(-1)
    words = np.zeros(TRAILER_BYTES // 4, dtype="<u4")
    words[:6] = (TRAILER_MAGIC, LAYOUT_VERSION_F32S, N, K, group_size, 0)
    blob[lay["trailer_offset"]:] = words.view(np.uint8)
    return blob


def unpack_scale_bits_f32s(blob: np.ndarray, N: int, K: int, group_size: int) -> np.ndarray:
    lay = packed_layout_f32s(N, K, group_size)
    raw = np.ascontiguousarray(np.asarray(blob, np.uint8)[lay["scales_offset"]:lay["scales_offset"] + lay["scales_bytes"]])
    return raw.view("<u4").reshape(lay["G"], N).copy()


# ----------------------------------------------------------------------------
# Dequantisation with fp32 scales
# ----------------------------------------------------------------------------
def dequant_w32_f32s(codes: np.ndarray, scale_bits32: np.ndarray, group_size: int) -> np.ndarray:
    """w32[n, k] = fp32_RNE((code[n, k] - 8) * s32[k // gs, n]) as float32 [N, K].

    The product of a 4-bit integer and a 24-bit significand is exact in
    float64; numpy's float64 -> float32 conversion rounds it once, to nearest
    even (pinned against ``encode_fp32_rne`` in the tests).
    """
    codes = np.asarray(codes, dtype=np.int64)
    N, K = codes.shape
    s = fp32_bits_to_float(scale_bits32)                # [G, N] float64, exact
    s_nk = s[np.arange(K) // group_size, :].T            # s32[k // gs, n] -> [N, K]
    exact = (codes - ZERO_POINT).astype(np.float64) * s_nk
    with np.errstate(over="ignore"):   # products beyond float32 become inf, as in IEEE arithmetic
        return exact.astype(np.float32)


def dequant_w16_bits_f32s(codes: np.ndarray, scale_bits32: np.ndarray, group_size: int) -> np.ndarray:
    """fp16 operand bits: fp16_RNE(w32) of the version-2 weight."""
    w = dequant_w32_f32s(codes, scale_bits32, group_size).astype(np.float64)
    return float_to_fp16_bits_rne(w)


def dequant_w16_bits_f32s_fast(codes: np.ndarray, scale_bits32: np.ndarray, group_size: int) -> np.ndarray:
    """Same values as ``dequant_w16_bits_f32s`` through numpy's float32 -> float16
    conversion (round to nearest even; the tests check it against the loop)."""
    w = dequant_w32_f32s(codes, scale_bits32, group_size)
    with np.errstate(over="ignore"):
        return w.astype(np.float16).view(np.uint16)


def embedding_f32s(codes: np.ndarray, scale_bits32: np.ndarray, group_size: int, indices) -> np.ndarray:
    """Rows of the version-2 dequantised weight gathered by index: w32[idx[t], :]."""
    idx = np.asarray(indices, dtype=np.int64).reshape(-1)
    N = np.asarray(codes).shape[0]
    if idx.size and (idx.min() < 0 or idx.max() >= N):
        raise IndexError("embedding index outside [0, N)")
    return dequant_w32_f32s(np.asarray(codes)[idx], np.asarray(scale_bits32)[:, idx], group_size)


def linear_fwd_f32s(x_bits, codes, scale_bits32, group_size):
    """y[m, n] = sum_k x[m, k] w32[n, k] (fp64 sum of exact products); returns (y, bound)."""
    x = fp16_bits_to_float(x_bits)
    w = dequant_w32_f32s(codes, scale_bits32, group_size).astype(np.float64)
    return x @ w.T, np.abs(x) @ np.abs(w).T


def linear_bwd_input_f32s(dout_bits, codes, scale_bits32, group_size):
    """d_x[m, k] = sum_n d_out[m, n] w32[n, k]; returns (d_x, bound)."""
    d = fp16_bits_to_float(dout_bits)
    w = dequant_w32_f32s(codes, scale_bits32, group_size).astype(np.float64)
    return d @ w, np.abs(d) @ np.abs(w)


def qkv_fwd_f32s(x_bits, codes, scale_bits32, group_size, Nq: int, Nk: int, Nv: int):
    codes = np.asarray(codes)
    sb = np.asarray(scale_bits32)
    assert codes.shape[0] == Nq + Nk + Nv
    return tuple(linear_fwd_f32s(x_bits, codes[lo:hi], sb[:, lo:hi], group_size)
                 for lo, hi in ((0, Nq), (Nq, Nq + Nk), (Nq + Nk, Nq + Nk + Nv)))


# ----------------------------------------------------------------------------
# Frozen-base low-rank adapter
# ----------------------------------------------------------------------------
def adapter_fwd(x_bits, codes, scale_bits, group_size, a_bits, b_bits):
    """y = x dequant(W)^T + (x A^T) B^T; returns (y, bound).

    x fp16 [M, K], A fp16 [r, K], B fp16 [N, r] (bit patterns).  The bound is
    the base's sum_k |x||w| plus the adapter chain sum_j (sum_k |x||A_jk|) |B_nj|,
    which also covers the rounding of the intermediate x A^T.
    """
    y0, b0 = linear_fwd(x_bits, codes, scale_bits, group_size)
    x = fp16_bits_to_float(x_bits)
    A = fp16_bits_to_float(a_bits)
    B = fp16_bits_to_float(b_bits)
    u = x @ A.T                                   # [M, r]
    return y0 + u @ B.T, b0 + (np.abs(x) @ np.abs(A).T) @ np.abs(B).T


def adapter_bwd_input(dout_bits, codes, scale_bits, group_size, a_bits, b_bits):
    """d_x = d_out dequant(W) + (d_out B) A; returns (d_x, bound)."""
    d0, b0 = linear_bwd_input(dout_bits, codes, scale_bits, group_size)
    d = fp16_bits_to_float(dout_bits)
    A = fp16_bits_to_float(a_bits)
    B = fp16_bits_to_float(b_bits)
    v = d @ B                                     # [M, r]
    return d0 + v @ A, b0 + (np.abs(d) @ np.abs(B)) @ np.abs(A)


def adapter_intermediate(act_bits, proj_bits):
    """The low-rank intermediate act @ proj^T in fp64 (u = x A^T with proj = A,
    or v = d_out B with proj = B^T), for tests of the intermediate's rounding."""
    return fp16_bits_to_float(act_bits) @ fp16_bits_to_float(proj_bits).T


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "math", "np")]
_ = dequant_w32  # re-exported helpers above come from the base oracle


# ----------------------------------------------------------------------------
# linear_dq8ca_q4gsw: int8 dynamically quantised activations x q4gsw weights
# ----------------------------------------------------------------------------
# "Upstream the Gemma 4 Vulkan support we carry on our ExecuTorch fork", issue
# #1361, the fork's shader list: linear_dq8ca_q4gsw beside linear_q4gsw.  The
# page gives only the name: 8-bit dynamically quantised activations ("dq8"),
# quantised per channel-row with an asymmetric range ("ca"), times the 4-bit
# group-symmetric weight.  Reading taken here (every step an IEEE fp32 operation,
# round to nearest even, as a CPU or GPU computes it):
#   per token m, over its K features:
#     lo = min(0, min_k x[m, k]),  hi = max(0, max_k x[m, k])
#     a_s = (hi - lo) / 255            (1 when hi == lo)
#     a_z = clamp(rint(-128 - lo / a_s), -128, 127)
#     q[m, k] = clamp(rint(x[m, k] / a_s) + a_z, -128, 127)
#   y[m, n] = a_s[m] * sum_g s[g, n] * sum_{k in g} (q[m, k] - a_z[m]) (code[n, k] - 8)
# The inner sums are exact integers; the bound is a_s sum_g |s| sum |q - a_z| |c - 8|.
def dq8ca_quantize(x_bits):
    """x fp16 bits [M, K] -> (q int8 [M, K], a_s float32 [M], a_z int32 [M])."""
    x = fp16_bits_to_float(x_bits).astype(np.float32)          # exact: fp16 values are fp32 values
    M, K = x.shape
    q = np.zeros((M, K), np.int8)
    a_s = np.zeros(M, np.float32)
    a_z = np.zeros(M, np.int32)
    for m in range(M):
        lo = np.float32(min(np.float32(0), x[m].min()))
        hi = np.float32(max(np.float32(0), x[m].max()))
        s = np.float32(1) if hi == lo else np.float32(np.float32(hi - lo) / np.float32(255))
        z = np.rint(np.float32(np.float32(-128) - np.float32(lo / s)))
        z = int(min(127, max(-128, z)))
        qm = np.rint(x[m] / s).astype(np.int64) + z            # x / s rounded once in float32
        q[m] = np.clip(qm, -128, 127).astype(np.int8)
        a_s[m] = s
        a_z[m] = z
    return q, a_s, a_z


def linear_dq8ca_fwd(x_bits, codes, scale_bits, group_size):
    """y = a_s * sum_g s * sum (q - a_z)(c - 8) on the quantised activations; returns (y, bound)."""
    q, a_s, a_z = dq8ca_quantize(x_bits)
    codes = np.asarray(codes, dtype=np.int64)
    N, K = codes.shape
    G = K // group_size
    s = fp16_bits_to_float(scale_bits)                          # [G, N]
    qa = q.astype(np.int64) - a_z[:, None].astype(np.int64)      # [M, K] exact
    cw = codes - ZERO_POINT                                      # [N, K] exact
    y = np.zeros((q.shape[0], N))
    b = np.zeros((q.shape[0], N))
    for g in range(G):
        ks = slice(g * group_size, (g + 1) * group_size)
        t = (qa[:, ks] @ cw[:, ks].T).astype(np.float64)        # exact integers
        ta = (np.abs(qa[:, ks]) @ np.abs(cw[:, ks]).T).astype(np.float64)
        y += t * s[g][None, :]
        b += ta * np.abs(s[g])[None, :]
    return y * a_s[:, None].astype(np.float64), b * a_s[:, None].astype(np.float64)
