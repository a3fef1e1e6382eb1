"""FP8 (e4m3) compressed-cache oracle -- TEST INFRASTRUCTURE ONLY.

The Forcing-KV page says the compression composes with existing KV
quantization (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "与现有产品/工作流
的接口" item 3, and "与基线对比及工程启示" item 3) but fixes no format.  The
reading implemented here:

  * format: OCP FP8 E4M3 ("e4m3fn": bias 7, 3 mantissa bits, no infinities,
    largest finite 448, subnormal step 2^-9), round to nearest, ties to even,
    saturating to +-448;
  * one scale per (layer, head, segment) for K and one for V, where a
    segment is a history frame of the compressed cache or a frame of the
    current chunk: s = amax / 448 over the segment's T x D elements (s = 1
    for an all-zero segment), codes = e4m3(x * (448 / amax));
  * one scale per query row for Q, same rule over the row's D elements;
  * the fp8 attention is the exact softmax attention (``fkv_oracle.attention``)
    over the DEQUANTISED values code * scale.

The codes are an integer decided by floating point, so both sides take the
decision in the same precision, fp32 (the kernel's): the amax is exact, the
two divisions 448 / amax and amax / 448 and the product x * inv are each one
correctly rounded fp32 operation, then one rounding to e4m3.  Everything after
the codes is float64.

``attention_tolerance`` states how far an fp8 tensor-core evaluation may sit
from the exact attention over the dequantised cache: its probabilities are
rounded to e4m3 before the P.V product (relative error <= 2^-4 where normal,
absolute <= 2^-10 of the scaled unit where subnormal) and its output is rounded
to bf16.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUB_STEP = 2.0 ** -9


def _round_half_even(x: np.ndarray) -> np.ndarray:
    """Nearest integer, ties to the even one (numpy's rint is exactly that)."""
    return np.rint(x)


def e4m3_encode(x) -> np.ndarray:
    """fp32 values -> e4m3 codes (uint8), RNE, saturating to +-448.

    Works from the format's definition: a value below 2^-6 is a multiple of
    2^-9 (exponent field 0); otherwise (1 + m/8) * 2^e with e in [-6, 8] and
    exponent field e + 7.  NaN maps to the NaN code 0x7f (with its sign).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    sign = np.signbit(x).astype(np.uint8) << 7
    code = np.zeros(x.shape, dtype=np.uint8)

    sub = a < E4M3_MIN_NORMAL
    # subnormal range: code = round(a / 2^-9); 8 lands exactly on 2^-6 = code 8
    code[sub] = _round_half_even(a[sub] / E4M3_SUB_STEP).astype(np.uint8)

    nrm = ~sub & np.isfinite(a)
    an = a[nrm]
    m_frac, e2 = np.frexp(an)                 # an = m_frac * 2^e2, m_frac in [0.5, 1)
    e = e2.astype(np.int64) - 1               # an = (2 m_frac) * 2^e, 2 m_frac in [1, 2)
    mant = _round_half_even((2.0 * m_frac - 1.0) * 8.0).astype(np.int64)
    carry = mant == 8
    e = e + carry
    mant = np.where(carry, 0, mant)
    over = (e > 8) | ((e == 8) & (mant == 7))  # 480 and above do not exist: saturate
    c = ((e + 7) << 3) | mant
    c = np.where(over, 0x7E, c)
    code[nrm] = c.astype(np.uint8)

    code[np.isnan(a)] = 0x7F
    code[np.isinf(a)] = 0x7E                  # satfinite
    return code | sign


def e4m3_decode(code) -> np.ndarray:
    """e4m3 codes -> float64 values (0x7f / 0xff decode to NaN)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    val = np.where(E == 0, M * E4M3_SUB_STEP, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    val = np.where((E == 15) & (M == 7), np.nan, val)
    return s * val


def scale_of(amax: np.float32) -> Tuple[np.float32, np.float32]:
    """(scale, inverse) of a block whose largest magnitude is amax, in fp32.

    scale = amax / 448 and inverse = 448 / amax, each one correctly rounded
    fp32 division; an all-zero block gets (1, 1).
    """
    amax = np.float32(amax)
    if amax == np.float32(0):
        return np.float32(1.0), np.float32(1.0)
    return np.float32(amax / np.float32(E4M3_MAX)), np.float32(np.float32(E4M3_MAX) / amax)


def quantize_block(x) -> Tuple[np.ndarray, np.float32]:
    """One block (a segment, or a query row) -> (codes, scale).

    codes = e4m3(fp32(x * inverse)) with the block's own fp32 inverse.
    """
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    scale, inv = scale_of(amax)
    return e4m3_encode((x * inv).astype(np.float32)), scale


def quantize_segments(x, seg_len: int) -> Tuple[np.ndarray, np.ndarray]:
    """Rows [n_seg * seg_len][D] -> (codes [rows][D], scales [n_seg]): one scale per segment."""
    x = np.asarray(x, dtype=np.float32)
    n_seg = x.shape[0] // seg_len
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(n_seg, dtype=np.float32)
    for g in range(n_seg):
        rows = slice(g * seg_len, (g + 1) * seg_len)
        codes[rows], scales[g] = quantize_block(x[rows])
    return codes, scales


def quantize_rows(x) -> Tuple[np.ndarray, np.ndarray]:
    """Rows [n][D] -> (codes [n][D], scales [n]): one scale per row (the queries)."""
    x = np.asarray(x, dtype=np.float32)
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros(x.shape[0], dtype=np.float32)
    for r in range(x.shape[0]):
        codes[r], scales[r] = quantize_block(x[r])
    return codes, scales


def dequantize(codes, scales, seg_len: int) -> np.ndarray:
    """codes [rows][D] with one scale per seg_len rows -> float64 values."""
    v = e4m3_decode(codes)
    s = np.repeat(np.asarray(scales, dtype=np.float64), seg_len)[: v.shape[0]]
    return v * s[:, None]


def compact_quantized(k_hist, v_hist, kept, T: int):
    """The fp8 compressed cache of one head: the kept frames (ascending), each
    quantized as its own segment.

    Returns (k_codes [cnt*T][D], sk [cnt], v_codes, sv [cnt]).
    """
    kept = np.asarray(kept, dtype=np.int64)
    D = np.asarray(k_hist).shape[1]
    kc = np.zeros((len(kept) * T, D), dtype=np.uint8)
    vc = np.zeros((len(kept) * T, D), dtype=np.uint8)
    sk = np.zeros(len(kept), dtype=np.float32)
    sv = np.zeros(len(kept), dtype=np.float32)
    for p, f in enumerate(kept):
        src = slice(int(f) * T, (int(f) + 1) * T)
        dst = slice(p * T, (p + 1) * T)
        kc[dst], sk[p] = quantize_block(np.asarray(k_hist, dtype=np.float32)[src])
        vc[dst], sv[p] = quantize_block(np.asarray(v_hist, dtype=np.float32)[src])
    return kc, sk, vc, sv


def attention_tolerance(q, keys, v_codes, v_scale_per_key, scale: float,
                        out_ref: np.ndarray, sigmas: float = 6.0) -> np.ndarray:
    """Per-element bound on |fp8 tensor-core attention - exact attention| for
    rows of q over dequantised keys, with V given as codes and a scale per key.

    Model of the evaluation (its only departures from the exact result beyond
    fp32 rounding): probabilities are formed relative to a running row max
    that trails the true max by at most 2^8 (in base 2), multiplied by
    r_j = sv_j / max(sv) <= 1 and rounded to e4m3, then P.V' is accumulated
    and divided by the fp32 row sum, and the output rounded to bf16.  With
    w_j the exact softmax weights and u_j = exp(s_j - max s) * r_j a lower
    bound of key j's scaled probability:
      normal keys (u_j >= 2^-6): relative rounding error <= 2^-4,
      possibly subnormal keys (u_j < 2^-6): absolute error <= 2^-10 in units of
        max(sv) and the running row sum, which is >= L = sum_j exp(s_j - max s).
    The errors of distinct keys are independent and zero-mean, so the bound
    is `sigmas` standard deviations of their sum (uniform errors: variance
    h^2 / 3 for half-width h), plus the bf16 rounding of the output.
    """
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    v8 = e4m3_decode(v_codes)
    sv = np.asarray(v_scale_per_key, dtype=np.float64)
    sv_max = float(np.max(sv)) if sv.size else 1.0
    r = sv / sv_max
    vals = v8 * sv[:, None]
    s = (q @ keys.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    L = e.sum(axis=1, keepdims=True)
    w = e / L
    u = e * r[None, :]
    normal = u >= E4M3_MIN_NORMAL
    var_n = ((w * normal) ** 2 * (2.0 ** -4) ** 2 / 3.0) @ (vals ** 2)
    var_s = ((~normal).astype(np.float64) * (2.0 ** -10) ** 2 / 3.0) @ (v8 ** 2)
    var_s = var_s * (sv_max / L) ** 2
    return sigmas * np.sqrt(var_n + var_s) + 2.0 ** -8 * np.abs(out_ref) + 1e-6
