"""FP8 (e4m3) quantization of Q and K for low-precision chunk attention, fp64 otherwise.

What it computes ([RT] kernel table: the attention's QK^T product in 8-bit
integers, SageAttention 2.2, at 65 % of the RTX 5090's INT8 peak -- the pages'
own speed lever on this path; here the 8-bit format is the tensor cores' e4m3):

  * e4m3: 1 sign, 4 exponent (bias 7) and 3 mantissa bits; subnormals
    m * 2^-9; the largest finite magnitude is 448 (exponent 15, mantissa 6);
    exponent 15 with mantissa 7 is NaN; there is no infinity.
  * rounding of a real to e4m3: to the nearest representable value, ties to
    the even mantissa; magnitudes above 448 saturate to 448 (the
    "satfinite" conversion; a NaN stays NaN).
  * block quantization of a [L, H, D] tensor: per block of 128 consecutive
    rows (tokens) and one head, amax = max |x| over the block (fp32),
    inv = 448 / amax and scale = amax / 448 (both one fp32 division),
    code = e4m3(fp32(x * inv)); the block dequantizes to code * scale
    (amax = 0: every code and the scale are 0).
  * low-precision attention: softmax(scale_attn * Q~ K~^T) V with Q~, K~ the
    dequantized blocks, V unquantized, everything else exact (fp64).

Readings: the block is 128 tokens x one head (the kernel's tile), the fp32
steps are written out so that a kernel taking the same steps makes the same
integer decisions (the code of every element), and V stays in bf16 (the
pages quantize only QK^T).  In the chunk rollout what is quantized is the
tensor the bf16 path would hold: RoPE'd Q and K rounded once to bf16
(``round_bf16``); the blocks follow the attention's tiles -- 128 consecutive
tokens of one cached (or auxiliary) frame, 128 consecutive tokens of the
current chunk for its own queries and keys (``fp8_operand``).

Parity: pinned (every finite code rounds to itself; ties to even; agreement
with torch's float8_e4m3fn conversion below the saturation point; the
quantization error bound; exactly representable blocks with amax 448 give
the plain attention exactly).
"""
from __future__ import annotations

import numpy as np

from .attn import attention

E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """Values of the 256 e4m3 codes (index = code), NaN for the two NaN codes."""
    out = np.empty(256, dtype=np.float64)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            v = np.nan
        elif e == 0:
            v = m * 2.0 ** -9
        else:
            v = (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out[c] = -v if s else v
    return out


_POS = e4m3_values()[:127]   # codes 0 .. 126: the finite non-negative values, ascending


def e4m3_round(x) -> np.ndarray:
    """Round to e4m3 (nearest, ties to even mantissa, saturating at +-448); float64 out."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    i = np.clip(np.searchsorted(_POS, a, side="left"), 1, _POS.size - 1)
    lo, hi = _POS[i - 1], _POS[i]
    d_lo, d_hi = a - lo, hi - a
    # the nearer neighbour; on a tie the one with the even code (even mantissa)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (i % 2 == 0))
    r = np.where(pick_hi, hi, lo)
    r = np.where(a >= _POS[-1], E4M3_MAX, r)            # satfinite
    r = np.where(a <= 0.0, 0.0, r)
    r = np.where(np.isnan(x), np.nan, r)
    return np.copysign(r, x)


def quantize_blocks(x, rows: int = 128):
    """Block-quantize x [L, H, D] (values exact in fp32): returns (codes' values [L, H, D]
    float64, scales [n_blocks, H] float32); block b of head h is rows [b*rows, (b+1)*rows)."""
    x = np.asarray(x, dtype=np.float32)
    L, H, _ = x.shape
    nb = (L + rows - 1) // rows
    codes = np.zeros(x.shape, dtype=np.float64)
    scales = np.zeros((nb, H), dtype=np.float32)
    for b in range(nb):
        blk = x[b * rows:(b + 1) * rows]                  # [r, H, D]
        amax = np.abs(blk).max(axis=(0, 2)).astype(np.float32)    # [H]
        for h in range(H):
            if amax[h] == 0:
                continue
            inv = np.float32(E4M3_MAX) / amax[h]
            y = (blk[:, h, :] * inv).astype(np.float32)
            codes[b * rows:(b + 1) * rows, h, :] = e4m3_round(y)
            scales[b, h] = amax[h] / np.float32(E4M3_MAX)
    return codes, scales


def dequantize_blocks(codes, scales, rows: int = 128) -> np.ndarray:
    """codes [L, H, D] * the scale of each element's (block, head), float64."""
    codes = np.asarray(codes, dtype=np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), rows, axis=0)[:codes.shape[0]]
    return codes * s[:, :, None]


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits, ties to the even
    significand; spacing 2^-133 below the normal range); float64 out."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                           # 2^(e-1) <= |x| < 2^e
    q = np.maximum(e - 8, -133).astype(np.float64)
    step = np.exp2(q)
    return np.where(x == 0, x, np.rint(x / step) * step)


def fp8_operand(x, rows: int = 128) -> np.ndarray:
    """What the low-precision product sees of a [L, H, D] operand: x rounded to bf16,
    block-quantized to e4m3 per 128 rows and head, dequantized (float64)."""
    codes, scales = quantize_blocks(round_bf16(x), rows)
    return dequantize_blocks(codes, scales, rows)


def attention_fp8_qk(q, k, v, scale: float, rows: int = 128):
    """Attention with Q and K block-quantized to e4m3 (per 128 rows and head), V as given:
    ([Lq, H, D] O, [H, Lq] LSE) in fp64."""
    qc, qs = quantize_blocks(q, rows)
    kc, ks = quantize_blocks(k, rows)
    return attention(dequantize_blocks(qc, qs, rows), dequantize_blocks(kc, ks, rows),
                     np.asarray(v, dtype=np.float64), scale)
