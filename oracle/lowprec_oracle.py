"""fp64 CPU oracle for attention with a low-precision V: the FP8 E4M3 format,
per-channel quantization of V and masked attention over the dequantized V.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA product path
never imports this module, and this module imports nothing from it.

Source:
  [FVAttn §3.4]  the GPU quantizes V as a separate step, which the runtime
                 overlaps with CPU-side scheduling; the attention kernel then
                 consumes the quantized V. The pages name no format.

Readings of what the pages leave open (each one is listed in the design notes):
  * format: FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
    no infinities, the all-ones pattern is NaN, largest finite value 448), the
    8-bit format the Blackwell tensor cores multiply.
  * granularity: one fp32 scale per (batch, head, channel), over the valid
    tokens of the head: scale_c = amax_c / 448, so each channel's largest
    magnitude maps to 448.
  * encoding: code = RN-even_e4m3(fp32(v * fp32(448 / amax_c))), saturating at
    +-448, sign of zero kept. The two fp32 operations are IEEE round-to-nearest,
    so the integer code is decided in fp32 on both sides. A channel whose amax
    is below 2^-100 (so 448/amax could overflow fp32) is the zero channel:
    codes 0, scale 0. Pad rows (>= N) get code 0.
  * dequantized value: V^ = value(code) * scale_c (exact in fp64).
  * attention: the masked softmax attention of the FVAttn oracle with V^ in
    place of V. How the kernel rounds P for its 8-bit P.V product is the
    kernel's arithmetic, not part of this definition; its error is bounded in
    the tests, not reproduced here.
"""

from __future__ import annotations

import numpy as np

from .fvattn_oracle import masked_attention, num_blocks

E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F
AMAX_ZERO = 2.0 ** -100


def e4m3_value(code: int) -> float:
    """The real number an E4M3 byte encodes (NaN for the two NaN patterns).
    [FVAttn §3.4] names no format; E4M3 is the reading (module header)."""
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = m * 2.0 ** -9                      # subnormal: m/8 * 2^(1-7)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def e4m3_table() -> np.ndarray:
    """float64 [256]: value of every code."""
    return np.array([e4m3_value(c) for c in range(256)])


_TABLE = e4m3_table()
_POS = _TABLE[:E4M3_NAN_CODE]          # codes 0x00..0x7E, strictly increasing, 0 .. 448


def e4m3_encode(x) -> np.ndarray:
    """Round each value to the nearest finite E4M3 number, ties to the even
    code (mantissa LSB 0), magnitudes above 448 to 448 (saturating). Returns the
    codes as uint8; the sign bit follows the sign of x, zero included.
    [FVAttn §3.4]; rounding rule: the reading in the module header."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")          # _POS[hi-1] < a <= _POS[hi]
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == _POS[hi], hi, code).astype(np.uint8)   # exact values
    return code | (np.signbit(x).astype(np.uint8) << 7)


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, np.uint8)]


def quantize_v(v, N: int):
    """Per-channel E4M3 quantization of V [B, H, Npad, d] (the bf16 values as
    float32). Returns (codes uint8 [B, H, Npad, d], scale float32 [B, H, d]).
    [FVAttn §3.4: the GPU quantizes V before attention]; granularity and scale:
    the reading in the module header."""
    v32 = np.asarray(v, np.float32)
    amax = np.abs(v32[:, :, :N, :]).max(axis=2)                      # exact
    nz = amax >= np.float32(AMAX_ZERO)
    inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, amax, np.float32(1)),
                   np.float32(0)).astype(np.float32)               # fp32 IEEE division
    x = (v32 * inv[:, :, None, :]).astype(np.float32)               # fp32 IEEE product
    codes = e4m3_encode(x)
    codes[:, :, N:, :] = 0
    scale = np.where(nz, amax / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    return codes, scale


def dequantize_v(codes, scale) -> np.ndarray:
    """V^ = value(code) * scale_c in fp64, [B, H, Npad, d]."""
    return e4m3_decode(codes) * np.asarray(scale, np.float64)[:, :, None, :]


def masked_attention_qv(qp, kp, codes, scale, mask, N: int, bs: int, sm_scale: float,
                        blocks=None) -> np.ndarray:
    """Block-sparse attention with the quantized V: the masked softmax over the
    selected blocks' valid keys, times V^. [FVAttn §2.1 (the masked attention),
    §3.4 (V quantized)]"""
    return masked_attention(qp, kp, dequantize_v(codes, scale), mask, N, bs, sm_scale, blocks)


def masked_softmax_weights(qp, kp, mask_row, N: int, bs: int, sm_scale: float, i: int):
    """[FVAttn §2.1] Softmax weights of the valid rows of query block ``i`` of one head over
    the valid keys of its selected blocks. Returns (cols, w): the key positions
    and the fp64 weights [rows, len(cols)], each row summing to one."""
    qp = np.asarray(qp, np.float64)
    kp = np.asarray(kp, np.float64)
    lo, hi = i * bs, min((i + 1) * bs, N)
    cols = np.concatenate([np.arange(j * bs, min((j + 1) * bs, N))
                           for j in np.nonzero(np.asarray(mask_row))[0]])
    logits = (qp[lo:hi] @ kp[cols].T) * sm_scale
    logits = logits - logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    return cols, w / w.sum(axis=-1, keepdims=True)


__all__ = ["E4M3_MAX", "e4m3_value", "e4m3_table", "e4m3_encode", "e4m3_decode", "quantize_v",
           "dequantize_v", "masked_attention_qv", "masked_softmax_weights", "num_blocks"]
