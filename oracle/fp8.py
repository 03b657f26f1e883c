"""FP8 (e4m3) latent cache for the oracle: the codec, the per-page quantizer
and the dequantized rows a decode over such a cache attends to.

TEST INFRASTRUCTURE, under the same rules as ``mla_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
it, and it imports nothing from the product package.

yunthe.com, "多头潜在注意力机制：内存优化与推理加速的革新方案", section
"一、技术演进背景": 8-bit (or 4-bit) quantization is named as a way to shrink
the KV cache, at some cost in precision.  The page fixes no format, so this
module takes a plain reading, stated once here and in the design notes:

* Format: FP8 E4M3 -- 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
  bits; exponent field 0 holds the subnormals m * 2^-9; no infinities; the
  pattern S.1111.111 is NaN; the largest finite magnitude is 448.
* Scale: one fp32 scale per cache page and tensor (the latent rows of a page,
  and separately its rope rows) = (largest finite |x| on the page) / 448,
  both operands fp32 and the quotient rounded to fp32; 1 when the page holds
  no nonzero finite value.
* Codes: x / scale computed in fp32 (rounded to fp32), then rounded to the
  nearest E4M3 value, ties to the even code, magnitudes past 448 saturated to
  448; NaN stays NaN.  (The quantized code is an integer decided by floating
  point, so the oracle takes that decision in fp32, as the kernel does.)
* Dequantized value: decode(code) * scale, here in fp64.

Parity of the device decode over an FP8 cache is checked against
``mla_oracle.decode`` run on the dequantized rows: the quantization error is
the format's, pinned separately by closed-form bounds, and is not part of the
decode's tolerance.
"""
from __future__ import annotations

import numpy as np

from .mla_oracle import DEFAULT_ROPE_BASE, rope

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode(codes) -> np.ndarray:
    """Values (fp64) of E4M3 codes (any integer array of bytes)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * m * 2.0 ** -9
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, out)


# the 127 non-negative finite values in code order (codes 0x00 .. 0x7E), increasing
_POS_VALUES = e4m3_decode(np.arange(0x7F))


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (uint8) of fp32 values: nearest value, ties to the even code,
    saturating at 448; NaN -> 0x7F (0xFF for a negative NaN)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    mag = np.abs(x)
    neg = np.signbit(x)
    nan = np.isnan(x)
    m = np.where(nan, 0.0, np.minimum(mag, E4M3_MAX))
    hi = np.searchsorted(_POS_VALUES, m, side="left")          # first value >= m
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    exact = _POS_VALUES[hi] == m
    d_lo = m - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - m
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(exact, hi, np.where(pick_hi, hi, lo)).astype(np.int64)
    code = np.where(nan, E4M3_NAN, code) | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def page_scale(x) -> np.float32:
    """fp32 scale of one page's values (any shape): largest finite |x| / 448."""
    a = np.abs(np.asarray(x, dtype=np.float32))
    a = a[np.isfinite(a)]
    amax = np.float32(a.max()) if a.size else np.float32(0.0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E4M3_MAX))


def quantize_pages(pool):
    """Pool [P, page_size, d] (values of the bf16 cache) -> (codes uint8 of the
    same shape, scales fp32 [P])."""
    pool = np.asarray(pool, dtype=np.float32)
    scales = np.array([page_scale(pool[p]) for p in range(pool.shape[0])], dtype=np.float32)
    q = (pool / scales[:, None, None]).astype(np.float32)      # fp32 quotient, as the kernel forms it
    return e4m3_encode(q), scales


def dequantize_pages(codes, scales) -> np.ndarray:
    """fp64 values of a quantized pool."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None, None]


def unrotate(k_rot, tok_pos, rope_base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """Raw positional keys whose rotation at tok_pos is k_rot (the inverse
    rotation, RoPE at -tok_pos), for an oracle that rotates raw keys itself."""
    return rope(np.asarray(k_rot, dtype=np.float64), -np.asarray(tok_pos, dtype=np.float64), rope_base)


def dequantized_rows(lat_codes, lat_scales, rope_codes, rope_scales, tok_seq, tok_pos, page_table,
                     page_size: int = 64, rope_base: float = DEFAULT_ROPE_BASE):
    """The cached rows a decode over the quantized pools reads, in the packed
    order of (tok_seq, tok_pos): latent rows and raw (un-rotated) rope keys."""
    lat = dequantize_pages(lat_codes, lat_scales)
    rop = dequantize_pages(rope_codes, rope_scales)
    tok_seq = np.asarray(tok_seq, dtype=np.int64)
    tok_pos = np.asarray(tok_pos, dtype=np.int64)
    pages = np.asarray(page_table, dtype=np.int64)[tok_seq, tok_pos // page_size]
    slots = tok_pos % page_size
    return lat[pages, slots], unrotate(rop[pages, slots], tok_pos, rope_base)
