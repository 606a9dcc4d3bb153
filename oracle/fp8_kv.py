"""Oracle: tree attention over an 8-bit (E4M3) KV cache (TEST INFRASTRUCTURE) -- the first step of the next row
"FP8 KV cache variant of the attention".

The pages do not mention 8-bit caches; the row carries the paged attention of [JF] technical summary section 3
(and its mask, section 2) over to a cache stored in 8 bits.  Readings used:

  * E4M3 is the 8-bit float with 1 sign, 4 exponent (bias 7) and 3 mantissa bits and no infinities: exponent field
    0 gives subnormals (m / 8) * 2^-6, the codes S.1111.111 are NaN, the largest magnitude is 448;
  * one scale per cache (one for K, one for V): a stored code c stands for decode(c) * scale;
  * encoding rounds to the nearest code (ties to the even mantissa) after clamping to [-448, 448], so values past
    the range saturate instead of becoming NaN;
  * the attention is the bf16 path's definition (tree_attention) applied to the decoded, scaled values.

Pinned by tests/test_oracle_fp8.py: named codes from the format's definition, all 256 codes and random values
against torch's float8_e4m3fn conversion (an independent implementation), ties to even, saturation, and two closed
forms of the scales (the V scale multiplies the output; the K scale acts as a factor on the softmax scale).
"""
from __future__ import annotations

import numpy as np

from .tree_attention import tree_attention

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """uint8 codes -> float64 values (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# every finite non-negative value, increasing with its code (codes 0 .. 0x7E)
_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(x):
    """float -> uint8 codes: clamp to +-448, then the nearest code, ties to the even mantissa.  NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")          # first code whose value >= a
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - _POS[lo], _POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(a == _POS[hi], hi, np.where(pick_hi, hi, lo)).astype(np.int64)
    code = np.where(np.signbit(x), code | 0x80, code)  # negative values (and -0) keep their sign
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize_cache(cache, scale):
    """Cache values -> E4M3 codes for the given scale (value / scale, encoded)."""
    return e4m3_encode(np.asarray(cache, dtype=np.float64) / float(scale))


def tree_attention_fp8(q, k_codes, v_codes, k_scale, v_scale, block_table, prefix_lens, tree_offsets, parent,
                       sm_scale, num_kv_heads=None, rows=None):
    """tree_attention over the decoded caches decode(k_codes) * k_scale, decode(v_codes) * v_scale."""
    k = e4m3_decode(k_codes) * float(k_scale)
    v = e4m3_decode(v_codes) * float(v_scale)
    return tree_attention(q, k, v, block_table, prefix_lens, tree_offsets, parent, sm_scale, num_kv_heads, rows)
