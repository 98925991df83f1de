"""Plain CPU oracle for the latent-cache append (the write that precedes the
decode step): the q_len new tokens' 576-wide latent rows go into their cache
pages through the block table, as bf16 copies or as fp8-e4m3 codes with one
fp32 scale per token.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). Written from:

* zubnet.ai (es/fr), "LightSeek TokenSpeed 580 TPS ... B200", second
  paragraph: the KV cache lives in pages and is reached through index
  indirection instead of copies. Token j of sequence b sits in physical page
  ``block_table[b, j // 64]``, slot ``j % 64``.
* The decode oracle's causal reading: the q_len new tokens of a step are the
  last q_len positions, already counted in ``seqlens`` (positions
  L_b - q_len .. L_b - 1).
* The fp8 rule, which the pages do not give (this library's reading):
  sigma = amax_d |x_d| / 448 per token (1 for an all-zero row), code =
  e4m3(x / sigma) rounded to nearest, ties to even, saturated to +-448. Both
  divisions are taken in fp32 (IEEE round to nearest) so that the codes, an
  integer decided by floating point, are decided in the same precision as the
  kernel's; x is the bf16 row, exactly representable in fp32.
* OCP 8-bit Floating Point Specification v1.0, section 5.3 (E4M3): 1 sign,
  4 exponent (bias 7), 3 mantissa bits; largest finite magnitude 448.

The encoder is pinned by ``tests/test_oracle_pins.py`` (round trip over every
finite code, ties, saturation, torch's independent conversion, hand-computed
rows).
"""

from __future__ import annotations

import numpy as np

from .mla_oracle import D_QK, FP8_DATA_BYTES, FP8_PAGE_BYTES, PAGE, decode_bf16, decode_e4m3

E4M3_MAX = 448.0

# The 127 non-negative finite e4m3 magnitudes, code 0x00 .. 0x7E, increasing
# with the code (the format is sign-magnitude with the exponent above the
# mantissa, so codes order like their magnitudes).
_E4M3_POS = decode_e4m3(np.arange(0x7F, dtype=np.uint8))


def encode_e4m3(y) -> np.ndarray:
    """fp32 values -> e4m3 codes (uint8): nearest representable magnitude,
    ties to the even code (even mantissa), magnitudes above 448 saturated to
    448, the sign kept (so -0.0 -> 0x80). Inputs must not be NaN."""
    y = np.asarray(y, dtype=np.float32)
    if np.isnan(y).any():
        raise ValueError("encode_e4m3: NaN input")
    a = np.minimum(np.abs(y.astype(np.float64)), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first magnitude >= a
    hi = np.minimum(hi, len(_E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    exact = d_hi == 0
    pick_hi = exact | (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(y), code | 0x80, code).astype(np.uint8)


def quantise_rows_fp8(row_bits):
    """bf16 rows (uint16 [R, 576]) -> (e4m3 codes uint8 [R, 576], sigma fp32 [R])."""
    x = decode_bf16(row_bits).astype(np.float32)               # exact in fp32
    amax = np.abs(x).max(axis=-1)
    sigma = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / sigma[..., None]).astype(np.float32)              # fp32 division, nearest
    return encode_e4m3(y), sigma


def cache_append_ref(cache, kv_dtype, new_bits, block_table, seqlens):
    """Returns a copy of the page pool with the new rows written.

    cache: uint16 [pages, 64, 576] (bf16) or uint8 [pages, 37120] (fp8 codes,
    then 64 fp32 scales); new_bits: uint16 [B, T, 576] bf16 rows of the T new
    tokens of each sequence; block_table int32 [B, max_pages]; seqlens [B]
    (L_b, counting the new tokens). Sequences with L_b < T or whose rows would
    fall outside the block table are left untouched, as are pages outside the
    pool.
    """
    out = np.array(cache, copy=True)
    new_bits = np.asarray(new_bits, dtype=np.uint16)
    B, T, _ = new_bits.shape
    max_pages = block_table.shape[1]
    for b in range(B):
        L = int(seqlens[b])
        if L < T or L > max_pages * PAGE:
            continue
        for t in range(T):
            j = L - T + t
            page = int(block_table[b, j // PAGE])
            if page < 0 or page >= out.shape[0]:
                continue
            slot = j % PAGE
            if kv_dtype == "bf16":
                out[page, slot, :] = new_bits[b, t]
            elif kv_dtype == "fp8":
                codes, sigma = quantise_rows_fp8(new_bits[b, t][None, :])
                out[page, slot * D_QK:(slot + 1) * D_QK] = codes[0]
                out[page, FP8_DATA_BYTES + 4 * slot:FP8_DATA_BYTES + 4 * slot + 4] = (
                    sigma.astype("<f4").view(np.uint8))
            else:
                raise ValueError(kv_dtype)
    assert out.shape[1:] == ((PAGE, D_QK) if kv_dtype == "bf16" else (FP8_PAGE_BYTES,))
    return out
