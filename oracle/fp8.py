"""FP8 e4m3 ("fn" variant of the OCP 8-bit floating point formats) for the
oracle: decoding from the format's definition, and round-to-nearest-even
encoding with saturation (used for the pooled block keys of the two-stage
indexer, whose precision the pages leave open).

Definition: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
encodes subnormals m/8 * 2^-6; 0x7F and 0xFF are NaN; there is no infinity;
the largest finite magnitude is 1.75 * 2^8 = 448. The input contract of the
indexer (the pages' "lower precision" indexer, LSA section 2.1) uses these
bytes with one fp32 scale per row.
"""
import numpy as np

E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """fp64 value of every byte 0..255 (NaN for 0x7F / 0xFF)."""
    tab = np.empty(256, dtype=np.float64)
    for b in range(256):
        sign = -1.0 if (b >> 7) & 1 else 1.0
        e = (b >> 3) & 0xF
        m = b & 0x7
        if e == 0xF and m == 0x7:
            tab[b] = np.nan
        elif e == 0:
            tab[b] = sign * (m / 8.0) * 2.0 ** (1 - 7)
        else:
            tab[b] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return tab


_TABLE = e4m3_decode_table()


def e4m3_decode(b) -> np.ndarray:
    """Decode a uint8 array of e4m3 bytes to fp64 (exact)."""
    return _TABLE[np.asarray(b, dtype=np.uint8)]


# non-negative finite codes 0x00..0x7E in increasing order of value
_POS_CODES = np.arange(0x7F, dtype=np.uint8)
_POS_VALS = _TABLE[:0x7F]


def e4m3_quantize_rne(x) -> np.ndarray:
    """Encode fp32/fp64 values to e4m3 bytes: nearest representable value,
    ties to the even mantissa (even byte), magnitudes above 448 saturate to
    448. NaN inputs are not expected and raise."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN input")
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS_VALS, a, side="left")       # first value >= a
    hi = np.minimum(hi, len(_POS_VALS) - 1)
    lo = np.maximum(hi - 1, 0)
    vlo, vhi = _POS_VALS[lo], _POS_VALS[hi]
    dlo, dhi = a - vlo, vhi - a                            # exact in fp64
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((_POS_CODES[hi] & 1) == 0))
    code = np.where(a == vhi, _POS_CODES[hi], np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo]))
    sign = (x < 0) & (code != 0)
    return (code | (sign.astype(np.uint8) << 7)).astype(np.uint8)


def quantize_rows(x):
    """Per-row encoding of the indexer's inputs (the input contract of the
    lower-precision indexer, LSA section 2.1): scale = amax / 448 in fp32
    (1 for an all-zero row), bytes = e4m3_quantize_rne(x / scale) with the
    division in fp32 (IEEE round to nearest). Returns (uint8 bytes, fp32
    scales)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / scale[..., None]).astype(np.float32)
    return e4m3_quantize_rne(y), scale
