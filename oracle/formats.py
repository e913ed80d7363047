"""Number formats used by NVFP4: E2M1 elements, E4M3 block scales, BF16, FP32.

Oracle module (test infrastructure only, see ``oracle/__init__``).

[QUADS-fr §1] and [QUADS-es §1] state that the FP4 element grid is E2M1 with
only eight non-negative representable levels per sign; [format] fixes those
levels to {0, 0.5, 1, 1.5, 2, 3, 4, 6}, the block scale to E4M3 (bias 7,
max 448, no infinities) and round-to-nearest-even with saturation.
"""
import numpy as np

# The eight non-negative E2M1 magnitudes, indexed by the 3-bit code.
E2M1_LEVELS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
E4M3_MAX = 448.0
# 6 * 448: the largest block scale times the largest element.
NVFP4_RANGE = E2M1_MAX * E4M3_MAX


def f32(v):
    """Round float64 values to float32 (round-to-nearest-even), kept in float64.

    Used after every operation that the method performs in float32."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_rne(v):
    """Round float32 values to bfloat16 (nearest, ties to even), returned as float64.

    Done on the bit pattern: add 0x7fff plus the bit that becomes the last
    kept mantissa bit, then drop the 16 low bits."""
    u = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def bf16_bits(v):
    """BF16 bit patterns (uint16) of float values that are already BF16-exact."""
    u = np.asarray(v, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_from_bits(b):
    """Float64 values of BF16 bit patterns."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def e2m1_value(code):
    """Value of 4-bit E2M1 codes: bit 3 is the sign, bits 0-2 index the levels."""
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_LEVELS[code & 7]
    return np.where(code & 8, -mag, mag)


def e2m1_rne_code(v):
    """Round float values to E2M1 codes: nearest level, ties to the even code,
    magnitudes above 6 saturate to 6, the sign bit follows the input's sign
    (so -0.1 gives code 8, negative zero)."""
    v = np.asarray(v, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    lo_idx = np.clip(np.searchsorted(E2M1_LEVELS, a, side="right") - 1, 0, 7)
    hi_idx = np.minimum(lo_idx + 1, 7)
    lo = E2M1_LEVELS[lo_idx]
    hi = E2M1_LEVELS[hi_idx]
    d_lo = a - lo
    d_hi = hi - a
    go_up = (d_hi < d_lo) | ((d_hi == d_lo) & (lo_idx % 2 == 1))
    idx = np.where(a >= E2M1_MAX, 7, lo_idx + go_up.astype(np.int64))
    return (neg.astype(np.int64) << 3 | idx).astype(np.uint8)


def e4m3_value(code):
    """Value of E4M3 (fn variant) codes: sign, 4 exponent bits (bias 7), 3
    mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); 0x7f/0xff are NaN."""
    code = np.asarray(code, dtype=np.int64)
    s = (code >> 7) & 1
    e = (code >> 3) & 15
    m = code & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_rn_satfinite_code(t):
    """Round non-negative float values to E4M3 codes: nearest, ties to even,
    values above 448 saturate to 448 (code 0x7e).

    The quantum in the binade [2^e, 2^(e+1)) is 2^(e-3); below the smallest
    normal 2^-6 it is the subnormal step 2^-9.  Rounding t / quantum to the
    nearest integer with ties to even rounds the last mantissa bit to even."""
    t = np.asarray(t, dtype=np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("block scale inputs must be non-negative and not NaN")
    tt = np.minimum(t, E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(tt > 0, tt, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    r = np.rint(tt / quantum) * quantum          # np.rint: ties to even
    r = np.minimum(r, E4M3_MAX)
    # encode r (exactly representable now)
    code = np.zeros(r.shape, dtype=np.int64)
    nz = r > 0
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(nz, r, 1.0)))
    sub = nz & (er < -6)
    nrm = nz & ~sub
    code = np.where(sub, np.rint(r / 2.0 ** -9), code)
    mant = np.rint((r / np.exp2(er) - 1.0) * 8.0)
    code = np.where(nrm, ((er + 7).astype(np.int64) << 3) | mant.astype(np.int64), code)
    return code.astype(np.uint8)


def pack_nibbles(codes):
    """Pack 4-bit codes two per byte along the last axis: element 2j goes to
    the low nibble of byte j, element 2j+1 to the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.shape[-1] % 2:
        raise ValueError("last axis must be even")
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """Inverse of ``pack_nibbles``."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def scale_tile_offset(row, col, n_col_tiles):
    """Byte offset of block scale (row, col) in the tiled scale layout that
    the block-scaled tensor-core MMA reads: tiles of 128 rows x 4 scales
    (512 bytes), tiles in row-major order over (row // 128, col // 4); inside
    a tile, row r and column c sit at (r % 32) * 16 + (r // 32) * 4 + c."""
    row = np.asarray(row, dtype=np.int64)
    col = np.asarray(col, dtype=np.int64)
    tile = (row // 128) * n_col_tiles + col // 4
    r = row % 128
    return tile * 512 + (r % 32) * 16 + (r // 32) * 4 + col % 4


def scales_to_tiled(scales):
    """Lay a [rows, K/16] scale matrix out in the tiled layout, padding rows to
    a multiple of 128 and columns to a multiple of 4 with zero scales."""
    s = np.asarray(scales, dtype=np.uint8)
    rows, cols = s.shape
    rp = -(-rows // 128) * 128
    cp = -(-cols // 4) * 4
    out = np.zeros(rp * cp, dtype=np.uint8)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    out[scale_tile_offset(rr, cc, cp // 4)] = s
    return out


def scales_from_tiled(flat, rows, cols):
    """Inverse of ``scales_to_tiled`` (drops the padding)."""
    cp = -(-cols // 4) * 4
    rr, cc = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
    return np.asarray(flat, dtype=np.uint8)[scale_tile_offset(rr, cc, cp // 4)]
