"""4-bit block-scaled weight format (MXFP4): decoding, storage index, quantiser.

Test infrastructure only (see the package header).

The FreeToken pages name the format only ("MXFP4" for DeepSeek-V4-Flash on the
jansverre.net page, section "Hvor raskt kjører modellene?"; "FP4 pool of about
140 GB" on the aiforradalom.hu page, section "A Mixture-of-Experts (MoE)
kihívásai és a FreeToken megoldásai").  MXFP4 is the OCP Microscaling format:
blocks of 32 e2m1 elements sharing one UE8M0 (power-of-two) scale.  Everything
below is that definition written out, in fp64.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# element and scale decoding
# ---------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """Value of a 4-bit e2m1 code: sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent 0 encodes the subnormal 0.5 * m."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = 0.5 * m if e == 0 else math.ldexp(1.0 + 0.5 * m, e - 1)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
# signed zero of code 8 is kept (numpy stores -0.0)
E2M1_TABLE[8] = -0.0


def ue8m0_value(byte: int) -> float:
    """UE8M0 block scale: 2^(byte - 127); 255 is NaN."""
    if byte == 255:
        return math.nan
    return math.ldexp(1.0, int(byte) - 127)


UE8M0_TABLE = np.array([ue8m0_value(b) for b in range(256)], dtype=np.float64)


# ---------------------------------------------------------------------------
# storage format of one expert blob
# ---------------------------------------------------------------------------

def _pad(v: int, m: int) -> int:
    return -(-v // m) * m


def layout(hidden: int, inter: int) -> dict:
    """Byte offsets of one expert blob.

    Codes, row-major with K contiguous, two elements per byte (element 2i in
    the low nibble): Wg [I, H], Wu [I, H], Wd [H, I].  Then the scale regions
    of Wg, Wu, Wd, each a whole number of 512-byte scale atoms
    (128 rows x 4 blocks).  The blob is zero-padded to a multiple of 256 bytes.
    """
    H, I = hidden, inter
    off = {}
    off["wg"] = 0
    off["wu"] = I * H // 2
    off["wd"] = 2 * (I * H // 2)
    end = off["wd"] + H * I // 2
    gu_sf = _pad(I, 128) * _pad(H // 32, 4)
    d_sf = _pad(H, 128) * _pad(I // 32, 4)
    off["wg_sf"] = end
    off["wu_sf"] = end + gu_sf
    off["wd_sf"] = end + 2 * gu_sf
    off["used"] = end + 2 * gu_sf + d_sf
    off["stride"] = _pad(off["used"], 256)
    return off


def scale_index(row: int, kblock: int, n_kblocks: int) -> int:
    """Byte offset, inside a matrix's scale region, of the scale of block
    ``kblock`` (32 elements along K) of ``row``.

    Scale atoms hold 128 rows x 4 blocks in 512 bytes: row r sits in byte group
    (r mod 32) of 16 bytes, in the 4-byte word (r mod 128) div 32, at byte
    (kblock mod 4).  Atoms run along K first, then down the rows.  This is the
    block-scale layout the tcgen05 block-scaled MMA reads through
    ``tcgen05.cp .32x128b.warpx4``.
    """
    atoms_k = _pad(int(n_kblocks), 4) // 4
    atom = (row // 128) * atoms_k + kblock // 4
    return atom * 512 + (row % 32) * 16 + ((row % 128) // 32) * 4 + kblock % 4


def dequant_matrix(blob: np.ndarray, which: str, hidden: int, inter: int) -> np.ndarray:
    """Dequantise Wg / Wu / Wd of a blob to fp64 [rows, K] (exact)."""
    off = layout(hidden, inter)
    rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
    blob = np.asarray(blob, dtype=np.uint8)
    codes = blob[off[which]: off[which] + rows * K // 2].reshape(rows, K // 2)
    elem = np.empty((rows, K), dtype=np.uint8)
    elem[:, 0::2] = codes & 0x0F
    elem[:, 1::2] = codes >> 4
    vals = E2M1_TABLE[elem]
    kb = K // 32
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(kb, dtype=np.int64)[None, :]
    scales = UE8M0_TABLE[blob[off[which + "_sf"] + scale_index(r, b, kb)]]
    return vals * np.repeat(scales, 32, axis=1)


# ---------------------------------------------------------------------------
# OCP MX quantiser (per 32 values along the last axis)
# ---------------------------------------------------------------------------

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _round_to_grid(a: float) -> int:
    """Magnitude code (0..7) of a >= 0: nearest grid value, ties to the code
    with an even mantissa bit (round-to-nearest-even), saturating at 6."""
    if a >= 6.0:
        return 7
    best = None
    for c, g in enumerate(E2M1_GRID):
        d = abs(a - g)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return best[1]


def block_scale_byte(amax: float) -> int:
    """UE8M0 scale of a block: floor(log2 amax) - emax(e2m1) with emax = 2,
    biased by 127 and clamped to [0, 254]; amax = 0 gives 0."""
    if amax == 0.0:
        return 0
    _, ex = math.frexp(amax)          # amax = m * 2^ex, m in [0.5, 1)
    return int(min(max((ex - 1) + 127 - 2, 0), 254))


def quantize_block(v: np.ndarray) -> tuple[np.ndarray, int]:
    """Quantise 32 finite values: returns (codes uint8[32], scale byte)."""
    v = np.asarray(v, dtype=np.float64)
    e = block_scale_byte(float(np.max(np.abs(v))))
    inv = math.ldexp(1.0, 127 - e)
    codes = np.empty(v.shape, dtype=np.uint8)
    for i, x in enumerate(v):
        mag = _round_to_grid(abs(x) * inv)
        codes[i] = mag | (8 if math.copysign(1.0, x) < 0 else 0)
    return codes, e


def round_to_grid_vec(a: np.ndarray) -> np.ndarray:
    """Vectorised ``_round_to_grid`` for arrays of magnitudes a >= 0: among the
    nearest grid values take the one whose code is even."""
    a = np.asarray(a, dtype=np.float64)
    d = np.abs(a[..., None] - E2M1_GRID)
    nearest = d == d.min(axis=-1, keepdims=True)
    even = nearest & (np.arange(8) % 2 == 0)
    pick_even = even.any(axis=-1)
    code = np.where(pick_even, np.argmax(even, axis=-1), np.argmax(nearest, axis=-1))
    return np.where(a >= 6.0, 7, code).astype(np.uint8)


def quantize_rows(v: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantise each row of v [R, K] in blocks of 32 (same rule as
    ``quantize_block``): element codes [R, K] and scale bytes [R, K/32]."""
    v = np.asarray(v, dtype=np.float64)
    R, K = v.shape
    blocks = v.reshape(R, K // 32, 32)
    amax = np.abs(blocks).max(axis=-1)
    _, ex = np.frexp(amax)
    e = np.clip((ex - 1) + 127 - 2, 0, 254)
    e = np.where(amax == 0.0, 0, e).astype(np.int64)
    scaled = np.abs(blocks) * np.ldexp(1.0, 127 - e)[..., None]
    mag = round_to_grid_vec(scaled)
    neg = np.signbit(blocks)
    codes = (mag | np.where(neg, 8, 0)).astype(np.uint8).reshape(R, K)
    return codes, e.astype(np.uint8)


def dequant_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Inverse of ``quantize_rows`` (element codes, not packed)."""
    return E2M1_TABLE[codes] * np.repeat(UE8M0_TABLE[scales], 32, axis=1)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Element codes [R, K] -> packed bytes [R, K/2], element 2i in the low nibble."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


# ---------------------------------------------------------------------------
# bf16 rounding of fp64 results
# ---------------------------------------------------------------------------

def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (8 significant bits, 8-bit exponent),
    nearest with ties to even, directly from fp64 (no intermediate fp32).
    Returns the bf16 bit patterns as uint16."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a == 0.0, 1.0, a))       # a in [2^(ex-1), 2^ex)
    ulp_exp = np.maximum(ex - 1, -126) - 7              # bf16 ulp; subnormals at 2^-133
    q = np.ldexp(a, -ulp_exp)                            # exact
    r = np.floor(q)
    frac = q - r
    r = r + ((frac > 0.5) | ((frac == 0.5) & (np.fmod(r, 2.0) == 1.0)))
    val = np.ldexp(r, ulp_exp)
    bits = (val.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint32)
    bits = np.where(val >= 2.0 ** 128, 0x7F80, bits)
    bits = np.where(a == 0.0, 0, bits)
    bits = bits | np.where(np.signbit(v), 0x8000, 0)
    bits = np.where(np.isnan(v), 0x7FC0, bits)
    return bits.astype(np.uint16)


def round_bf16_scalar(x: float) -> int:
    """Scalar form of ``round_bf16`` (used to pin the vectorised one)."""
    x = float(x)
    if math.isnan(x):
        return 0x7FC0
    sign = 0x8000 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a == 0.0:
        return sign
    _, ex = math.frexp(a)               # a in [2^(ex-1), 2^ex)
    q_exp = max(ex - 1, -126) - 7       # bf16 ulp; subnormals at 2^-133
    q = a / math.ldexp(1.0, q_exp)      # exact
    r = math.floor(q)
    frac = q - r
    if frac > 0.5 or (frac == 0.5 and (r & 1)):
        r += 1
    val = r * math.ldexp(1.0, q_exp)
    if val >= math.ldexp(1.0, 128):
        return sign | 0x7F80
    return sign | int(np.array([val], dtype=np.float32).view(np.uint32)[0] >> 16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)
