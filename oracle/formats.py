"""Expert weight formats besides MXFP4: BF16 and NVFP4 blobs, decoded to fp64.

Test infrastructure only (see the package header).

The FreeToken pages run Qwen3.6-35B-A3B with BF16 experts and an
NVFP4-quantised build of the same model (jansverre.net page, sections "Hvor
raskt kjører modellene?" and "Hvorfor er båndbredden viktigere enn antall
kjerner?"); they name the formats and define neither.  The definitions used
here are the public ones:

* BF16: the top 16 bits of an IEEE binary32 (sign, 8 exponent bits, 7 fraction
  bits), stored little-endian.
* NVFP4: e2m1 elements (the same 4-bit codes as MXFP4, element 2i in the low
  nibble), one E4M3 scale per 16 consecutive elements along K, and one fp32
  scale per matrix; an element's value is code value x block scale x matrix
  scale.  E4M3 here is the variant without infinities: sign, 4 exponent bits
  with bias 7, 3 fraction bits; exponent 0 is subnormal (m/8 x 2^-6); the one
  pattern S.1111.111 is NaN; the largest finite value is 448.  Block scales
  are non-negative (sign bit 0).

Blob layouts (one expert; the readings chosen here, so that each matrix is
K-contiguous as in the MXFP4 blob and the block scales sit in the same
128-row x 4-block atoms the tcgen05 block-scaled MMA reads):

* BF16: Wg [I][H], Wu [I][H], Wd [H][I] as bf16, then zero padding to a
  multiple of 256 bytes.
* NVFP4: codes of Wg, Wu, Wd exactly as in the MXFP4 blob; then the E4M3
  scale regions of Wg, Wu, Wd, each a whole number of 512-byte atoms of 128
  rows x 4 blocks of 16 elements (the MXFP4 atom index with 16-element
  blocks); then the three fp32 matrix scales (Wg, Wu, Wd, little-endian) and
  4 zero bytes; then zero padding to a multiple of 256 bytes.
"""
from __future__ import annotations

import math

import numpy as np

from . import fp4


def _pad(v: int, m: int) -> int:
    return -(-v // m) * m


# ---------------------------------------------------------------------------
# element decoding
# ---------------------------------------------------------------------------

def e4m3_value(byte: int) -> float:
    """Value of an E4M3 byte (no infinities; S.1111.111 is NaN)."""
    s = (byte >> 7) & 1
    e = (byte >> 3) & 15
    m = byte & 7
    if e == 15 and m == 7:
        return math.nan
    mag = math.ldexp(m / 8.0, -6) if e == 0 else math.ldexp(1.0 + m / 8.0, e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)
E4M3_TABLE[0x80] = -0.0


def bf16_value(bits: int) -> float:
    """Value of a bf16 bit pattern: sign, 8 exponent bits (bias 127), 7
    fraction bits; exponent 0 is subnormal, 255 is infinity or NaN."""
    s = (bits >> 15) & 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0xFF:
        mag = math.inf if m == 0 else math.nan
    elif e == 0:
        mag = math.ldexp(m / 128.0, -126)
    else:
        mag = math.ldexp(1.0 + m / 128.0, e - 127)
    return -mag if s else mag


# ---------------------------------------------------------------------------
# BF16 blob
# ---------------------------------------------------------------------------

def bf16_layout(hidden: int, inter: int) -> dict:
    H, I = hidden, inter
    off = {"wg": 0, "wu": 2 * I * H, "wd": 4 * I * H, "used": 6 * I * H}
    off["stride"] = _pad(off["used"], 256)
    return off


def bf16_matrix(blob: np.ndarray, which: str, hidden: int, inter: int) -> np.ndarray:
    """Wg / Wu / Wd of a BF16 blob as fp64 [rows, K] (exact)."""
    off = bf16_layout(hidden, inter)
    rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
    raw = np.asarray(blob, dtype=np.uint8)[off[which]: off[which] + 2 * rows * K].reshape(rows * K, 2)
    bits = raw[:, 0].astype(np.uint32) | (raw[:, 1].astype(np.uint32) << 8)
    return (bits << np.uint32(16)).view(np.float32).astype(np.float64).reshape(rows, K)


# ---------------------------------------------------------------------------
# NVFP4 blob
# ---------------------------------------------------------------------------

def nvfp4_layout(hidden: int, inter: int) -> dict:
    H, I = hidden, inter
    off = {"wg": 0, "wu": I * H // 2, "wd": I * H}
    end = I * H + H * I // 2
    gu_sf = _pad(I, 128) * _pad(H // 16, 4)
    d_sf = _pad(H, 128) * _pad(I // 16, 4)
    off["wg_sf"] = end
    off["wu_sf"] = end + gu_sf
    off["wd_sf"] = end + 2 * gu_sf
    off["tensor_scales"] = end + 2 * gu_sf + d_sf
    off["used"] = off["tensor_scales"] + 16
    off["stride"] = _pad(off["used"], 256)
    return off


def nvfp4_tensor_scales(blob: np.ndarray, hidden: int, inter: int) -> dict:
    """The fp32 scales of Wg, Wu, Wd."""
    off = nvfp4_layout(hidden, inter)["tensor_scales"]
    v = np.asarray(blob, dtype=np.uint8)[off: off + 12].copy().view("<f4").astype(np.float64)
    return {"wg": float(v[0]), "wu": float(v[1]), "wd": float(v[2])}


def nvfp4_matrix(blob: np.ndarray, which: str, hidden: int, inter: int) -> np.ndarray:
    """Wg / Wu / Wd of an NVFP4 blob as fp64 [rows, K]: e2m1 code value x E4M3
    scale of its 16-element block x the matrix's fp32 scale (each product is
    exact in fp64)."""
    off = nvfp4_layout(hidden, inter)
    rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
    blob = np.asarray(blob, dtype=np.uint8)
    codes = blob[off[which]: off[which] + rows * K // 2].reshape(rows, K // 2)
    elem = np.empty((rows, K), dtype=np.uint8)
    elem[:, 0::2] = codes & 0x0F
    elem[:, 1::2] = codes >> 4
    nb = K // 16
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(nb, dtype=np.int64)[None, :]
    block = E4M3_TABLE[blob[off[which + "_sf"] + fp4.scale_index(r, b, nb)]]
    ts = nvfp4_tensor_scales(blob, hidden, inter)[which]
    return fp4.E2M1_TABLE[elem] * np.repeat(block, 16, axis=1) * ts


# ---------------------------------------------------------------------------
# dispatch by format
# ---------------------------------------------------------------------------

FORMATS = ("mxfp4", "nvfp4", "bf16")


def weight_matrix(blob: np.ndarray, which: str, hidden: int, inter: int, weights: str = "mxfp4") -> np.ndarray:
    if weights == "mxfp4":
        return fp4.dequant_matrix(blob, which, hidden, inter)
    if weights == "nvfp4":
        return nvfp4_matrix(blob, which, hidden, inter)
    if weights == "bf16":
        return bf16_matrix(blob, which, hidden, inter)
    raise ValueError(f"unknown weight format {weights!r}")


# ---------------------------------------------------------------------------
# NVFP4 activations (the prefill path of NVFP4 experts)
# ---------------------------------------------------------------------------
#
# The pages name NVFP4 and do not define how activations are scaled.  The
# reading taken is the usual two-level one for a block-scaled FP4 product: a
# per-tensor fp32 scale s = amax / (448 * 6) over the whole matrix the GEMM
# reads (all tokens of x; all h rows of the layer), so that the block scale of
# the largest block lands on E4M3's largest value; per 16 values a block scale
# E4M3(amax_block / (6 s)); codes e2m1(v / (block scale * s)).  The two
# divisions are taken as multiplications by rounded reciprocals, one per
# tensor and one per block.  Each step is a rounding that decides a byte, so
# it is taken in fp32, as the kernel takes it, every operation rounded to
# nearest even:
#   s  = amax / 2688                   g = 1 / (s * 6)
#   b  = amax_block * g                e = E4M3(b), ties to even, at most 448
#   dq = E4M3 value of e * s           r = 1 / dq
#   code = e2m1(v * r), ties to even, saturating at 6, sign kept
# A tensor whose largest magnitude is below 2^-100 quantises to zero (s = 0,
# every byte 0), which keeps g, r and the products finite; a block with
# dq == 0 has all codes +0.
# Dequantised value: code x block scale x s.

NVFP4_GLOBAL_DIV = np.float32(448.0 * 6.0)
_E4M3_POS = E4M3_TABLE[:0x7F]          # bytes 0x00 .. 0x7e: 0 .. 448, ascending


def e4m3_round(v: float) -> int:
    """E4M3 byte of v >= 0 by brute force: the nearest of the 127 finite
    non-negative values, ties to the even byte (even mantissa), values at or
    above 448 saturating to 448 (0x7e)."""
    if v >= 448.0:
        return 0x7E
    best = None
    for b in range(0x7F):
        d = abs(v - _E4M3_POS[b])
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    return best[1]


def e4m3_round_vec(v: np.ndarray) -> np.ndarray:
    """Vectorised ``e4m3_round`` (v >= 0): the two table neighbours of each
    value, the nearer one, ties to the even byte."""
    v = np.asarray(v, dtype=np.float64)
    hi = np.clip(np.searchsorted(_E4M3_POS, v, side="left"), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    dl = np.abs(v - _E4M3_POS[lo])
    dh = np.abs(_E4M3_POS[hi] - v)
    pick = np.where(dl < dh, lo, np.where(dh < dl, hi, np.where(lo % 2 == 0, lo, hi)))
    return np.where(v >= 448.0, 0x7E, pick).astype(np.uint8)


NVFP4_MIN_AMAX = 2.0 ** -100


def nvfp4_global_scale(amax) -> np.float32:
    """Per-tensor scale: fp32(amax) / 2688, one fp32 division; 0 below 2^-100."""
    a = np.float32(amax)
    if not a >= NVFP4_MIN_AMAX:
        return np.float32(0.0)
    return np.float32(a / NVFP4_GLOBAL_DIV)


def nvfp4_quantize_rows(v: np.ndarray, s=None) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """Quantise v [R, K] (values exact in fp32) to NVFP4: element codes [R, K],
    E4M3 block-scale bytes [R, K/16] and the per-tensor scale s (fp32; None:
    from the maximum magnitude of v)."""
    v32 = np.asarray(v, dtype=np.float32)
    R, K = v32.shape
    if s is None:
        s = nvfp4_global_scale(np.abs(v32).max() if v32.size else 0.0)
    s = np.float32(s)
    blocks = v32.reshape(R, K // 16, 16)
    if s == 0:
        return np.zeros((R, K), np.uint8), np.zeros((R, K // 16), np.uint8), s
    with np.errstate(all="ignore"):
        g = np.float32(np.float32(1.0) / np.float32(s * np.float32(6.0)))
        b = (np.abs(blocks).max(axis=-1) * g).astype(np.float32)
        e = e4m3_round_vec(b)
        dq = (E4M3_TABLE[e].astype(np.float32) * s).astype(np.float32)
        r = (np.float32(1.0) / np.where(dq > 0, dq, np.float32(1.0))).astype(np.float32)
        q = (blocks * r[..., None]).astype(np.float32)
    mag = fp4.round_to_grid_vec(np.abs(q).astype(np.float64))
    codes = mag | np.where(np.signbit(q), 8, 0)
    codes = np.where((dq > 0)[..., None], codes, 0).astype(np.uint8).reshape(R, K)
    return codes, e.astype(np.uint8), s


def nvfp4_dequant_rows(codes: np.ndarray, scales: np.ndarray, s) -> np.ndarray:
    """Inverse of ``nvfp4_quantize_rows`` in fp64 (exact products)."""
    return fp4.E2M1_TABLE[codes] * np.repeat(E4M3_TABLE[scales], 16, axis=1) * float(np.float32(s))
