"""Seeded synthetic inputs for the MoE layer: expert blobs, activations, router
weights, routing traces and router logits.

This module holds no arithmetic of the method itself (no routing, no
quantisation rule, no FFN).  It only draws random bytes and numbers, so that the
CUDA path and the CPU oracle can be fed identical inputs.  Everything is keyed
by a counter-based generator (the splitmix64 finaliser applied to a counter),
so any expert of any layer can be regenerated on its own, and the CUDA filler in
``synth/pool.cu`` produces the same bytes for the same key.

Expert blobs
------------
The pages describe 4-bit experts streamed from a host pool (FreeToken pages:
"MXFP4" for DeepSeek-V4-Flash; an FP4 pool of about 140 GB).  A blob holds, for
one expert, the e2m1 codes of the gate, up and down matrices followed by their
UE8M0 block scales.  Weights ~N(0, 0.02) quantised per 32 values give block
scales near 2^-7 and codes whose magnitudes follow a quantised Gaussian of
standard deviation about 2.2 grid units; the generator draws codes and scale
bytes directly from such histograms (``MAG_COUNTS`` and ``SCALE_*`` below)
instead of quantising, because quantising is part of the method under test.

Region boundaries of a blob (``blob_regions``) follow the storage format:
codes of Wg [I, H/2], Wu [I, H/2], Wd [H, I/2], then the three scale regions,
each padded to whole 128-row x 4-block scale atoms, then zero padding to a
multiple of 256 bytes.  Scale bytes are i.i.d., so the generator needs no
knowledge of where a given row's scale sits inside a region.
"""
from __future__ import annotations

import numpy as np

M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GOLDEN = np.uint64(0x9E3779B97F4A7C15)
STREAM_MUL = np.uint64(0xD1B54A32D192ED03)

# Histogram of code magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, out of 128.
MAG_COUNTS = (12, 23, 21, 18, 23, 19, 9, 3)
MAG_CUM = np.cumsum(MAG_COUNTS).astype(np.uint64)  # thresholds on a 7-bit draw
# Scale byte = SCALE_BASE - 1, SCALE_BASE, SCALE_BASE + 1 with
# probabilities 64/256, 128/256, 64/256.
SCALE_BASE = 120

REGION_CODES = 0
REGION_SCALES = 1


def _mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function, vectorised over uint64 arrays."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def stream_base(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) ^ (np.uint64(stream & 0xFFFFFFFFFFFFFFFF) * STREAM_MUL)
    return _mix64(np.array([s], dtype=np.uint64))[0]


def words(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Counter-based 64-bit words ``w[i] = mix64(base + (i + 1) * GOLDEN)``."""
    base = stream_base(seed, stream)
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = base + (i + np.uint64(1)) * GOLDEN
    return _mix64(z)


def blob_stream(layer: int, expert: int, region: int) -> int:
    return (((layer & 0xFFFF) << 16 | (expert & 0xFFFF)) << 8) | region


def pad_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


def blob_regions(hidden: int, inter: int) -> dict:
    """Byte offsets of the regions of one expert blob (storage format)."""
    H, I = hidden, inter
    wg = 0
    wu = wg + I * H // 2
    wd = wu + I * H // 2
    codes_end = wd + H * I // 2
    sf_gu = pad_up(I, 128) * pad_up(H // 32, 4)   # one of Wg/Wu scale regions
    sf_d = pad_up(H, 128) * pad_up(I // 32, 4)
    wg_sf = codes_end
    wu_sf = wg_sf + sf_gu
    wd_sf = wu_sf + sf_gu
    used = wd_sf + sf_d
    return dict(wg=wg, wu=wu, wd=wd, codes_end=codes_end, wg_sf=wg_sf, wu_sf=wu_sf,
                wd_sf=wd_sf, used=used, stride=pad_up(used, 256))


def blob_stride(hidden: int, inter: int) -> int:
    return blob_regions(hidden, inter)["stride"]


def code_bytes(seed: int, layer: int, expert: int, nbytes: int) -> np.ndarray:
    """``nbytes`` bytes of packed e2m1 codes (two per byte, element 2i low)."""
    nw = (nbytes + 3) // 4
    w = words(seed, blob_stream(layer, expert, REGION_CODES), 0, nw)
    # each word gives four 16-bit fields -> four code bytes
    f = np.stack([(w >> np.uint64(16 * q)) & np.uint64(0xFFFF) for q in range(4)], axis=1).reshape(-1)
    lo8 = f & np.uint64(0xFF)
    hi8 = (f >> np.uint64(8)) & np.uint64(0xFF)

    def draw(b):
        mag = np.searchsorted(MAG_CUM, b & np.uint64(0x7F), side="right").astype(np.uint64)
        sign = (b >> np.uint64(7)) & np.uint64(1)
        return (sign << np.uint64(3)) | mag

    out = (draw(lo8) | (draw(hi8) << np.uint64(4))).astype(np.uint8)
    return out[:nbytes]


def scale_bytes(seed: int, layer: int, expert: int, nbytes: int) -> np.ndarray:
    nw = (nbytes + 7) // 8
    w = words(seed, blob_stream(layer, expert, REGION_SCALES), 0, nw)
    b = np.stack([(w >> np.uint64(8 * q)) & np.uint64(0xFF) for q in range(8)], axis=1).reshape(-1)
    s = np.full(b.shape, SCALE_BASE, dtype=np.int64)
    s[b < 64] = SCALE_BASE - 1
    s[b >= 192] = SCALE_BASE + 1
    return s.astype(np.uint8)[:nbytes]


def expert_blob(seed: int, layer: int, expert: int, hidden: int, inter: int) -> np.ndarray:
    """The full blob (``stride`` bytes) of one expert, as uint8."""
    r = blob_regions(hidden, inter)
    blob = np.zeros(r["stride"], dtype=np.uint8)
    blob[: r["codes_end"]] = code_bytes(seed, layer, expert, r["codes_end"])
    nsf = r["used"] - r["codes_end"]
    blob[r["codes_end"]: r["used"]] = scale_bytes(seed, layer, expert, nsf)
    return blob


# ---------------------------------------------------------------------------
# BF16 and NVFP4 expert blobs
# ---------------------------------------------------------------------------
# BF16 blob: Wg [I][H], Wu [I][H], Wd [H][I] as little-endian bf16, zero padded
# to a multiple of 256 bytes.  Each weight takes 16 random bits: 7 fraction
# bits, a sign bit and an 8-bit draw of its binade [2^e, 2^(e+1)) from
# BF16_BINADE_COUNTS (e = -14 .. -4, out of 256: the binade probabilities of
# N(0, 0.02); the lowest binade also takes the mass below it), so that the
# bytes are integer functions of the counter and a GPU filler can match them.
BF16_BINADE_COUNTS = (1, 1, 2, 5, 10, 20, 38, 67, 81, 30, 1)
BF16_BINADE_CUM = np.cumsum(BF16_BINADE_COUNTS).astype(np.uint64)
BF16_EXP_LOW = 127 - 14                      # biased exponent of the lowest binade
# NVFP4 blob: the MXFP4 code region (same code histogram), E4M3 block scales
# (one per 16 elements) drawn uniformly from NVFP4_SCALE_BYTES, then the three
# fp32 matrix scales NVFP4_TENSOR_SCALES (Wg, Wu, Wd) and 4 zero bytes.
NVFP4_SCALE_BYTES = (0x72, 0x73, 0x74, 0x75)  # 160, 176, 192, 208
NVFP4_TENSOR_SCALES = (0.875 * 2.0 ** -14, 1.125 * 2.0 ** -14, 1.375 * 2.0 ** -14)

REGION_BF16 = 2
REGION_E4M3 = 3


def bf16_blob_regions(hidden: int, inter: int) -> dict:
    H, I = hidden, inter
    used = 6 * I * H
    return dict(wg=0, wu=2 * I * H, wd=4 * I * H, used=used, stride=pad_up(used, 256))


def nvfp4_blob_regions(hidden: int, inter: int) -> dict:
    H, I = hidden, inter
    codes_end = I * H + H * I // 2
    sf_gu = pad_up(I, 128) * pad_up(H // 16, 4)
    sf_d = pad_up(H, 128) * pad_up(I // 16, 4)
    ts = codes_end + 2 * sf_gu + sf_d
    return dict(wg=0, wu=I * H // 2, wd=I * H, codes_end=codes_end, wg_sf=codes_end, wu_sf=codes_end + sf_gu,
                wd_sf=codes_end + 2 * sf_gu, tensor_scales=ts, used=ts + 16, stride=pad_up(ts + 16, 256))


def bf16_weight_bits(seed: int, layer: int, expert: int, n: int) -> np.ndarray:
    """``n`` bf16 bit patterns (uint16) of one expert's weights, in blob order."""
    w = words(seed, blob_stream(layer, expert, REGION_BF16), 0, (n + 3) // 4)
    f = np.stack([(w >> np.uint64(16 * q)) & np.uint64(0xFFFF) for q in range(4)], axis=1).reshape(-1)[:n]
    binade = np.searchsorted(BF16_BINADE_CUM, f & np.uint64(0xFF), side="right").astype(np.uint64)
    frac = (f >> np.uint64(8)) & np.uint64(0x7F)
    sign = (f >> np.uint64(15)) & np.uint64(1)
    return ((sign << np.uint64(15)) | ((binade + np.uint64(BF16_EXP_LOW)) << np.uint64(7)) | frac).astype(np.uint16)


def expert_blob_bf16(seed: int, layer: int, expert: int, hidden: int, inter: int) -> np.ndarray:
    r = bf16_blob_regions(hidden, inter)
    blob = np.zeros(r["stride"], dtype=np.uint8)
    blob[: r["used"]] = bf16_weight_bits(seed, layer, expert, r["used"] // 2).astype("<u2").view(np.uint8)
    return blob


def e4m3_scale_bytes(seed: int, layer: int, expert: int, nbytes: int) -> np.ndarray:
    w = words(seed, blob_stream(layer, expert, REGION_E4M3), 0, (nbytes + 7) // 8)
    b = np.stack([(w >> np.uint64(8 * q)) & np.uint64(0xFF) for q in range(8)], axis=1).reshape(-1)[:nbytes]
    return np.asarray(NVFP4_SCALE_BYTES, dtype=np.uint8)[(b & np.uint64(3)).astype(np.int64)]


def expert_blob_nvfp4(seed: int, layer: int, expert: int, hidden: int, inter: int) -> np.ndarray:
    r = nvfp4_blob_regions(hidden, inter)
    blob = np.zeros(r["stride"], dtype=np.uint8)
    blob[: r["codes_end"]] = code_bytes(seed, layer, expert, r["codes_end"])
    blob[r["codes_end"]: r["tensor_scales"]] = e4m3_scale_bytes(seed, layer, expert,
                                                                  r["tensor_scales"] - r["codes_end"])
    blob[r["tensor_scales"]: r["tensor_scales"] + 12] = np.asarray(NVFP4_TENSOR_SCALES, dtype="<f4").view(np.uint8)
    return blob


# ---------------------------------------------------------------------------
# wide-range MXFP4 blobs (parity tests of the extremes of the format)
# ---------------------------------------------------------------------------
# The matrices named in ``wide`` get codes uniform over all 16 e2m1 codes and
# UE8M0 scale bytes uniform over ``wide_range`` (by default 0 .. 254: every
# finite scale, 2^-127 .. 2^127); the other matrices keep the usual code
# histogram with their scale bytes moved from SCALE_BASE +- 1 to
# ``narrow_base`` +- 1.  Pure byte draws
# from the same counter-based generator (stream region REGION_WIDE).
REGION_WIDE = 4


def expert_blob_wide(seed: int, layer: int, expert: int, hidden: int, inter: int,
                     wide=("wg", "wu"), narrow_base: int = SCALE_BASE, wide_range=(0, 254)) -> np.ndarray:
    r = blob_regions(hidden, inter)
    blob = expert_blob(seed, layer, expert, hidden, inter)
    code_rng = {"wg": (r["wg"], r["wu"]), "wu": (r["wu"], r["wd"]), "wd": (r["wd"], r["codes_end"])}
    sc_rng = {"wg": (r["wg_sf"], r["wu_sf"]), "wu": (r["wu_sf"], r["wd_sf"]), "wd": (r["wd_sf"], r["used"])}
    shift = int(narrow_base) - SCALE_BASE
    for name in ("wg", "wu", "wd"):
        a, b = sc_rng[name]
        if name not in wide and shift:
            blob[a:b] = (blob[a:b].astype(np.int64) + shift).astype(np.uint8)
    n_draw = 0
    for name in wide:
        for a, b in (code_rng[name], sc_rng[name]):
            n = b - a
            w = words(seed, blob_stream(layer, expert, REGION_WIDE), n_draw, (n + 3) // 4)
            n_draw += (n + 3) // 4
            f = np.stack([(w >> np.uint64(16 * q)) & np.uint64(0xFFFF) for q in range(4)], axis=1).reshape(-1)[:n]
            if (a, b) == code_rng[name]:
                blob[a:b] = (f & np.uint64(0xFF)).astype(np.uint8)       # two uniform 4-bit codes
            else:
                lo, hi = wide_range                                       # 0 .. 254 by default
                blob[a:b] = (np.uint64(lo) + f % np.uint64(hi - lo + 1)).astype(np.uint8)
    return blob


def expert_blob_bf16_wide(seed: int, layer: int, expert: int, hidden: int, inter: int) -> np.ndarray:
    """A BF16 blob of uniform 16-bit patterns over every finite bf16 value
    (both signs, zeros, subnormals, every exponent up to 254; exponent 255,
    infinity and NaN, is moved to 254).  Byte draws from the wide stream."""
    r = bf16_blob_regions(hidden, inter)
    n = r["used"] // 2
    w = words(seed, blob_stream(layer, expert, REGION_WIDE), 0, (n + 3) // 4)
    f = np.stack([(w >> np.uint64(16 * q)) & np.uint64(0xFFFF) for q in range(4)], axis=1).reshape(-1)[:n]
    f = f.astype(np.uint16)
    inf_nan = (f & 0x7F80) == 0x7F80
    f[inf_nan] = f[inf_nan] & np.uint16(0xFF7F)          # exponent 255 -> 254
    blob = np.zeros(r["stride"], dtype=np.uint8)
    blob[: r["used"]] = f.astype("<u2").view(np.uint8)
    return blob


def expert_blob_nvfp4_wide(seed: int, layer: int, expert: int, hidden: int, inter: int,
                           wide=("wg", "wu", "wd"), tensor_scales=(2.0 ** -8, 2.0 ** -8, 2.0 ** -8)) -> np.ndarray:
    """An NVFP4 blob whose matrices named in ``wide`` get codes uniform over
    all 16 and E4M3 block-scale bytes uniform over 0x00 .. 0x7e (zero, the
    seven subnormals and every normal value up to 448); the other matrices
    keep the usual bytes.  The matrix scales are ``tensor_scales`` (Wg, Wu,
    Wd).  Byte draws from the wide stream (REGION_WIDE)."""
    r = nvfp4_blob_regions(hidden, inter)
    blob = expert_blob_nvfp4(seed, layer, expert, hidden, inter)
    code_rng = {"wg": (r["wg"], r["wu"]), "wu": (r["wu"], r["wd"]), "wd": (r["wd"], r["codes_end"])}
    sc_rng = {"wg": (r["wg_sf"], r["wu_sf"]), "wu": (r["wu_sf"], r["wd_sf"]), "wd": (r["wd_sf"], r["tensor_scales"])}
    n_draw = 0
    for name in wide:
        for a, b in (code_rng[name], sc_rng[name]):
            n = b - a
            w = words(seed, blob_stream(layer, expert, REGION_WIDE), n_draw, (n + 3) // 4)
            n_draw += (n + 3) // 4
            f = np.stack([(w >> np.uint64(16 * q)) & np.uint64(0xFFFF) for q in range(4)], axis=1).reshape(-1)[:n]
            if (a, b) == code_rng[name]:
                blob[a:b] = (f & np.uint64(0xFF)).astype(np.uint8)     # two uniform 4-bit codes
            else:
                blob[a:b] = (f % np.uint64(0x7F)).astype(np.uint8)     # E4M3 bytes 0x00 .. 0x7e
    blob[r["tensor_scales"]: r["tensor_scales"] + 12] = np.asarray(tensor_scales, dtype="<f4").view(np.uint8)
    return blob


# ---------------------------------------------------------------------------
# activations, router weights, traces, logits
# ---------------------------------------------------------------------------

def _rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed & 0xFFFFFFFF, tag & 0xFFFFFFFF]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    r = ((u + rounding) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations_bf16(seed: int, tag: int, T: int, H: int, std: float = 1.0) -> np.ndarray:
    """bf16 bits [T, H], values ~N(0, std) rounded to bf16."""
    x = _rng(seed, 0x1000 + tag).standard_normal((T, H), dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(x)


def router_weights(seed: int, layer: int, E: int, H: int, std: float = 0.02) -> np.ndarray:
    """fp32 [E, H] router matrix ~N(0, std)."""
    return (_rng(seed, 0x2000 + layer).standard_normal((E, H), dtype=np.float32) * np.float32(std)).astype(np.float32)


def zipf_trace(seed: int, layer: int, n_tokens: int, E: int, k: int, s: float, rho: float,
               stream: int = 0) -> np.ndarray:
    """Expert sets of one sequence at one layer: int32 [n_tokens, k].

    Popularity of expert pi[r] is proportional to 1/(r+1)^s for a random
    permutation pi of the experts.  Token t keeps each expert of token t-1 with
    probability rho, then fills up to k experts by popularity-weighted draws
    without replacement.  Row order: kept experts (in the previous order), then
    new ones in draw order.
    """
    g = _rng(seed, 0x3000 + layer * 97 + stream * 7919)
    pi = g.permutation(E)
    pop = 1.0 / np.power(np.arange(1, E + 1, dtype=np.float64), s)
    p_expert = np.empty(E)
    p_expert[pi] = pop / pop.sum()
    out = np.empty((n_tokens, k), dtype=np.int32)
    prev: list[int] = []
    for t in range(n_tokens):
        cur = [e for e in prev if g.random() < rho]
        while len(cur) < k:
            p = p_expert.copy()
            p[cur] = 0.0
            p /= p.sum()
            cur.append(int(g.choice(E, p=p)))
        out[t] = cur
        prev = cur
    return out


def logits_for_sets(seed: int, tag: int, sets: np.ndarray, E: int) -> np.ndarray:
    """fp32 router logits [T, E] whose top-k is exactly ``sets`` (in row order).

    Chosen experts get 6 - 2j/k for rank j (inside [4, 6], strictly ordered);
    the others get N(0, 1) clipped below 3.5.
    """
    T, k = sets.shape
    g = _rng(seed, 0x4000 + tag)
    lg = np.clip(g.standard_normal((T, E)), -8.0, 3.5).astype(np.float32)
    for j in range(k):
        lg[np.arange(T), sets[:, j]] = np.float32(6.0 - 2.0 * j / k)
    return lg


def near_uniform_sets(seed: int, tag: int, T: int, E: int, k: int) -> np.ndarray:
    """k distinct experts per token, uniformly at random (prefill routing)."""
    g = _rng(seed, 0x5000 + tag)
    return np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
