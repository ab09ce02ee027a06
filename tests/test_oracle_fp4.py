"""Pins of the oracle's MXFP4 decoding, storage index, quantiser and bf16
rounding against definitions that do not go through the oracle's own code."""
import math

import numpy as np
import pytest
import torch

from oracle import fp4
import synth

# OCP Microscaling spec v1.0, table of FP4 (E2M1) values: positive codes 0..7.
OCP_E2M1_POSITIVE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_table_matches_spec():
    for c in range(8):
        assert fp4.E2M1_TABLE[c] == OCP_E2M1_POSITIVE[c]
        assert fp4.E2M1_TABLE[c + 8] == -OCP_E2M1_POSITIVE[c]
    assert math.copysign(1.0, fp4.E2M1_TABLE[8]) < 0  # code 8 is -0.0


def test_ue8m0_table():
    for e in range(255):
        assert fp4.UE8M0_TABLE[e] == 2.0 ** (e - 127)
    assert math.isnan(fp4.UE8M0_TABLE[255])


def test_scale_index_hand_values():
    # offsets worked out by hand from the 128x4 atom definition (8 blocks per row)
    cases = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (64, 0): 8, (96, 0): 12,
             (0, 1): 1, (0, 3): 3, (0, 4): 512, (33, 5): 512 + 16 + 4 + 1,
             (127, 7): 512 + 31 * 16 + 3 * 4 + 3, (128, 0): 1024, (130, 5): 1536 + 32 + 1}
    for (r, kb), want in cases.items():
        assert fp4.scale_index(r, kb, 8) == want


def test_scale_index_is_a_bijection():
    rows, kb = 384, 12
    idx = {fp4.scale_index(r, b, kb) for r in range(rows) for b in range(kb)}
    assert idx == set(range(rows * kb))


@pytest.mark.parametrize("H,I,stride", [(256, 128, 52224), (2048, 512, 1671168), (4096, 2048, 13369344),
                                        (6144, 2048, 20054016)])
def test_blob_layout_sizes(H, I, stride):
    # B_e = 3*H*I*(1/2 + 1/32) for shapes whose scale regions fill whole atoms
    off = fp4.layout(H, I)
    assert off["stride"] == stride == 3 * H * I * 17 // 32
    assert off["used"] == stride
    # the input generator uses the same region boundaries
    r = synth.blob_regions(H, I)
    for k in ("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "stride"):
        assert r[k] == off[k]


def test_dequant_exhaustive_codes_times_scales():
    """Every (code, scale byte) pair, placed by the pinned index, against the
    closed form sign * magnitude * 2^(e - 127)."""
    H, I = 512, 256          # Wg is 256 rows x 16 blocks = 4096 (row, block) cells
    off = fp4.layout(H, I)
    blob = np.zeros(off["stride"], np.uint8)
    codes = np.zeros((I, H), np.uint8)
    scales = np.zeros((I, H // 32), np.int64)
    cell = 0
    for r in range(I):
        for b in range(H // 32):
            scales[r, b] = cell % 255          # bytes 0..254
            codes[r, 32 * b:32 * b + 32] = (np.arange(32) + cell) % 16
            cell += 1
    blob[off["wg"]:off["wg"] + I * H // 2] = fp4.pack_codes(codes).reshape(-1)
    for r in range(I):
        for b in range(H // 32):
            blob[off["wg_sf"] + fp4.scale_index(r, b, H // 32)] = scales[r, b]
    got = fp4.dequant_matrix(blob, "wg", H, I)
    seen = set()
    for r in range(0, I, 7):
        for k in range(H):
            c = int(codes[r, k])
            e = int(scales[r, k // 32])
            mag = OCP_E2M1_POSITIVE[c & 7]
            want = (-mag if c & 8 else mag) * 2.0 ** (e - 127)
            assert got[r, k] == want
            assert math.copysign(1, got[r, k]) == (-1 if c & 8 else 1)
            seen.add((c, e))
    # all 16 x 255 finite combinations occur somewhere in the matrix
    allpairs = {(int(codes[r, k]), int(scales[r, k // 32])) for r in range(I) for k in range(H)}
    assert len(allpairs) == 16 * 255


def test_quantiser_ties_and_saturation():
    # scaled magnitudes at grid midpoints go to the even code (spec RNE)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for a, want in ties.items():
        assert OCP_E2M1_POSITIVE[fp4._round_to_grid(a)] == want
        assert OCP_E2M1_POSITIVE[int(fp4.round_to_grid_vec(np.array([a]))[0])] == want
    for a in (6.0, 6.5, 7.99, 100.0):
        assert fp4._round_to_grid(a) == 7
    # just off a midpoint goes to the nearer value
    assert fp4._round_to_grid(0.2500001) == 1
    assert fp4._round_to_grid(4.9999) == 6


def test_quantiser_scale_rule_all_bf16_amax():
    """For every positive finite bf16 amax, amax / 2^(e-127) lies in [4, 8)
    (the block scale is floor(log2 amax) - 2) unless e is clamped."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32) << np.uint32(16)
    amax = bits.view(np.float32).astype(np.float64)
    for a in amax[::37]:
        e = fp4.block_scale_byte(float(a))
        q = a / 2.0 ** (e - 127)
        if 0 < e < 254:
            assert 4.0 <= q < 8.0
        elif e == 0:
            assert q < 8.0


def test_quantise_vectorised_matches_scalar():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((6, 128)) * np.exp(rng.uniform(-20, 20, (6, 1)))
    v[0, :32] = 0.0
    v[1, 5] = -0.0
    codes, scales = fp4.quantize_rows(v)
    for r in range(6):
        for b in range(4):
            c, e = fp4.quantize_block(v[r, 32 * b:32 * b + 32])
            assert e == scales[r, b]
            assert (c == codes[r, 32 * b:32 * b + 32]).all()


def test_quantiser_keeps_the_sign_of_values_that_round_to_zero():
    """A negative value whose scaled magnitude rounds to zero is stored as
    code 8 (-0), a positive one as code 0, in both quantiser forms: the
    element's sign bit is its input's sign bit (OCP MX: sign, then the
    rounded magnitude)."""
    v = np.zeros(32)
    v[0] = 6.0                            # amax 6: scale 2^0, the grid itself
    v[1], v[2], v[3], v[4] = -0.2, 0.2, -0.25, -0.0
    c, e = fp4.quantize_block(v)
    assert e == 127
    assert (int(c[1]), int(c[2]), int(c[3]), int(c[4])) == (8, 0, 8, 8)
    assert int(c[0]) == 7 and (c[5:] == 0).all()
    rc, rs = fp4.quantize_rows(v[None, :])
    assert (rc[0] == c).all() and int(rs[0, 0]) == 127


def test_quantise_idempotent_on_representable_blocks():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, (64, 96)).astype(np.uint8)
    codes[:, ::32] = 7          # amax of every block is 6 * scale
    scales = rng.integers(1, 250, (64, 3)).astype(np.uint8)
    v = fp4.dequant_rows(codes, scales)
    c2, s2 = fp4.quantize_rows(v)
    assert (s2 == scales).all()
    # -0 and +0 decode to the same value; compare values and signs of non-zeros
    assert (fp4.dequant_rows(c2, s2) == v).all()
    nz = (codes & 7) != 0
    assert (c2[nz] == codes[nz]).all()


def test_round_bf16_against_torch_on_fp32_exact_inputs():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 3.3895314e38, 0.0, -0.0])])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = fp4.round_bf16(v.astype(np.float64))
    assert (got == want).all()
    for x in v[:300]:
        assert fp4.round_bf16_scalar(float(x)) == fp4.round_bf16(np.array([x], np.float64))[0]


def test_round_bf16_direct_from_fp64():
    # 1 + 2^-8 + 2^-30 is above the bf16 midpoint: rounds up, whereas a detour
    # through fp32 (which drops 2^-30) would hit the tie and round to even.
    v = np.array([1 + 2 ** -8 + 2 ** -30, 1 + 2 ** -8])
    got = fp4.bf16_to_f64(fp4.round_bf16(v))
    assert got[0] == 1 + 2 ** -7
    assert got[1] == 1.0
