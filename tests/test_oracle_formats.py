"""Pins of the oracle's BF16 and NVFP4 expert formats: exhaustive E4M3 and
bf16 decoding against torch's converters and spec values, hand-computed blob
layouts, an exhaustive NVFP4 code x scale matrix against the closed form, the
orientation and byte order of BF16 matrices, and the two-expert worked example
in both formats (same closed-form output as the MXFP4 one)."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import formats, fp4, layer

# e2m1 magnitudes of codes 0..7 (OCP MX v1.0)
E2M1_POSITIVE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def torch_e4m3(b):
    return torch.tensor(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_table_against_torch_and_spec():
    ref = torch_e4m3(np.arange(256))
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(formats.E4M3_TABLE), nan)
    assert np.array_equal(formats.E4M3_TABLE[~nan], ref[~nan])
    spec = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x40: 2.0,
            0x48: 4.0, 0xB8: -1.0, 0x72: 160.0, 0x75: 208.0}
    for b, v in spec.items():
        assert formats.E4M3_TABLE[b] == v and formats.e4m3_value(b) == v
    assert math.copysign(1.0, formats.E4M3_TABLE[0x80]) < 0 and formats.E4M3_TABLE[0x80] == 0.0


def test_bf16_values_against_torch():
    bits = np.arange(65536, dtype=np.uint32)
    ref = torch.tensor(bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16).double().numpy()
    mine = np.array([formats.bf16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    assert formats.bf16_value(0x3F80) == 1.0 and formats.bf16_value(0xC040) == -3.0
    assert formats.bf16_value(0x0001) == 2.0 ** -133


@pytest.mark.parametrize("H,I,used,stride", [(256, 128, 196608, 196608), (2048, 512, 6291456, 6291456)])
def test_bf16_layout(H, I, used, stride):
    off = formats.bf16_layout(H, I)
    assert (off["wg"], off["wu"], off["wd"], off["used"], off["stride"]) == (0, 2 * I * H, 4 * I * H, used, stride)
    assert synth.bf16_blob_regions(H, I) == {k: off[k] for k in ("wg", "wu", "wd", "used", "stride")}


@pytest.mark.parametrize("H,I,sf,ts,used,stride", [
    # codes 3HI/2; scales: Wg and Wu I x H/16 each, Wd H x I/16 (whole atoms); 16 bytes of matrix scales
    (256, 128, (49152, 51200, 53248), 55296, 55312, 55552),
    (2048, 512, (1572864, 1638400, 1703936), 1769472, 1769488, 1769728),
])
def test_nvfp4_layout(H, I, sf, ts, used, stride):
    off = formats.nvfp4_layout(H, I)
    assert (off["wg"], off["wu"], off["wd"]) == (0, I * H // 2, I * H)
    assert (off["wg_sf"], off["wu_sf"], off["wd_sf"]) == sf
    assert (off["tensor_scales"], off["used"], off["stride"]) == (ts, used, stride)
    r = synth.nvfp4_blob_regions(H, I)
    assert {k: r[k] for k in off} == off
    # 4.5 bits per weight: 4 for the code, 8 per 16 for the block scale
    assert (used - 16) * 8 == 3 * H * I * 4.5


def test_nvfp4_dequant_exhaustive_codes_times_scales():
    """Wg of a 256 x 128 blob: every 16-element block holds the 16 codes in a
    rotated order and one of the 127 non-negative finite E4M3 bytes 0x00 to
    0x7E (cycled over the blocks); the matrix scale is not a power of two.  Every element
    must equal spec e2m1 value x torch's E4M3 value x the matrix scale."""
    H, I = 256, 128
    off = formats.nvfp4_layout(H, I)
    blob = np.zeros(off["stride"], np.uint8)
    nb = H // 16
    codes = np.empty((I, H), np.uint8)
    sbyte = np.empty((I, nb), np.uint8)
    finite = [b for b in range(0x7F)]                     # 0x00 .. 0x7E
    for r in range(I):
        for b in range(nb):
            codes[r, 16 * b:16 * b + 16] = (np.arange(16) + r + b) % 16
            sbyte[r, b] = finite[(r * nb + b) % len(finite)]
            blob[off["wg_sf"] + fp4.scale_index(r, b, nb)] = sbyte[r, b]
    blob[off["wg"]:off["wg"] + I * H // 2] = fp4.pack_codes(codes).reshape(-1)
    ts = np.float32(0.1)                                  # fp32 nearest to 0.1
    blob[off["tensor_scales"]:off["tensor_scales"] + 12] = np.array([ts, 1, 1], "<f4").view(np.uint8)
    got = formats.nvfp4_matrix(blob, "wg", H, I)
    mag = np.array(E2M1_POSITIVE)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    want = mag * np.repeat(torch_e4m3(sbyte), 16, axis=1) * float(ts)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_bf16_matrix_orientation_and_byte_order():
    """Wd [H][I] of a BF16 blob: element (r, c) = 2^(r mod 16 - 8) x (1 + (c mod
    128)/128), exact in bf16, stored little-endian at (r, c) row-major."""
    H, I = 256, 128
    off = formats.bf16_layout(H, I)
    r = np.arange(H)[:, None]
    c = np.arange(I)[None, :]
    want = np.ldexp(1.0 + (c % 128) / 128.0, (r % 16) - 8)
    bits = (want.astype(np.float32).view(np.uint32) >> 16).astype("<u2")
    blob = np.zeros(off["stride"], np.uint8)
    blob[off["wd"]:off["wd"] + 2 * H * I] = bits.reshape(-1).view(np.uint8)
    assert np.array_equal(formats.bf16_matrix(blob, "wd", H, I), want)
    assert not formats.bf16_matrix(blob, "wg", H, I).any()


def _bf16_blob(H, I, g, u, d):
    """Every row of Wg / Wu / Wd holds one value at one column: (value, column)."""
    off = formats.bf16_layout(H, I)
    b = np.zeros(off["stride"], np.uint8)
    for which, rows, K, (v, col) in (("wg", I, H, g), ("wu", I, H, u), ("wd", H, I, d)):
        m = np.zeros((rows, K), np.float32)
        m[:, col] = v
        b[off[which]:off[which] + 2 * rows * K] = (m.view(np.uint32) >> 16).astype("<u2").reshape(-1).view(np.uint8)
    return b


def _nvfp4_blob(H, I, g, u, d):
    """Every row holds one code at one column, every block the same E4M3 scale
    byte, and each matrix its fp32 scale: (code, column, scale byte, matrix scale)."""
    off = formats.nvfp4_layout(H, I)
    b = np.zeros(off["stride"], np.uint8)
    ts = []
    for which, rows, K, (code, col, sb, t) in (("wg", I, H, g), ("wu", I, H, u), ("wd", H, I, d)):
        c = np.zeros((rows, K), np.uint8)
        c[:, col] = code
        b[off[which]:off[which] + rows * K // 2] = fp4.pack_codes(c).reshape(-1)
        for r in range(rows):
            for kb in range(K // 16):
                b[off[which + "_sf"] + fp4.scale_index(r, kb, K // 16)] = sb
        ts.append(t)
    b[off["tensor_scales"]:off["tensor_scales"] + 12] = np.array(ts, "<f4").view(np.uint8)
    return b


def _worked(weights, blobs):
    H = I = 32
    x = np.zeros((1, H))
    x[0, 0], x[0, 1] = 1.0, -1.0
    lg = np.array([[0.0, math.log(3.0)]], np.float32)
    r = layer.moe_layer(fp4.round_bf16(x), lambda e: blobs[e], H, I, 2, 2, logits=lg, weights=weights)
    # g0 = 1, u0 = 2 -> y0 = 0.5 * 2 silu(1); g1 = -2, u1 = -1 -> y1 = 2 * 2/(1 + e^2)
    w1 = math.exp(float(lg[0, 1])) / (1 + math.exp(float(lg[0, 1])))
    want = (1 - w1) * (0.5 * 2.0 / (1.0 + math.exp(-1.0))) + w1 * (2.0 * 2.0 / (1.0 + math.exp(2.0)))
    assert abs(want - 0.5403734107238539) < 1e-7
    assert list(r["ids"][0]) == [1, 0]
    assert np.allclose(r["out_f64"], want, rtol=1e-14, atol=0)
    assert (fp4.bf16_to_f64(r["out_bits"]) == 0.5390625).all()


def test_worked_example_bf16_weights():
    H = I = 32
    _worked("bf16", [_bf16_blob(H, I, (1.0, 0), (2.0, 0), (0.5, 0)),
                     _bf16_blob(H, I, (2.0, 1), (1.0, 1), (2.0, 0))])


def test_worked_example_nvfp4_weights():
    """The same layer with every weight split over code x block scale x matrix
    scale: expert 0 Wg = 1.0 (code 1.0) x 2.0 (0x40) x 0.5, Wu = 2.0 x 1.0 x 1.0,
    Wd = 0.5 x 0.5 (0x30) x 2.0; expert 1 Wg = 2.0 x 1.0 x 1.0, Wu = 1.0 x 4.0
    (0x48) x 0.25, Wd = 4.0 x 1.0 x 0.5."""
    H = I = 32
    _worked("nvfp4", [_nvfp4_blob(H, I, (2, 0, 0x40, 0.5), (4, 0, 0x38, 1.0), (1, 0, 0x30, 2.0)),
                      _nvfp4_blob(H, I, (4, 1, 0x38, 1.0), (2, 1, 0x48, 0.25), (6, 0, 0x38, 0.5))])


def test_new_formats_are_decode_only():
    H, I = 256, 128
    blob = synth.expert_blob_bf16(1, 0, 0, H, I)
    x = np.ones((1, H))
    layer.expert_ffn(blob, H, I, x, weights="bf16")
    with pytest.raises(ValueError):
        layer.expert_ffn(blob, H, I, x, mxfp4=True, weights="bf16")
    with pytest.raises(ValueError):
        formats.weight_matrix(blob, "wg", H, I, "fp8")
