"""The decode GEMV's activation re-encoding, as the design states it: per
32-element block one power-of-two factor maps the block's largest magnitude
into [2^14, 2^15) (biased exponent eb of the maximum, at least 15; factor
2^(141 - eb)), then each value is rounded to f16 (nearest even).  A numpy model
of that rule checks the claims the error analysis rests on: bf16 inputs come
back exactly down to 2^-28 of their block's maximum, fp32 inputs keep 11
significant bits, and nothing overflows f16."""
import numpy as np


def reencode(block):
    """Round trip of one 32-element fp32 block through the f16 re-encoding."""
    bits = block.astype(np.float32).view(np.uint32)
    eb = max(int(((bits & 0x7F800000) >> 23).max()), 15)
    f = np.float32(2.0 ** (141 - eb))
    h = (block.astype(np.float32) * f).astype(np.float16)        # round to nearest even
    assert np.all(np.isfinite(h[np.isfinite(block)]))            # the scaled maximum fits f16
    return h.astype(np.float64) * 2.0 ** (eb - 141)


def bf16(x):
    b = np.asarray(x, np.float32).view(np.uint32)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)   # round to nearest even
    return b.view(np.float32)


def test_bf16_blocks_come_back_exactly_down_to_2_to_the_minus_28():
    rng = np.random.default_rng(7)
    for scale in (1e-30, 1e-8, 1.0, 3.0, 1e4, 1e30):
        for _ in range(200):
            # magnitudes spread over 28 binades below the block maximum
            x = bf16(scale * rng.standard_normal(32) * 2.0 ** rng.uniform(-28, 0, 32))
            m = np.abs(x).max()
            back = reencode(x)
            keep = np.abs(x) >= m * 2.0 ** -28
            assert np.array_equal(back[keep], x[keep].astype(np.float64))


def test_fp32_blocks_keep_11_significant_bits():
    rng = np.random.default_rng(8)
    for _ in range(500):
        x = (rng.standard_normal(32) * 2.0 ** rng.uniform(-10, 10)).astype(np.float32)
        m = np.abs(x).max()
        back = reencode(x)
        keep = np.abs(x) >= m * 2.0 ** -14           # inside f16's normal range after scaling
        rel = np.abs(back[keep] - x[keep]) / np.abs(x[keep])
        assert rel.max() <= 2.0 ** -11


def test_zero_and_tiny_blocks():
    assert np.array_equal(reencode(np.zeros(32, np.float32)), np.zeros(32))
    tiny = np.full(32, 1e-40, np.float32)              # subnormal fp32: the factor is capped, values flush
    assert np.all(np.abs(reencode(tiny)) <= 1e-40)
