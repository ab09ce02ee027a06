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


def reencode_rows(v):
    """Re-encode every 32-element block of each row of v (fp32) as above."""
    v = np.asarray(v, np.float32)
    out = np.empty(v.shape, np.float64)
    for r in range(v.shape[0]):
        for b in range(0, v.shape[1], 32):
            out[r, b:b + 32] = reencode(v[r, b:b + 32])
    return out


def gemv_fp32(w, x):
    """Block-scaled GEMV in the kernel's precision: per 32-element block an fp32
    sum of exact products, the blocks then summed in fp32 in ascending order."""
    w32, x32 = w.astype(np.float32), x.astype(np.float32)
    K = w.shape[1]
    acc = np.zeros(w.shape[0], np.float32)
    for b in range(0, K, 32):
        acc = acc + (w32[:, b:b + 32] * x32[b:b + 32]).sum(axis=1, dtype=np.float32)
    return acc


def test_a_35b_class_layer_under_the_decode_arithmetic_stays_inside_the_tolerance():
    """One token through a 35B-class layer (hidden 2048, intermediate 512, 8
    routed experts + 1 shared) with the decode arithmetic: bf16 x re-encoded
    per block, fp32 block sums, h = silu(g) * u in fp32 re-encoded to 11 bits,
    the combine in fp32 over the ranks in order, one bf16 rounding.  Against
    the fp64 oracle the error before that rounding is about 2e-4 (relative
    L2; mostly the 11-bit h, as the A/B with h kept in fp32 shows), while
    rounding the exact result to bf16 alone
    gives about 1.6e-3: the arithmetic raises the output's error by under 5 %
    over that floor, and the output meets the layer tolerance (max abs 2e-2,
    relative L2 2e-3)."""
    import synth
    from oracle import formats, fp4, layer
    H, I, E, k, seed = 2048, 512, 256, 8, 1002
    xb = synth.activations_bf16(seed, 1, 1, H)
    sets = synth.zipf_trace(seed, 0, 3, E, k, 1.1, 0.6)[-1:]
    lg = synth.logits_for_sets(seed, 2, sets, E)
    blobs = {int(e): synth.expert_blob(seed, 0, int(e), H, I) for e in list(sets[0]) + [E]}
    r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, logits=lg, shared_blob=blobs[E])
    x = reencode_rows(fp4.bf16_to_f64(xb))[0]
    assert np.array_equal(x, fp4.bf16_to_f64(xb)[0])             # bf16 x passes exactly

    def expert(blob, h11=True):
        g = gemv_fp32(formats.weight_matrix(blob, "wg", H, I), x)
        u = gemv_fp32(formats.weight_matrix(blob, "wu", H, I), x)
        h = (g / (np.float32(1) + np.exp(-g))) * u                 # fp32
        hq = reencode_rows(h[None, :])[0] if h11 else h.astype(np.float64)
        return gemv_fp32(formats.weight_matrix(blob, "wd", H, I), hq)

    def layer_out(h11):
        acc = np.zeros(H, np.float32)
        for j in range(k):
            acc = np.float32(r["w"][0, j]) * expert(blobs[int(r["ids"][0, j])], h11) + acc
        return acc + expert(blobs[E], h11)
    acc = layer_out(True)
    want = r["out_f64"][0]
    nrm = np.linalg.norm(want)
    pre = np.linalg.norm(acc.astype(np.float64) - want) / nrm
    # the A/B: the same arithmetic with h kept in fp32 (no 11-bit rounding)
    pre_exact_h = np.linalg.norm(layer_out(False).astype(np.float64) - want) / nrm
    print(f"relative L2 before the bf16 rounding: 11-bit h {pre:.2e}, fp32 h {pre_exact_h:.2e}")
    assert pre_exact_h < pre
    out = fp4.bf16_to_f64(fp4.round_bf16(acc.astype(np.float64)))
    rel = np.linalg.norm(out - want) / nrm
    floor = np.linalg.norm(fp4.bf16_to_f64(r["out_bits"][0]) - want) / nrm   # the exact result, rounded
    assert pre < 3e-4 and pre < floor / 5
    assert rel < 1.05 * floor
    assert np.abs(out - want).max() <= 2e-2 and rel <= 2e-3
