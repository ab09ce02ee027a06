"""Pins of the oracle's expert FFN and combine: a hand-built two-expert layer
whose output has a closed form, and the partition invariant of the combine."""
import math

import numpy as np

from oracle import fp4, layer
import synth


def _blob(H, I, g, u, d):
    """Blob whose every row of Wg / Wu / Wd holds one code at one column.
    g, u, d = (code, column, scale byte)."""
    off = fp4.layout(H, I)
    b = np.zeros(off["stride"], np.uint8)
    for which, rows, K, (code, col, sb) in (("wg", I, H, g), ("wu", I, H, u), ("wd", H, I, d)):
        c = np.zeros((rows, K), np.uint8)
        c[:, col] = code
        b[off[which]:off[which] + rows * K // 2] = fp4.pack_codes(c).reshape(-1)
        for r in range(rows):
            for kb in range(K // 32):
                b[off[which + "_sf"] + fp4.scale_index(r, kb, K // 32)] = sb
    return b


def worked_example():
    """H = I = 32, two experts, top-2, one token x = e0 - e1, logits (0, ln 3).
    Expert 0: Wg rows 1.0 at column 0, Wu rows 2.0 at column 0, Wd rows 0.5 at
    column 0 (all scales 2^0).  Expert 1: Wg rows 2.0 at column 1, Wu rows 1.0
    at column 1 (scale 2^0), Wd rows code 4.0 at column 0 with scale 2^-1."""
    H = I = 32
    b0 = _blob(H, I, (2, 0, 127), (4, 0, 127), (1, 0, 127))
    b1 = _blob(H, I, (4, 1, 127), (2, 1, 127), (6, 0, 126))
    x = np.zeros((1, H))
    x[0, 0], x[0, 1] = 1.0, -1.0
    lg = np.array([[0.0, math.log(3.0)]], np.float32)
    return H, I, [b0, b1], fp4.round_bf16(x), lg


def test_worked_example_decode():
    H, I, blobs, xb, lg = worked_example()
    r = layer.moe_layer(xb, lambda e: blobs[e], H, I, 2, 2, logits=lg)
    # closed form: g0=1,u0=2 -> h0 = 2 silu(1); y0 = 0.5 h0.  g1=-2,u1=-1 ->
    # h1 = 2/(1+e^2); y1 = 2 h1.  out = y0/4 + 3 y1/4.
    w1 = math.exp(float(lg[0, 1])) / (1 + math.exp(float(lg[0, 1])))
    y0 = 0.5 * 2.0 / (1.0 + math.exp(-1.0))
    y1 = 2.0 * 2.0 / (1.0 + math.exp(2.0))
    want = (1 - w1) * y0 + w1 * y1
    assert abs(want - 0.5403734107238539) < 1e-7
    assert list(r["ids"][0]) == [1, 0]
    assert np.allclose(r["out_f64"], want, rtol=1e-14, atol=0)
    assert (fp4.bf16_to_f64(r["out_bits"]) == 0.5390625).all()


def test_worked_example_mxfp4():
    H, I, blobs, xb, lg = worked_example()
    r = layer.moe_layer(xb, lambda e: blobs[e], H, I, 2, 2, logits=lg, mxfp4=True)
    # x quantises exactly; h0 = 1.4621 -> scale 2^-2, 5.85 -> 6 -> 1.5, y0 = 0.75;
    # h1 = 0.2384 -> scale 2^-5, 7.63 saturates to 6 -> 0.1875, y1 = 0.375.
    w1 = math.exp(float(lg[0, 1])) / (1 + math.exp(float(lg[0, 1])))
    want = (1 - w1) * 0.75 + w1 * 0.375
    assert np.allclose(r["out_f64"], want, rtol=1e-14, atol=0)
    assert (fp4.bf16_to_f64(r["out_bits"]) == 0.46875).all()


def test_mxfp4_mode_sees_x_only_through_its_quantisation():
    """In MXFP4-activation mode the expert reads x only as quantise(x):
    feeding the dequantised codes instead gives the same output bit for bit
    (quantisation is idempotent on representable blocks), while x itself is
    not representable, so an expert that skipped the quantisation of x would
    give a different output."""
    H, I, seed = 256, 128, 1001
    blob = synth.expert_blob(seed, 0, 3, H, I)
    x = fp4.bf16_to_f64(synth.activations_bf16(seed, 2, 4, H))
    xq = fp4.dequant_rows(*fp4.quantize_rows(x))
    assert (xq != x).mean() > 0.5
    y = layer.expert_ffn(blob, H, I, x, mxfp4=True)
    assert (layer.expert_ffn(blob, H, I, xq, mxfp4=True) == y).all()
    assert not np.allclose(layer.expert_ffn(blob, H, I, x, mxfp4=False),
                           layer.expert_ffn(blob, H, I, xq, mxfp4=False), rtol=1e-3, atol=0)


def test_partition_invariant_tiny_config():
    """Splitting a token's selected experts into any two groups, computing each
    group's weighted sum separately and adding the two gives the full output
    (the pages: partial results are summed, nothing is approximated)."""
    H, I, E, k, T, seed = 256, 128, 16, 2, 8, 1001
    blobs = {e: synth.expert_blob(seed, 0, e, H, I) for e in range(E)}
    xb = synth.activations_bf16(seed, 0, T, H)
    wr = synth.router_weights(seed, 0, E, H)
    r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, router_w=wr)
    x = fp4.bf16_to_f64(xb)
    rng = np.random.default_rng(0)
    for t in range(T):
        ys = [layer.expert_ffn(blobs[int(e)], H, I, x[t:t + 1])[0] for e in r["ids"][t]]
        for _ in range(4):
            mask = rng.random(k) < 0.5
            a = sum((r["w"][t, j] * ys[j] for j in range(k) if mask[j]), np.zeros(H))
            b = sum((r["w"][t, j] * ys[j] for j in range(k) if not mask[j]), np.zeros(H))
            full = r["out_f64"][t]
            assert np.allclose(a + b, full, rtol=1e-12, atol=1e-15)


def test_partition_invariant_with_shared_expert():
    H, I, E, k, T, seed = 256, 128, 8, 3, 3, 1002
    blobs = {e: synth.expert_blob(seed, 0, e, H, I) for e in range(E + 1)}
    xb = synth.activations_bf16(seed, 1, T, H)
    sets = np.array([[1, 5, 2], [0, 1, 7], [7, 6, 5]], np.int32)
    lg = synth.logits_for_sets(seed, 0, sets, E)
    r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, logits=lg, shared_blob=blobs[E])
    assert (r["ids"] == sets).all()
    x = fp4.bf16_to_f64(xb)
    for t in range(T):
        parts = [r["w"][t, j] * layer.expert_ffn(blobs[int(sets[t, j])], H, I, x[t:t + 1])[0] for j in range(k)]
        parts.append(layer.expert_ffn(blobs[E], H, I, x[t:t + 1])[0])
        assert np.allclose(sum(parts[::-1]), r["out_f64"][t], rtol=1e-12, atol=1e-15)


def test_swiglu_against_scipy_expit():
    import scipy.special
    z = np.linspace(-30, 30, 1001)
    assert np.allclose(layer.silu(z), z * scipy.special.expit(z), rtol=1e-13, atol=1e-300)
