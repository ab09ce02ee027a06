"""The prefill (MXFP4-activation) arithmetic against the oracle, on the CPU.
The oracle quantises x and h to MXFP4 itself, so a GPU that accumulates in
fp32 can differ from it only where an h value lands close enough to an e2m1
rounding boundary for the fp32 sums to move it across.  A numpy model of the
tensor-core path (exact FP4 x FP4 products, fp32 sums over K, h = silu(g) * u
in fp32, h quantised by the oracle's rule, fp32 down and combine, one bf16
rounding) on a 35B-class-width layer shows that this does not happen here:
no h code differs, and the output's error is the bf16 rounding floor."""
import numpy as np

import synth
from oracle import fp4, layer


def test_fp32_prefill_arithmetic_flips_no_h_code_and_sits_on_the_rounding_floor():
    H, I, E, k, T, seed = 2048, 512, 16, 2, 128, 2003
    xb = synth.activations_bf16(seed, 1, T, H)
    wr = synth.router_weights(seed, 0, E, H)
    blobs = {e: synth.expert_blob(seed, 0, e, H, I) for e in range(E)}
    r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, router_w=wr, mxfp4=True)
    xq = fp4.dequant_rows(*fp4.quantize_rows(fp4.bf16_to_f64(xb)))
    out = np.zeros((T, H), np.float32)
    flips = total = 0
    for e in range(E):
        rows = np.nonzero((r["ids"] == e).any(axis=1))[0]
        if len(rows) == 0:
            continue
        wg, wu, wd = (fp4.dequant_matrix(blobs[e], m, H, I) for m in ("wg", "wu", "wd"))
        x32 = xq[rows].astype(np.float32)
        g, u = x32 @ wg.astype(np.float32).T, x32 @ wu.astype(np.float32).T
        h32 = (g / (np.float32(1) + np.exp(-g))) * u
        h64 = layer.silu(xq[rows] @ wg.T) * (xq[rows] @ wu.T)
        c32, s32 = fp4.quantize_rows(h32.astype(np.float64))
        c64, s64 = fp4.quantize_rows(h64)
        flips += int((c32 != c64).sum()) + int((s32 != s64).sum())
        total += c32.size
        y = fp4.dequant_rows(c32, s32).astype(np.float32) @ wd.astype(np.float32).T
        for i, t in enumerate(rows):
            j = list(r["ids"][t]).index(e)
            out[t] = np.float32(r["w"][t, j]) * y[i] + out[t]
    assert total > 100_000 and flips == 0
    want = r["out_f64"]
    got = fp4.bf16_to_f64(fp4.round_bf16(out.astype(np.float64)))
    nrm = np.linalg.norm(want)
    rel = np.linalg.norm(got - want) / nrm
    floor = np.linalg.norm(fp4.bf16_to_f64(r["out_bits"]) - want) / nrm
    assert rel < 1.01 * floor and rel <= 2e-3 and np.abs(got - want).max() <= 2e-2
