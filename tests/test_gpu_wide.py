"""GPU parity on wide-range MXFP4 expert blobs, against the oracle: every
UE8M0 scale byte 0 .. 254 (block scales 2^-127 .. 2^127) and every e2m1 code,
through the decode kernels (per layer and the persistent stack kernel), the
prefill tcgen05 block-scaled GEMMs, and the dequantisation export.

The seeded generator draws the selected matrices' codes uniformly over all 16
codes and their scale bytes uniformly over 0 .. 254 (``synth.expert_blob_wide``).
Two variants keep the outputs finite:
* "gate_up": wide Wg and Wu; x ~ N(0, 1) * 2^-127 (mostly bf16 subnormals), so
  that a block scaled by 2^127 meets x of order 2^-127; Wd keeps the usual
  code histogram with scale bytes 109 .. 111.
* "down": wide Wd; x ~ N(0, 1); Wg and Wu scale bytes 65 .. 67, so that h
  lies in 2^-120 .. 2^-106 (normal fp32 values: fp32 arithmetic would lose
  bits below 2^-126) and a Wd block scaled by up to 2^127 meets it.  The
  prefill variant uses scale bytes 69 .. 71 (h in 2^-111 .. 2^-94, within
  MXFP4's range, whose block scale byte clamps at 0, i.e. 2^-127).
One block near the top of the scale range dominates each row, so outputs span
many binades; the layer tolerance is applied to the outputs divided by their
largest magnitude (``assert_close_scaled``).

Pages: MXFP4 weights, e2m1 values with per-32 power-of-two scales
(jansverre.net, "Hvor raskt kjører modellene?"); the partial results of the
experts are summed exactly (jansverre.net, "Hvorfor er båndbredden viktigere
enn antall kjerner?")."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
from oracle import fp4
from oracle import layer as olayer

from _gpu import Ctx, assert_close_scaled, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, S = 2048, 512, 16, 8, 1
VARIANTS = {
    "gate_up": dict(wide=("wg", "wu"), narrow_base=110, xstd=2.0 ** -127, seed=5101),
    "down": dict(wide=("wd",), narrow_base=66, xstd=1.0, seed=5102),
}
PREFILL_BASE = {"gate_up": 110, "down": 70}


def blobs_of(variant, layer, narrow_base=None):
    v = VARIANTS[variant]
    nb = v["narrow_base"] if narrow_base is None else narrow_base
    return {e: synth.expert_blob_wide(v["seed"], layer, e, H, I, wide=v["wide"], narrow_base=nb)
            for e in range(E + S)}


def pool_of(blobs):
    return torch.from_numpy(np.concatenate([blobs[e] for e in range(E + S)])).cuda()


def routing(seed, tag, T):
    sets = np.stack([np.random.default_rng([seed, tag, t]).choice(E, K, replace=False) for t in range(T)])
    return synth.logits_for_sets(seed, tag, sets, E)


def oracle_out(blobs, xb, lg, mxfp4=False):
    return olayer.moe_layer(xb, blobs.__getitem__, H, I, E, K, logits=lg, mxfp4=mxfp4,
                            shared_blob=blobs[E])["out_f64"]


@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("T", [1, 2, 4])
def test_wide_decode_layer_and_one_layer_stack(variant, T):
    """k_route + k_dec_gate_up + k_dec_down (ft_moe_layer_forward), and the
    persistent kernel on a one-layer stack, against the oracle; the two decode
    paths agree bit for bit."""
    v = VARIANTS[variant]
    blobs = blobs_of(variant, 0)
    xb = synth.activations_bf16(v["seed"], T, T, H, std=v["xstd"])
    lg = routing(v["seed"], T, T)
    want = oracle_out(blobs, xb, lg)
    with Ctx(ft.make_desc(H, I, E, K, 1, S, 0, 16), None, [pool_of(blobs)]) as c:
        x = x_dev(xb)
        lgd = torch.from_numpy(lg).cuda()
        out_l, out_s = torch.empty_like(x), torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, lgd, out_l, ft.FT_ROUTE_RENORM)
        ft.ft_moe_stack_forward(c.h, 0, 1, x, T, lgd[None].contiguous(), out_s, ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got_l, got_s = bf16_bits(out_l), bf16_bits(out_s)
    assert_close_scaled(got_l, want)
    assert (got_s == got_l).all()


@pytest.mark.parametrize("T", [1, 2, 4])
def test_wide_decode_stack_two_layers(T):
    """Two wide-Wd layers through the persistent kernel (layer 1 reads layer
    0's output from the kernel's own hand-over), bit for bit against layer by
    layer, and each layer against the oracle on the input the GPU gave it."""
    v = VARIANTS["down"]
    bl = [blobs_of("down", layer) for layer in range(2)]
    xb = synth.activations_bf16(v["seed"], 10 + T, T, H, std=v["xstd"])
    lg = np.stack([routing(v["seed"], 20 + 2 * T + layer, T) for layer in range(2)])
    with Ctx(ft.make_desc(H, I, E, K, 2, S, 0, 16), None, [pool_of(b) for b in bl]) as c:
        x = x_dev(xb)
        lgd = torch.from_numpy(lg).cuda()
        mid, out_l, out_s = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, lgd[0], mid, ft.FT_ROUTE_RENORM)
        ft.ft_moe_layer_forward(c.h, 1, mid, T, None, lgd[1], out_l, ft.FT_ROUTE_RENORM)
        ft.ft_moe_stack_forward(c.h, 0, 2, x, T, lgd, out_s, ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        mid_b, got_l, got_s = bf16_bits(mid), bf16_bits(out_l), bf16_bits(out_s)
    assert (got_s == got_l).all()
    assert_close_scaled(mid_b, oracle_out(bl[0], xb, lg[0]))
    assert_close_scaled(got_l, oracle_out(bl[1], mid_b, lg[1]))


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_wide_prefill(variant):
    """Prefill (FT_ACT_MXFP4): x and h quantised to MXFP4, tcgen05
    block-scaled GEMMs with the wide weight scales."""
    v = VARIANTS[variant]
    T = 300
    blobs = blobs_of(variant, 0, PREFILL_BASE[variant])
    xb = synth.activations_bf16(v["seed"], 99, T, H, std=v["xstd"])
    lg = routing(v["seed"], 99, T)
    with Ctx(ft.make_desc(H, I, E, K, 1, S, 0, T), None, [pool_of(blobs)]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lg).cuda(), out,
                                ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    assert_close_scaled(got, oracle_out(blobs, xb, lg, mxfp4=True))


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_wide_dequant_bit_exact(variant):
    """ft_debug_dequant (the decode tile's staging and decoder) on every code
    and every scale byte: bit patterns equal the oracle's values rounded to
    fp32 (products beyond the fp32 range are infinities on both sides)."""
    blob = blobs_of(variant, 0)[3]
    with Ctx(ft.make_desc(H, I, E, K)) as c:
        d = torch.from_numpy(blob).cuda()
        for mat, name, shape in ((0, "wg", (I, H)), (1, "wu", (I, H)), (2, "wd", (H, I))):
            out = torch.empty(shape, dtype=torch.float32, device="cuda")
            ft.ft_debug_dequant(c.h, d, mat, out)
            with np.errstate(over="ignore"):
                want = fp4.dequant_matrix(blob, name, H, I).astype(np.float32)
            assert (out.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all(), name
