"""GPU parity of NVFP4 experts over the whole E4M3 scale range: block-scale
bytes uniform over 0x00 .. 0x7e (zero, the seven subnormals m * 2^-9 and
every normal value up to 448) and codes uniform over all 16
(``synth.expert_blob_nvfp4_wide``).  Through the decode tile's
dequantisation (bit for bit), a decode layer, a stacked decode against layer
by layer (bit for bit), and the NVFP4 prefill path, whose tensor cores
decode the E4M3 scales themselves; one prefill case is built so that its
outputs depend on subnormal scales alone, on both the weight and the
activation side.

Page: the NVFP4 build of Qwen3.6-35B-A3B (jansverre.net, "Hvor raskt kjører
modellene?"); the format is the public NVFP4 (see oracle/formats.py)."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
from oracle import formats
from oracle import layer as olayer

from _gpu import Ctx, assert_close_scaled, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, S, SEED = 2048, 512, 16, 4, 1, 6201
NV = ft.FT_FMT_NVFP4


def wide_blobs(layer=0):
    return {e: synth.expert_blob_nvfp4_wide(SEED, layer, e, H, I) for e in range(E + S)}


def pool_of(blobs, n):
    return torch.from_numpy(np.concatenate([blobs[e] for e in range(n)])).cuda()


def routing(tag, T):
    sets = np.stack([np.random.default_rng([SEED, tag, t]).choice(E, K, replace=False) for t in range(T)])
    return synth.logits_for_sets(SEED, tag, sets, E)


def test_wide_nvfp4_dequant_bit_exact():
    """Every E4M3 byte 0x00 .. 0x7e through the decode tile's own staging and
    decoder, against the oracle's table, bit for bit."""
    blob = synth.expert_blob_nvfp4_wide(SEED, 0, 3, H, I)
    r = synth.nvfp4_blob_regions(H, I)
    assert len(np.unique(blob[r["wg_sf"]:r["tensor_scales"]])) == 127
    d = torch.from_numpy(blob).cuda()
    with Ctx(ft.make_desc(H, I, E, K, weight_format=NV)) as c:
        for mat, name, shape in ((0, "wg", (I, H)), (1, "wu", (I, H)), (2, "wd", (H, I))):
            out = torch.empty(shape, dtype=torch.float32, device="cuda")
            ft.ft_debug_dequant(c.h, d, mat, out)
            want = formats.weight_matrix(blob, name, H, I, "nvfp4").astype(np.float32)
            assert (out.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all(), name


@pytest.mark.parametrize("T", [1, 2])
def test_wide_nvfp4_decode_layer_and_stack(T):
    """The decode layer against the oracle (outputs span many binades: the
    tolerance is taken relative to the largest); a two-layer stack against
    the same layers run one at a time, bit for bit."""
    blobs = [wide_blobs(layer) for layer in range(2)]
    pools = [pool_of(b, E + S) for b in blobs]
    xb = synth.activations_bf16(SEED, T, T, H)
    lgs = [routing(10 * T + layer, T) for layer in range(2)]
    with Ctx(ft.make_desc(H, I, E, K, 2, S, 0, 16, weight_format=NV), None, pools) as c:
        x = x_dev(xb)
        lgd = [torch.from_numpy(lg).cuda() for lg in lgs]
        o1 = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, lgd[0], o1, ft.FT_ROUTE_RENORM)
        o2 = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 1, o1, T, None, lgd[1], o2, ft.FT_ROUTE_RENORM)
        st = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, 2, x, T, torch.from_numpy(np.stack(lgs)).cuda(), st, ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got1, got2, gst = bf16_bits(o1), bf16_bits(o2), bf16_bits(st)
    want = olayer.moe_layer(xb, blobs[0].__getitem__, H, I, E, K, logits=lgs[0], shared_blob=blobs[0][E],
                            weights="nvfp4")["out_f64"]
    assert_close_scaled(got1, want)
    assert (gst == got2).all()


def test_wide_nvfp4_prefill():
    T = 96
    blobs = wide_blobs()
    xb = synth.activations_bf16(SEED, 7, T, H)
    lg = routing(77, T)
    with Ctx(ft.make_desc(H, I, E, K, 1, S, 0, T, weight_format=NV), None, [pool_of(blobs, E + S)]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lg).cuda(), out,
                                ft.FT_ACT_NVFP4 | ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    want = olayer.moe_layer(xb, blobs.__getitem__, H, I, E, K, logits=lg, shared_blob=blobs[E], weights="nvfp4",
                            nvfp4=True)["out_f64"]
    assert_close_scaled(got, want)


def test_nvfp4_prefill_honours_subnormal_scales():
    """Outputs that depend on subnormal E4M3 scales alone, on both operands
    of the block-scaled MMA.  Token 0 is 2^16 times larger than the others,
    so x's per-tensor scale leaves the other tokens' blocks with subnormal
    scales (checked below on the oracle's quantiser); token 0 is routed to
    experts 0 .. 3, whose weights are all zero, so h's per-tensor scale comes
    from the other tokens; those run on experts 4 .. 7, whose block scales
    are all subnormal (bytes 0x01 .. 0x07; matrix scale 64).  A tensor core
    that flushed subnormal scales to zero would give those tokens zero."""
    H2, I2, E2, K2, T = 256, 256, 8, 4, 16
    r = synth.nvfp4_blob_regions(H2, I2)
    rng = np.random.default_rng(SEED)
    blobs = {}
    for e in range(E2):
        b = synth.expert_blob_nvfp4(SEED, 1, e, H2, I2)
        if e < 4:
            b[:r["codes_end"]] = 0
        else:
            b[:r["codes_end"]] = rng.integers(0, 256, r["codes_end"], dtype=np.uint8)
            b[r["codes_end"]:r["tensor_scales"]] = rng.integers(1, 8, r["tensor_scales"] - r["codes_end"],
                                                                dtype=np.uint8)
            b[r["tensor_scales"]:r["tensor_scales"] + 12] = np.full(3, 64.0, "<f4").view(np.uint8)
        blobs[e] = b
    xf = rng.standard_normal((T, H2)).astype(np.float32)
    xf[0] *= np.float32(2.0 ** 16)
    xb = synth.f32_to_bf16_bits(xf)
    sets = np.stack([np.arange(4)] + [np.arange(4, 8)] * (T - 1))
    lg = synth.logits_for_sets(SEED, 5, sets, E2)
    # the other tokens' x blocks do take subnormal scales
    _, xs, _ = formats.nvfp4_quantize_rows(synth.bf16_bits_to_f32(xb))
    assert ((xs[1:] > 0) & (xs[1:] < 8)).mean() > 0.9
    with Ctx(ft.make_desc(H2, I2, E2, K2, 1, 0, 0, T, weight_format=NV), None, [pool_of(blobs, E2)]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lg).cuda(), out,
                                ft.FT_ACT_NVFP4 | ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    want = olayer.moe_layer(xb, blobs.__getitem__, H2, I2, E2, K2, logits=lg, weights="nvfp4",
                            nvfp4=True)["out_f64"]
    assert (want[0] == 0).all() and (got[0] & 0x7FFF == 0).all()
    assert np.abs(want[1:]).max() > 0
    assert_close_scaled(got[1:], want[1:])
