"""GPU parity of the prefill path (FT_ACT_MXFP4): activation quantiser into
expert segments, tcgen05 block-scaled grouped GEMMs, combine; and the
double-buffered prefetch from a pinned host pool."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

MX = ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM


def run_prefill(H, I, E, k, S, T, seed, use_router):
    """The GPU layer output [T, H] and the oracle's result on every row.  The
    oracle reads the blobs from the seeded pool copied back to the host (the
    input filler writes the numpy generator's bytes, checked here on three
    experts), which spares regenerating 256 blobs in numpy."""
    pool = synth.gpu.layer_pool(H, I, E + S, seed, 0)
    xb = synth.activations_bf16(seed, 1, T, H)
    if use_router:
        wr = synth.router_weights(seed, 0, E, H)
        lg = None
    else:
        wr = None
        lg = synth.logits_for_sets(seed, 3, synth.near_uniform_sets(seed, 0, T, E, k), E)
    with Ctx(ft.make_desc(H, I, E, k, 1, S, 0, T), None, [pool]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, torch.from_numpy(wr).cuda() if use_router else None,
                                torch.from_numpy(lg).cuda() if lg is not None else None, out, MX)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    stride = synth.blob_stride(H, I)
    host = pool.cpu().numpy()
    for e in sorted({0, E // 2, E + S - 1}):
        assert (host[e * stride:(e + 1) * stride] == synth.expert_blob(seed, 0, e, H, I)).all()

    def blob_of(e):
        return host[e * stride:(e + 1) * stride]
    r = olayer.moe_layer(xb, blob_of, H, I, E, k, logits=lg, router_w=wr, mxfp4=True,
                         shared_blob=blob_of(E) if S else None)
    return got, r


@pytest.mark.parametrize("T", [1, 7, 64, 300])
def test_prefill_small(T):
    got, r = run_prefill(256, 256, 16, 2, 0, T, 2001, True)
    assert_close(got, r["out_f64"])


def test_prefill_small_shared_expert():
    got, r = run_prefill(256, 256, 16, 4, 1, 200, 2002, False)
    assert_close(got, r["out_f64"])


def test_prefill_35b_class():
    """512 tokens at the 35B-class shape with a shared expert: every row."""
    got, r = run_prefill(2048, 512, 256, 8, 1, 512, 2003, False)
    assert_close(got, r["out_f64"])


def test_prefill_dsv4_class_4096_tokens():
    """The DSV4-class 4096-token chunk through the router GEMV: every row, so
    every expert segment and every 128-token tile of the grouped GEMMs (and
    each segment's ragged last tile) is compared."""
    got, r = run_prefill(4096, 2048, 256, 6, 0, 4096, 2004, True)
    counts = np.diff(r["offs"])
    assert (counts > 0).sum() == 256 and (counts % 128 != 0).any()
    assert_close(got, r["out_f64"])


def test_prefetch_double_buffer_matches_resident():
    """Layers served from the prefill staging buffers (prefetched from pinned
    host pools while the previous layer computes) give the same outputs as the
    same layers resident on the device."""
    H, I, E, k, L, T, seed = 256, 256, 16, 2, 4, 96, 2005
    stride = synth.blob_stride(H, I)
    host = []
    for layer in range(L):
        t = torch.empty(E * stride, dtype=torch.uint8).pin_memory()
        for e in range(E):
            t[e * stride:(e + 1) * stride] = torch.from_numpy(synth.expert_blob(seed, layer, e, H, I))
        host.append(t)
    dev = [h.cuda() for h in host]
    lgs = [torch.from_numpy(synth.logits_for_sets(seed, l, synth.near_uniform_sets(seed, l, T, E, k), E)).cuda()
           for l in range(L)]
    x0 = x_dev(synth.activations_bf16(seed, 1, T, H))
    with Ctx(ft.make_desc(H, I, E, k, L, 0, 0, T), host, None) as cs, Ctx(ft.make_desc(H, I, E, k, L, 0, 0, T), None, dev) as cr:
        # staged: prefetch layer 0, then before each layer prefetch the next one
        staged, resident = [], []
        ft.ft_prefetch_layer(cs.h, 0)
        for l in range(L):
            if l + 1 < L:
                ft.ft_prefetch_layer(cs.h, l + 1)
            o = torch.empty_like(x0)
            ft.ft_moe_layer_forward(cs.h, l, x0, T, None, lgs[l], o, MX)
            staged.append(o)
        for l in range(L):
            o = torch.empty_like(x0)
            ft.ft_moe_layer_forward(cr.h, l, x0, T, None, lgs[l], o, MX)
            resident.append(o)
        torch.cuda.synchronize()
        ft.ft_sync_status(cs.h)
        # a layer that was never prefetched (layer 1 left the staging buffers) is refused
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(cs.h, 1, x0, T, None, lgs[1], torch.empty_like(x0), MX)
        assert e.value.status == ft.FT_ERR_NOT_FOUND
        for l in range(L):
            a, b = bf16_bits(staged[l]), bf16_bits(resident[l])
            assert np.abs(b.astype(np.int32)).sum() > 0
            assert (a == b).all(), l
