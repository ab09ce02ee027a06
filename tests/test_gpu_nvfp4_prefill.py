"""GPU parity of the NVFP4 prefill path (FT_ACT_NVFP4): the two-level NVFP4
activation quantiser bit for bit (codes, E4M3 block scales, the per-tensor
scale), and the layer (per-tensor scale of x, quantiser into expert
segments, tcgen05 kind::mxf4nvf4 grouped GEMMs with the matrix scales in the
epilogues, fp32 h and its per-tensor scale, combine) against the oracle on
every row; the staged (prefetched) path bit for bit against the resident one.

Page: the NVFP4 build of Qwen3.6-35B-A3B (jansverre.net, "Hvor raskt kjører
modellene?")."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import formats, fp4
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

NV = ft.FT_ACT_NVFP4 | ft.FT_ROUTE_RENORM


@pytest.fixture(scope="module")
def ctx():
    c = Ctx(ft.make_desc(256, 128, 16, 2, 1, 0, 0, 16))
    yield c.h
    c.close()


def quantise_on_gpu(ctx, x):
    R, K = x.shape
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(fp4._pad(max(R, 1), 128) * (K // 16), dtype=torch.uint8, device="cuda")
    ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ft.ft_quantize_nvfp4(ctx, torch.from_numpy(x).cuda(), R, K, codes, scales, ts)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), ts.cpu().numpy()[0]


def check_quantiser(ctx, x):
    R, K = x.shape
    codes, sc, ts = quantise_on_gpu(ctx, x)
    wc, ws, wt = formats.nvfp4_quantize_rows(x)
    assert np.float32(ts).view(np.uint32) == np.float32(wt).view(np.uint32)
    assert (codes == fp4.pack_codes(wc)).all()
    r = np.arange(R)[:, None]
    b = np.arange(K // 16)[None, :]
    assert (sc[fp4.scale_index(r, b, K // 16)] == ws).all()


@pytest.mark.parametrize("R,K", [(1, 128), (7, 256), (130, 2048), (300, 512)])
def test_nvfp4_quantiser_bit_exact(ctx, R, K):
    rng = np.random.default_rng(R * 7 + K)
    x = (rng.standard_normal((R, K)) * np.exp(rng.uniform(-6, 6, (R, 1)))).astype(np.float32)
    x[0, :16] = 0.0                                      # a zero block
    x[0, 16:32] = -0.0                                   # negative zeros
    x[0, 32:48] = x[0, 32:48] * np.float32(1e-12)        # a block whose scale underflows
    check_quantiser(ctx, x)


def test_nvfp4_quantiser_ties_and_saturation(ctx):
    """Power-of-two scales so that the ties of the oracle's worked block land
    exactly: the largest magnitude 2688 gives s = 1 (see the oracle's pin);
    then every block of every row takes grid midpoints and the values above
    the block's largest representable scaled value."""
    R, K = 4, 256
    x = np.zeros((R, K), np.float32)
    x[0, 0] = 2688.0
    mids = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -6.0])
    for r in range(R):
        for blk in range(1, K // 16):
            x[r, 16 * blk:16 * blk + 16] = mids * np.float32(2.0 ** ((blk + r) % 5 - 2))
    check_quantiser(ctx, x)


def test_nvfp4_quantiser_tiny_tensor_is_zero(ctx):
    x = np.full((3, 128), 1e-31, np.float32)   # below 2^-100
    codes, sc, ts = quantise_on_gpu(ctx, x)
    assert ts == 0.0 and not codes.any() and not sc.any()


def run_nv_prefill(H, I, E, k, S, T, seed, use_router=False):
    pool = synth.gpu.layer_pool(H, I, E + S, seed, 0, fmt="nvfp4")
    xb = synth.activations_bf16(seed, 1, T, H)
    if use_router:
        wr, lg = synth.router_weights(seed, 0, E, H), None
    else:
        wr, lg = None, synth.logits_for_sets(seed, 3, synth.near_uniform_sets(seed, 0, T, E, k), E)
    with Ctx(ft.make_desc(H, I, E, k, 1, S, 0, T, weight_format=ft.FT_FMT_NVFP4), None, [pool]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, torch.from_numpy(wr).cuda() if use_router else None,
                                torch.from_numpy(lg).cuda() if lg is not None else None, out, NV)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    stride = synth.gpu.blob_stride_format(H, I, "nvfp4")
    host = pool.cpu().numpy()
    for e in sorted({0, E + S - 1}):
        assert (host[e * stride:(e + 1) * stride] == synth.expert_blob_nvfp4(seed, 0, e, H, I)).all()

    def blob_of(e):
        return host[e * stride:(e + 1) * stride]
    r = olayer.moe_layer(xb, blob_of, H, I, E, k, logits=lg, router_w=wr, weights="nvfp4", nvfp4=True,
                         shared_blob=blob_of(E) if S else None)
    return got, r


@pytest.mark.parametrize("T", [1, 7, 64, 300])
def test_nvfp4_prefill_small(T):
    got, r = run_nv_prefill(256, 256, 16, 2, 0, T, 2101, use_router=True)
    assert_close(got, r["out_f64"])


def test_nvfp4_prefill_small_shared_expert():
    got, r = run_nv_prefill(256, 256, 16, 4, 1, 200, 2102)
    assert_close(got, r["out_f64"])


def test_nvfp4_prefill_35b_class():
    """512 tokens at the 35B-class shape (the NVFP4 build's model) with a
    shared expert: every row."""
    got, r = run_nv_prefill(2048, 512, 256, 8, 1, 512, 2103)
    assert_close(got, r["out_f64"])


def test_nvfp4_prefill_dsv4_shape_1024_tokens():
    """The DSV4-class expert shape (hidden 4096, intermediate 2048, top-6 of
    256) at 1,024 tokens through the router GEMV: every row, every expert
    segment with its ragged last tile."""
    got, r = run_nv_prefill(4096, 2048, 256, 6, 0, 1024, 2104, use_router=True)
    counts = np.diff(r["offs"])
    assert (counts % 128 != 0).any()
    assert_close(got, r["out_f64"])


def test_nvfp4_prefill_flags_must_match_the_weights():
    H, I, E, k = 256, 256, 16, 2
    pool = synth.gpu.layer_pool(H, I, E, 2105, 0, fmt="nvfp4")
    mpool = synth.gpu.layer_pool(H, I, E, 2105, 0)
    lg = torch.from_numpy(synth.logits_for_sets(2105, 3, synth.near_uniform_sets(2105, 0, 8, E, k), E)).cuda()
    x = x_dev(synth.activations_bf16(2105, 1, 8, H))
    out = torch.empty_like(x)
    with Ctx(ft.make_desc(H, I, E, k, 1, 0, 0, 8, weight_format=ft.FT_FMT_NVFP4), None, [pool]) as c:
        for flags in (ft.FT_ACT_MXFP4, ft.FT_ACT_MXFP4 | ft.FT_ACT_NVFP4):
            with pytest.raises(ft.FtError) as e:
                ft.ft_moe_layer_forward(c.h, 0, x, 8, None, lg, out, flags)
            assert e.value.status == ft.FT_ERR_INVALID
    with Ctx(ft.make_desc(H, I, E, k, 1, 0, 0, 8), None, [mpool]) as c:
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(c.h, 0, x, 8, None, lg, out, ft.FT_ACT_NVFP4)
        assert e.value.status == ft.FT_ERR_INVALID


def test_nvfp4_prefill_staged_matches_resident():
    """Two NVFP4 layers served from the prefill staging buffers (prefetched
    from pinned host pools) give the resident path's output bit for bit."""
    H, I, E, k, T, L, seed = 1024, 512, 32, 4, 96, 2, 2106
    dev = [synth.gpu.layer_pool(H, I, E, seed, layer, fmt="nvfp4") for layer in range(L)]
    hp = []
    for d in dev:
        h = torch.empty(d.numel(), dtype=torch.uint8).pin_memory()
        h.copy_(d)
        hp.append(h)
    torch.cuda.synchronize()
    lgs = [torch.from_numpy(synth.logits_for_sets(seed, 10 + layer, synth.near_uniform_sets(seed, layer, T, E, k),
                                                  E)).cuda() for layer in range(L)]
    x0 = x_dev(synth.activations_bf16(seed, 1, T, H))
    desc = ft.make_desc(H, I, E, k, L, 0, 0, T, weight_format=ft.FT_FMT_NVFP4)
    outs = []
    for staged in (False, True):
        with Ctx(desc, hp if staged else None, None if staged else dev) as c:
            x = x0
            for layer in range(L):
                if staged:
                    ft.ft_prefetch_layer(c.h, layer)
                o = torch.empty_like(x)
                ft.ft_moe_layer_forward(c.h, layer, x, T, None, lgs[layer], o, NV)
                x = o
            ft.ft_sync_status(c.h)
            outs.append(bf16_bits(x))
    assert (outs[0] == outs[1]).all()
