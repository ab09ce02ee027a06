"""GPU parity of the NVFP4 and BF16 expert formats on the decode path,
against the oracle's format decoders (oracle/formats.py): the seeded GPU
filler, the dequantisation export (bit for bit), one decode layer (per-layer
kernels), the stacked decode (dataflow kernel and per-layer kernels, bit for
bit against layer by layer), and the expert cache over a host pool.

Pages: Qwen3.6-35B-A3B runs as BF16 experts and as an NVFP4-quantised build
(jansverre.net, "Hvor raskt kjører modellene?" and "Hvorfor er båndbredden
viktigere enn antall kjerner?"); the formats' definitions are the public
ones (see oracle/formats.py)."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import formats, lru as olru
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

FMT = {"nvfp4": ft.FT_FMT_NVFP4, "bf16": ft.FT_FMT_BF16}
GEN = {"nvfp4": synth.expert_blob_nvfp4, "bf16": synth.expert_blob_bf16}


@pytest.mark.parametrize("fmt", sorted(FMT))
@pytest.mark.parametrize("H,I", [(256, 128), (2048, 512)])
def test_filler_and_dequant_bit_exact(fmt, H, I):
    stride = synth.gpu.blob_stride_format(H, I, fmt)
    t = torch.empty(3 * stride, dtype=torch.uint8, device="cuda")
    synth.gpu.fill_blobs_format(t.data_ptr(), H, I, fmt, 77, 5, 10, 3)
    torch.cuda.synchronize()
    host = t.cpu().numpy()
    for i in range(3):
        assert (host[i * stride:(i + 1) * stride] == GEN[fmt](77, 5, 10 + i, H, I)).all()
    lay = ft.ft_blob_layout_format(H, I, FMT[fmt])
    assert lay["stride"] == stride
    with Ctx(ft.make_desc(H, I, 16, 2, weight_format=FMT[fmt])) as c:
        for mat, name, shape in ((0, "wg", (I, H)), (1, "wu", (I, H)), (2, "wd", (H, I))):
            out = torch.empty(shape, dtype=torch.float32, device="cuda")
            ft.ft_debug_dequant(c.h, t[stride:2 * stride], mat, out)
            want = formats.weight_matrix(host[stride:2 * stride], name, H, I, fmt).astype(np.float32)
            assert (out.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all(), name


def _case(fmt, H, I, E, k, S, L, T, seed):
    pools = [synth.gpu.layer_pool(H, I, E + S, seed, layer, fmt=fmt) for layer in range(L)]
    lgs = []
    for layer in range(L):
        sets = np.stack([synth.zipf_trace(seed, layer, 3, E, k, 1.1, 0.6, stream=t)[-1] for t in range(T)])
        lgs.append(synth.logits_for_sets(seed, 10 + layer, sets, E))
    return pools, lgs


@pytest.mark.parametrize("fmt", sorted(FMT))
@pytest.mark.parametrize("T", [1, 2, 3, 16])
def test_decode_layer_against_oracle(fmt, T):
    H, I, E, k, S, seed = 2048, 512, 64, 8, 1, 6101
    pools, lgs = _case(fmt, H, I, E, k, S, 1, T, seed)
    xb = synth.activations_bf16(seed, T, T, H)
    with Ctx(ft.make_desc(H, I, E, k, 1, S, 0, 16, weight_format=FMT[fmt]), None, pools) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lgs[0]).cuda(), out, ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    stride = synth.gpu.blob_stride_format(H, I, fmt)
    host = pools[0].cpu().numpy()
    assert (host[:stride] == GEN[fmt](seed, 0, 0, H, I)).all()

    def blob_of(e):
        return host[e * stride:(e + 1) * stride]
    r = olayer.moe_layer(xb, blob_of, H, I, E, k, logits=lgs[0], shared_blob=blob_of(E), weights=fmt)
    assert_close(got, r["out_f64"])


@pytest.mark.parametrize("fmt", sorted(FMT))
@pytest.mark.parametrize("T,flags", [(1, 1), (2, 1), (3, 1), (1, 1 | ft.FT_STACK_LAYERWISE)],
                         ids=["dataflow-1", "dataflow-2", "layerwise-3", "layerwise-1"])
def test_stack_matches_layer_by_layer(fmt, T, flags):
    H, I, E, k, S, L, seed = 2048, 512, 64, 8, 1, 3, 6102
    pools, lgs = _case(fmt, H, I, E, k, S, L, T, seed)
    lg_all = torch.from_numpy(np.stack(lgs)).cuda()
    xb = synth.activations_bf16(seed, 1, T, H)
    with Ctx(ft.make_desc(H, I, E, k, L, S, 0, 16, weight_format=FMT[fmt]), None, pools) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, out, flags)
        ft.ft_sync_status(c.h)
        cur, inputs = x, []
        for layer in range(L):
            inputs.append(bf16_bits(cur))
            nxt = torch.empty_like(x)
            ft.ft_moe_layer_forward(c.h, layer, cur, T, None, lg_all[layer], nxt, 1)
            cur = nxt
        ft.ft_sync_status(c.h)
        torch.cuda.synchronize()
        assert (bf16_bits(out) == bf16_bits(cur)).all()
    stride = synth.gpu.blob_stride_format(H, I, fmt)
    host = pools[L - 1].cpu().numpy()

    def blob_of(e):
        return host[e * stride:(e + 1) * stride]
    r = olayer.moe_layer(inputs[-1], blob_of, H, I, E, k, logits=lgs[-1], shared_blob=blob_of(E), weights=fmt)
    assert_close(bf16_bits(out), r["out_f64"])


@pytest.mark.parametrize("fmt", sorted(FMT))
def test_cache_path_against_oracle_lru_and_resident(fmt):
    H, I, E, k, L, seed = 256, 128, 16, 2, 3, 6103
    stride = synth.gpu.blob_stride_format(H, I, fmt)
    dp = [synth.gpu.layer_pool(H, I, E, seed, layer, fmt=fmt) for layer in range(L)]
    hp = [d.cpu().pin_memory() for d in dp]
    cap = 6
    ref = olru.LRUCache(cap)
    with Ctx(ft.make_desc(H, I, E, k, L, 0, cap * stride, 2, weight_format=FMT[fmt]), hp, None) as cache, \
            Ctx(ft.make_desc(H, I, E, k, L, 0, 0, 2, weight_format=FMT[fmt]), None, dp) as res:
        for step in range(30):
            layer, T = step % L, 1 + step % 2
            sets = np.stack([synth.zipf_trace(seed, layer, 30, E, k, 1.0, 0.5, stream=t)[step] for t in range(T)])
            lg = synth.logits_for_sets(seed, step, sets, E)
            x = x_dev(synth.activations_bf16(seed, step, T, H))
            lgd = torch.from_numpy(lg).cuda()
            o1, o2 = torch.empty_like(x), torch.empty_like(x)
            ft.ft_moe_layer_forward(cache.h, layer, x, T, None, lgd, o1, 1)
            ft.ft_moe_layer_forward(res.h, layer, x, T, None, lgd, o2, 1)
            torch.cuda.synchronize()
            assert (bf16_bits(o1) == bf16_bits(o2)).all(), step
            ids, _ = olayer.routing.topk(lg, k)
            assert [tuple(int(v) for v in e) for e in ft.ft_cache_trace(cache.h)] == ref.step(layer, ids.reshape(-1))
        st = ft.ft_cache_stats_get(cache.h)
        assert st["misses"] > 0 and st["h2d_bytes"] == st["misses"] * ft.ft_blob_layout_format(H, I, FMT[fmt])["used"]


@pytest.mark.parametrize("fmt", sorted(FMT))
def test_prefill_refuses_other_formats(fmt):
    H, I, E, k = 256, 256, 16, 2
    pool = synth.gpu.layer_pool(H, I, E, 1, 0, fmt=fmt)
    with Ctx(ft.make_desc(H, I, E, k, 1, 0, 0, 64, weight_format=FMT[fmt]), None, [pool]) as c:
        x = torch.zeros((64, H), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(c.h, 0, x, 64, None, torch.zeros((64, E), device="cuda"), torch.empty_like(x),
                                    ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM)
        assert e.value.status == ft.FT_ERR_INVALID and "MXFP4 weights only" in str(e.value)


def test_wide_bf16_dequant_bit_exact():
    """Every finite bf16 bit pattern class (zeros, subnormals, each exponent up
    to 254, both signs) through the decode tile's BF16 staging and its exact
    widening to fp32, against the oracle, bit for bit."""
    H, I = 2048, 512
    blob = synth.expert_blob_bf16_wide(6301, 0, 1, H, I)
    d = torch.from_numpy(blob).cuda()
    with Ctx(ft.make_desc(H, I, 16, 2, weight_format=ft.FT_FMT_BF16)) as c:
        for mat, name, shape in ((0, "wg", (I, H)), (1, "wu", (I, H)), (2, "wd", (H, I))):
            out = torch.empty(shape, dtype=torch.float32, device="cuda")
            ft.ft_debug_dequant(c.h, d, mat, out)
            want = formats.weight_matrix(blob, name, H, I, "bf16").astype(np.float32)
            assert (out.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all(), name
