"""The GLM-5.2-class slice (hidden 6144, 256 experts top-8, intermediate
2048; 20 MB blobs) on the GPU: a 2048-token prefill chunk against the oracle
on every row, and the decode cache path over pinned host pools against the
oracle LRU (every event) and the resident path (every output bit).

Page: GLM-5.2 has about 753B parameters with about 40B active per token and
runs on one workstation GPU with its experts offloaded (aiforradalom.hu, "A
Mixture-of-Experts (MoE) kihívásai és a FreeToken megoldásai")."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import layer as olayer
from oracle import lru as olru

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, SEED = 6144, 2048, 256, 8, 1005


def test_glm_class_prefill_2048_tokens_every_row():
    T = 2048
    pool = synth.gpu.layer_pool(H, I, E, SEED, 0)
    xb = synth.activations_bf16(SEED, 1, T, H)
    lg = synth.logits_for_sets(SEED, 3, synth.near_uniform_sets(SEED, 0, T, E, K), E)
    with Ctx(ft.make_desc(H, I, E, K, 1, 0, 0, T), None, [pool]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lg).cuda(), out,
                                ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
    stride = synth.blob_stride(H, I)
    host = pool.cpu().numpy()
    for e in (0, E - 1):
        assert (host[e * stride:(e + 1) * stride] == synth.expert_blob(SEED, 0, e, H, I)).all()
    r = olayer.moe_layer(xb, lambda e: host[e * stride:(e + 1) * stride], H, I, E, K, logits=lg, mxfp4=True)
    assert_close(got, r["out_f64"])


def test_glm_class_cache_trace_and_outputs():
    """3 layers with the slice's slot share (24 GiB = 1285 slots over 8
    layers, scaled to 3: 481 slots), 32 tokens of a Zipf(1.1) / 0.6-overlap
    trace.  The 32 tokens touch fewer distinct experts than that share, so the
    budget is cut to 48 slots at token 12 (evicting down to the 48 most recent
    keys, then every miss evicts) and restored at token 24; the last step's
    output against the oracle on its own input."""
    L, n_tok = 3, 32
    stride = synth.blob_stride(H, I)
    slots = 1285 * L // 8
    hp, dp = [], []
    for layer in range(L):
        d = synth.gpu.layer_pool(H, I, E, SEED, layer)
        h = torch.empty(d.numel(), dtype=torch.uint8).pin_memory()
        h.copy_(d)
        hp.append(h)
        dp.append(d)
    torch.cuda.synchronize()
    sets = np.stack([synth.zipf_trace(SEED, layer, n_tok, E, K, 1.1, 0.6) for layer in range(L)], axis=1)
    cache = Ctx(ft.make_desc(H, I, E, K, L, 0, slots * stride, 1), hp, None)
    res = Ctx(ft.make_desc(H, I, E, K, L, 0, 0, 1), None, dp)
    ref = olru.LRUCache(slots)
    try:
        x = x_dev(synth.activations_bf16(SEED, 2, 1, H))
        for p in range(n_tok):
            if p == 12:
                ft.ft_expert_cache_resize(cache.h, 48 * stride)
                assert [tuple(int(v) for v in e) for e in ft.ft_cache_trace(cache.h)] == ref.resize(48)
            if p == 24:
                ft.ft_expert_cache_resize(cache.h, slots * stride)
                ft.ft_cache_trace(cache.h)
                ref.resize(slots)
            for layer in range(L):
                lg = synth.logits_for_sets(SEED, p * 100 + layer, sets[p, layer][None], E)
                lgd = torch.from_numpy(lg).cuda()
                x_in = bf16_bits(x)
                o1, o2 = torch.empty_like(x), torch.empty_like(x)
                ft.ft_moe_layer_forward(cache.h, layer, x, 1, None, lgd, o1, ft.FT_ROUTE_RENORM)
                ft.ft_moe_layer_forward(res.h, layer, x, 1, None, lgd, o2, ft.FT_ROUTE_RENORM)
                torch.cuda.synchronize()
                assert (bf16_bits(o1) == bf16_bits(o2)).all(), (p, layer)
                ids, _ = olayer.routing.topk(lg, K)
                want = ref.step(layer, ids.reshape(-1))
                assert [tuple(int(v) for v in e) for e in ft.ft_cache_trace(cache.h)] == want, (p, layer)
                x = o1
        st = ft.ft_cache_stats_get(cache.h)
        assert st["misses"] > 0 and st["evictions"] > 0
        # layer-local oracle parity of the last step (layer L - 1, its own input)
        host = hp[L - 1].numpy()
        r = olayer.moe_layer(x_in, lambda e: host[e * stride:(e + 1) * stride], H, I, E, K, logits=lg)
        assert_close(bf16_bits(x), r["out_f64"])
    finally:
        cache.close()
        res.close()
