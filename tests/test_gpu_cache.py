"""GPU parity of the expert-cache decode path: LRU event sequences against the
oracle's LRU, outputs against the resident path, resize with moves, errors."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import lru as olru
from oracle import routing

from _gpu import Ctx, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, L, SEED = 256, 128, 16, 2, 4, 2024


def host_pools(n_blobs):
    stride = synth.blob_stride(H, I)
    pools = []
    for layer in range(L):
        t = torch.empty(n_blobs * stride, dtype=torch.uint8).pin_memory()
        for e in range(n_blobs):
            t[e * stride:(e + 1) * stride] = torch.from_numpy(synth.expert_blob(SEED, layer, e, H, I))
        pools.append(t)
    return pools


def oracle_events(ev):
    return [tuple(int(v) for v in e) for e in ev]


@pytest.mark.parametrize("serial", [False, True], ids=["overlapped", "serial"])
def test_cache_trace_matches_oracle_and_resident_outputs(serial):
    """The cache path against the oracle LRU (every event) and the resident
    path (every output bit).  By default the resident experts run while the
    misses' copies are in flight and each missed expert after its own copy;
    FT_CACHE_SERIAL waits for every copy first.  Both give the same bits."""
    flags = 1 | (ft.FT_CACHE_SERIAL if serial else 0)
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    dp = [p.cuda() for p in hp]
    cap = 10
    cache = Ctx(ft.make_desc(H, I, E, K, L, 0, cap * stride + 100, 4), hp, None)
    res = Ctx(ft.make_desc(H, I, E, K, L, 0, 0, 4), None, dp)
    ref = olru.LRUCache(cap)
    traces = [[synth.zipf_trace(SEED, layer, 60, E, K, 1.0, 0.5, stream=s) for s in range(2)] for layer in range(L)]
    try:
        for step in range(60):
            if step == 30:
                ft.ft_expert_cache_resize(cache.h, 5 * stride)
                assert oracle_events(ft.ft_cache_trace(cache.h)) == ref.resize(5)
                st = ft.ft_cache_stats_get(cache.h)
                assert st["capacity_slots"] == 5 and st["used_slots"] <= 5
            if step == 45:
                ft.ft_expert_cache_resize(cache.h, cap * stride)
                assert ft.ft_cache_trace(cache.h) == []
                ref.resize(cap)
            layer = step % L
            T = 1 + (step % 2)
            sets = np.stack([traces[layer][t][step] for t in range(T)])
            lg = synth.logits_for_sets(SEED, step, sets, E)
            xb = synth.activations_bf16(SEED, step, T, H)
            x = x_dev(xb)
            lgd = torch.from_numpy(lg).cuda()
            o1 = torch.empty_like(x)
            o2 = torch.empty_like(x)
            ft.ft_moe_layer_forward(cache.h, layer, x, T, None, lgd, o1, flags)
            ft.ft_moe_layer_forward(res.h, layer, x, T, None, lgd, o2, 1)
            torch.cuda.synchronize()
            assert (bf16_bits(o1) == bf16_bits(o2)).all(), step
            ids, _ = routing.topk(lg, K)
            want = ref.step(layer, ids.reshape(-1))
            assert oracle_events(ft.ft_cache_trace(cache.h)) == want, step
        st = ft.ft_cache_stats_get(cache.h)
        assert st["misses"] > 0 and st["hits"] > 0
        assert st["h2d_bytes"] == st["misses"] * ft.ft_blob_layout(H, I)["used"]
        assert st["h2d_ms"] > 0 and 0 <= st["overlap_ms"] <= st["hit_ms"] + 1e-3
        if serial:
            assert st["hit_ms"] == 0
    finally:
        cache.close()
        res.close()


def test_cache_no_space_and_lookup_insert():
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    c = Ctx(ft.make_desc(H, I, E, K, L, 0, 1 * stride, 4), hp, None)
    try:
        x = torch.zeros((1, H), dtype=torch.bfloat16, device="cuda")
        lg = torch.zeros((1, E), dtype=torch.float32, device="cuda")
        out = torch.empty_like(x)
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(c.h, 0, x, 1, None, lg, out, 1)   # 2 experts, 1 slot
        assert e.value.status == ft.FT_ERR_NO_SPACE
        ft.ft_cache_trace(c.h)
        assert ft.ft_expert_cache_lookup(c.h, 2, 3) == -1
        slot, ev = ft.ft_expert_cache_insert(c.h, 2, 3)
        assert slot == 0 and ev == -1
        assert ft.ft_expert_cache_lookup(c.h, 2, 3) == 0
        slot, ev = ft.ft_expert_cache_insert(c.h, 1, 5)
        assert slot == 0 and ev == 2 * E + 3
        evs = ft.ft_cache_trace(c.h)
        assert evs == [(ft.FT_EV_MISS, 2, 3, 0, -1), (ft.FT_EV_HIT, 2, 3, 0, -1), (ft.FT_EV_EVICT, 2, 3, 0, -1),
                       (ft.FT_EV_MISS, 1, 5, 0, -1)]
        ft.ft_expert_cache_resize(c.h, 0)
        with pytest.raises(ft.FtError) as e:
            ft.ft_expert_cache_insert(c.h, 0, 0)
        assert e.value.status == ft.FT_ERR_NO_SPACE
        with pytest.raises(ft.FtError):
            ft.ft_expert_cache_resize(c.h, -5)
    finally:
        c.close()


def test_cache_nonfinite_logit_is_reported():
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    c = Ctx(ft.make_desc(H, I, E, K, L, 0, 8 * stride, 4), hp, None)
    try:
        x = torch.zeros((1, H), dtype=torch.bfloat16, device="cuda")
        lg = torch.zeros((1, E), dtype=torch.float32, device="cuda")
        lg[0, 4] = float("nan")
        out = torch.empty_like(x)
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(c.h, 0, x, 1, None, lg, out, 1)
        assert e.value.status == ft.FT_ERR_NONFINITE
        lg[0, 4] = 0.0
        ft.ft_moe_layer_forward(c.h, 0, x, 1, None, lg, out, 1)   # recovers
        ft.ft_sync_status(c.h)
    finally:
        c.close()


def test_cache_trace_dsv4_shape_matches_oracle():
    """The DeepSeek-V4-Flash-class cache path (hidden 4096, 256 experts top-6,
    intermediate 2048; 13.4 MB blobs from pinned host pools) on 4 layers with
    the 32 GiB budget scaled to 4 of the 43 layers (239 slots), 48 tokens of a
    Zipf(1.0) / 0.5-overlap trace, the budget halved at token 16 and restored
    at token 32: every step's HIT/MISS/EVICT/MOVE sequence equals the oracle
    LRU's, and every output equals the resident path's bit for bit."""
    H3, I3, E3, k3, L3, seed, n_tok = 4096, 2048, 256, 6, 4, 1003, 48
    stride = synth.blob_stride(H3, I3)
    slots = int(32 * 2 ** 30 * L3 / 43) // stride
    hp, dp = [], []
    for layer in range(L3):
        d = synth.gpu.layer_pool(H3, I3, E3, seed, layer)
        h = torch.empty(d.numel(), dtype=torch.uint8).pin_memory()
        h.copy_(d)
        hp.append(h)
        dp.append(d)
    torch.cuda.synchronize()
    sets = np.stack([synth.zipf_trace(seed, layer, n_tok, E3, k3, 1.0, 0.5) for layer in range(L3)], axis=1)
    xb = synth.activations_bf16(seed, 1, 1, H3)
    cache = Ctx(ft.make_desc(H3, I3, E3, k3, L3, 0, slots * stride, 1), hp, None)
    res = Ctx(ft.make_desc(H3, I3, E3, k3, L3, 0, 0, 1), None, dp)
    ref = olru.LRUCache(slots)
    n_miss = 0
    try:
        x = x_dev(xb)
        for p in range(n_tok):
            if p == n_tok // 3:
                ft.ft_expert_cache_resize(cache.h, (slots // 2) * stride)
                assert oracle_events(ft.ft_cache_trace(cache.h, cap=1 << 16)) == ref.resize(slots // 2)
            if p == 2 * n_tok // 3:
                ft.ft_expert_cache_resize(cache.h, slots * stride)
                assert ft.ft_cache_trace(cache.h) == []
                ref.resize(slots)
            for layer in range(L3):
                lg = synth.logits_for_sets(seed, p * 100 + layer, sets[p, layer][None], E3)
                lgd = torch.from_numpy(lg).cuda()
                o1, o2 = torch.empty_like(x), torch.empty_like(x)
                ft.ft_moe_layer_forward(cache.h, layer, x, 1, None, lgd, o1, ft.FT_ROUTE_RENORM)
                ft.ft_moe_layer_forward(res.h, layer, x, 1, None, lgd, o2, ft.FT_ROUTE_RENORM)
                torch.cuda.synchronize()
                assert (bf16_bits(o1) == bf16_bits(o2)).all(), (p, layer)
                ids, _ = routing.topk(lg, k3)
                want = ref.step(layer, ids.reshape(-1))
                n_miss += sum(1 for e in want if e[0] == olru.MISS)
                assert oracle_events(ft.ft_cache_trace(cache.h, cap=1 << 16)) == want, (p, layer)
                x = o1
        st = ft.ft_cache_stats_get(cache.h)
        assert st["misses"] == n_miss and st["evictions"] > 0 and st["moves"] > 0
        # steps with misses ran their resident experts during the copies
        assert st["hit_ms"] > 0 and 0 < st["overlap_ms"] <= st["hit_ms"] + 1e-3
    finally:
        cache.close()
        res.close()


@pytest.mark.parametrize("per_layer", [1, 2])
def test_cache_prefetch_matches_oracle_and_resident_outputs(per_layer):
    """Decode-time next-layer prefetch: the event sequence, PREFETCH events
    included, equals the oracle's prefetching LRU step by step; prefetch and
    prefetch-hit counts agree; every output equals the resident path's (a
    prefetched expert hit before its copy landed waits for the copy)."""
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    dp = [p.cuda() for p in hp]
    cap = 10
    cache = Ctx(ft.make_desc(H, I, E, K, L, 0, cap * stride, 4), hp, None)
    res = Ctx(ft.make_desc(H, I, E, K, L, 0, 0, 4), None, dp)
    ref = olru.PrefetchingLRUCache(cap, L, E, per_layer)
    traces = [[synth.zipf_trace(SEED, layer, 80, E, K, 1.0, 0.5, stream=s) for s in range(2)] for layer in range(L)]
    try:
        ft.ft_cache_prefetch(cache.h, per_layer)
        for step in range(80):
            if step == 40:
                ft.ft_expert_cache_resize(cache.h, 6 * stride)
                assert oracle_events(ft.ft_cache_trace(cache.h)) == ref.resize(6)
            layer = step % L
            T = 1 + (step % 2)
            sets = np.stack([traces[layer][t][step] for t in range(T)])
            lg = synth.logits_for_sets(SEED, 500 + step, sets, E)
            x = x_dev(synth.activations_bf16(SEED, 500 + step, T, H))
            lgd = torch.from_numpy(lg).cuda()
            o1, o2 = torch.empty_like(x), torch.empty_like(x)
            ft.ft_moe_layer_forward(cache.h, layer, x, T, None, lgd, o1, 1)
            ft.ft_moe_layer_forward(res.h, layer, x, T, None, lgd, o2, 1)
            torch.cuda.synchronize()
            assert (bf16_bits(o1) == bf16_bits(o2)).all(), step
            ids, _ = routing.topk(lg, K)
            assert oracle_events(ft.ft_cache_trace(cache.h)) == ref.step(layer, ids.reshape(-1)), step
        st = ft.ft_cache_stats_get(cache.h)
        assert st["prefetches"] == ref.prefetches > 0 and st["prefetch_hits"] == ref.prefetch_hits
        assert st["prefetch_bytes"] == st["prefetches"] * ft.ft_blob_layout(H, I)["used"]
    finally:
        cache.close()
        res.close()
