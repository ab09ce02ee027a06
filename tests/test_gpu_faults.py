"""Failure detection without a GPU fault: a bounded device wait that runs out
(the persistent decode kernel's wait primitive, on a flag nothing sets), a
bounded host wait that runs out while the stream is busy, and an injected
failure of a host-to-device expert copy.  Each checks the reported status and
that the context keeps working afterwards."""
import time

import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import lru as olru

from _gpu import Ctx, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

SEED = 3031


def test_device_wait_runs_out_and_the_context_stays_usable():
    H, I, E, k, L, T = 1024, 512, 64, 4, 2, 1
    pools = [synth.gpu.layer_pool(H, I, E, SEED, layer) for layer in range(L)]
    sets = [np.stack([synth.zipf_trace(SEED, layer, 3, E, k, 1.1, 0.6)[-1]]) for layer in range(L)]
    lg = torch.from_numpy(np.stack([synth.logits_for_sets(SEED, layer, sets[layer], E) for layer in range(L)])).cuda()
    x = x_dev(synth.activations_bf16(SEED, 1, T, H))
    with Ctx(ft.make_desc(H, I, E, k, L, 0, 0, 4), None, pools) as c:
        with pytest.raises(ft.FtError) as e:
            ft.ft_debug_device_wait(c.h, 0)
        assert e.value.status == ft.FT_ERR_INVALID
        t0 = time.perf_counter()
        ft.ft_debug_device_wait(c.h, 20000)            # 20 ms on a flag nothing sets
        with pytest.raises(ft.FtError) as e:
            ft.ft_sync_status(c.h)
        elapsed = time.perf_counter() - t0
        assert e.value.status == ft.FT_ERR_TIMEOUT
        assert 0.019 <= elapsed < 2.0
        ft.ft_sync_status(c.h)                          # the status word was cleared
        # the persistent kernel and the per-layer kernels still agree bit for bit
        a = torch.empty_like(x)
        b = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg, a, 1)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg, b, 1 | ft.FT_STACK_LAYERWISE)
        ft.ft_sync_status(c.h)
        torch.cuda.synchronize()
        assert (bf16_bits(a) == bf16_bits(b)).all()


H, I, E, K, L = 256, 128, 16, 2, 4


def host_pools(n_blobs):
    stride = synth.blob_stride(H, I)
    pools = []
    for layer in range(L):
        t = torch.empty(n_blobs * stride, dtype=torch.uint8).pin_memory()
        for e in range(n_blobs):
            t[e * stride:(e + 1) * stride] = torch.from_numpy(synth.expert_blob(SEED, layer, e, H, I))
        pools.append(t)
    return pools


def test_host_wait_runs_out_while_the_stream_is_busy():
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    cache = Ctx(ft.make_desc(H, I, E, K, L, 0, 8 * stride, 4), hp, None)
    res = Ctx(ft.make_desc(H, I, E, K, L, 0, 0, 4), None, [p.cuda() for p in hp])
    try:
        with pytest.raises(ft.FtError) as e:
            ft.ft_debug_host_wait_limit(cache.h, 0.0)
        assert e.value.status == ft.FT_ERR_INVALID
        lg = torch.from_numpy(synth.logits_for_sets(SEED, 0, np.array([[3, 9]]), E)).cuda()
        x = x_dev(synth.activations_bf16(SEED, 0, 1, H))
        out = torch.empty_like(x)
        ft.ft_debug_host_wait_limit(cache.h, 0.05)
        ft.ft_debug_device_wait(cache.h, 500000)        # keeps the stream busy for 0.5 s
        t0 = time.perf_counter()
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(cache.h, 0, x, 1, None, lg, out, 1)
        assert e.value.status == ft.FT_ERR_TIMEOUT
        assert time.perf_counter() - t0 < 0.4
        assert ft.ft_cache_trace(cache.h) == []         # the LRU step did not run
        with pytest.raises(ft.FtError) as e:            # the device wait's own timeout
            ft.ft_sync_status(cache.h)
        assert e.value.status == ft.FT_ERR_TIMEOUT
        ft.ft_debug_host_wait_limit(cache.h, 30.0)
        ref = torch.empty_like(x)
        ft.ft_moe_layer_forward(cache.h, 0, x, 1, None, lg, out, 1)
        ft.ft_moe_layer_forward(res.h, 0, x, 1, None, lg, ref, 1)
        torch.cuda.synchronize()
        assert (bf16_bits(out) == bf16_bits(ref)).all()
        assert ft.ft_cache_trace(cache.h) == [(ft.FT_EV_MISS, 0, 3, 0, -1), (ft.FT_EV_MISS, 0, 9, 1, -1)]
    finally:
        cache.close()
        res.close()


def test_injected_copy_failure_drops_the_key_and_a_retry_recovers():
    stride = synth.blob_stride(H, I)
    hp = host_pools(E)
    cache = Ctx(ft.make_desc(H, I, E, K, L, 0, 8 * stride, 4), hp, None)
    res = Ctx(ft.make_desc(H, I, E, K, L, 0, 0, 4), None, [p.cuda() for p in hp])
    try:
        with pytest.raises(ft.FtError) as e:
            ft.ft_debug_fail_copy(cache.h, -1)
        assert e.value.status == ft.FT_ERR_INVALID
        lg = torch.from_numpy(synth.logits_for_sets(SEED, 1, np.array([[2, 5]]), E)).cuda()
        x = x_dev(synth.activations_bf16(SEED, 1, 1, H))
        out = torch.empty_like(x)
        ft.ft_debug_fail_copy(cache.h, 2)               # the second copy from now on fails
        with pytest.raises(ft.FtError) as e:
            ft.ft_moe_layer_forward(cache.h, 1, x, 1, None, lg, out, 1)
        assert e.value.status == ft.FT_ERR_CUDA
        assert ft.ft_cache_trace(cache.h) == [(ft.FT_EV_MISS, 1, 2, 0, -1), (ft.FT_EV_MISS, 1, 5, 1, -1),
                                              (ft.FT_EV_EVICT, 1, 5, 1, -1)]
        assert ft.ft_cache_stats_get(cache.h)["used_slots"] == 1
        # the retry (injection has fired and is off) fetches the dropped key
        ref = torch.empty_like(x)
        ft.ft_moe_layer_forward(cache.h, 1, x, 1, None, lg, out, 1)
        ft.ft_moe_layer_forward(res.h, 1, x, 1, None, lg, ref, 1)
        torch.cuda.synchronize()
        assert (bf16_bits(out) == bf16_bits(ref)).all()
        assert ft.ft_cache_trace(cache.h) == [(ft.FT_EV_HIT, 1, 2, 0, -1), (ft.FT_EV_MISS, 1, 5, 1, -1)]
        # the oracle LRU, replaying the step without the failure, ends in the same state
        ref_lru = olru.LRUCache(8)
        ref_lru.step(1, np.array([2, 5]))
        assert ft.ft_expert_cache_lookup(cache.h, 1, 2) == 0 and ft.ft_expert_cache_lookup(cache.h, 1, 5) == 1
        assert ref_lru.lookup(1, 2) == 0 and ref_lru.lookup(1, 5) == 1
        ft.ft_sync_status(cache.h)
    finally:
        cache.close()
        res.close()


@pytest.mark.parametrize("T", [1, 2])
def test_tagged_words_are_zeroed_when_the_launch_counter_wraps(T):
    """The dataflow stack kernel's tagged hand-over words carry a tag (launch
    counter << 7 | layer) that repeats every 2^25 launches.  Stale words of a
    launch 2^25 earlier would pass for the current launch's; the routing
    kernel zeroes every tagged word when the counter wraps.  Here each tagged
    word is overwritten with a NaN under the exact tag the wrapping launch uses
    for a layer, and the launches across the wrap must still equal the
    per-layer kernels bit for bit."""
    H, I, E, k, L = 2048, 512, 64, 8, 2
    pools = [synth.gpu.layer_pool(H, I, E + 1, SEED, layer) for layer in range(L)]
    sets = [np.stack([synth.zipf_trace(SEED, layer, 3, E, k, 1.1, 0.6, stream=t)[-1] for t in range(T)])
            for layer in range(L)]
    lg = torch.from_numpy(np.stack([synth.logits_for_sets(SEED, layer, sets[layer], E) for layer in range(L)])).cuda()
    x = x_dev(synth.activations_bf16(SEED, 2, T, H))
    with Ctx(ft.make_desc(H, I, E, k, L, 1, 0, 4), None, pools) as c:
        want = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg, want, 1 | ft.FT_STACK_LAYERWISE)
        ft.ft_sync_status(c.h)
        want_b = bf16_bits(want)
        for poison in range(L):
            ft.ft_debug_stack_epoch(c.h, (1 << 25) - 1, poison)   # the next launch wraps
            for rep in range(3):
                got = torch.empty_like(x)
                ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg, got, 1)
                ft.ft_sync_status(c.h)
                assert (bf16_bits(got) == want_b).all(), (poison, rep)
        ft.ft_debug_stack_epoch(c.h, (1 << 32) - 3)           # the 32-bit counter itself wraps too
        for rep in range(4):
            got = torch.empty_like(x)
            ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg, got, 1)
            ft.ft_sync_status(c.h)
            assert (bf16_bits(got) == want_b).all(), rep
