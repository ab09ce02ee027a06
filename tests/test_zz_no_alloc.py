"""ft_moe_layer_forward_noalloc, the decode forward for callers that cannot
allocate device memory (a process whose device memory is owned by another
allocator, or a path that cannot pay for cudaMalloc's synchronisation).

It must give the same layer output as ft_moe_layer_forward, call after call,
although its scratch lives in one static device array that every call reuses.
This file is collected last so that a failure here leaves every other test
already run; it also passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, bits_to_f64, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, S, SEED = 2048, 512, 256, 8, 1, 4242


def inputs(tag, T):
    xb = synth.activations_bf16(SEED, tag, T, H)
    sets = np.stack([synth.zipf_trace(SEED, tag, 2, E, K, 1.1, 0.6, stream=t)[-1] for t in range(T)])
    lg = synth.logits_for_sets(SEED, tag, sets, E)
    return x_dev(xb), torch.from_numpy(lg).cuda()


def test_noalloc_matches_context_forward_on_two_calls_in_a_row():
    """Against the context forward and against the oracle on the same
    inputs (decode mode), for two calls that reuse the static scratch."""
    pool = synth.gpu.layer_pool(H, I, E + S, SEED, 0)
    wr_host = synth.router_weights(SEED, 0, E, H)
    wr = torch.from_numpy(wr_host).cuda()
    stride = synth.blob_stride(H, I)
    host = pool.cpu().numpy()
    with Ctx(ft.make_desc(H, I, E, K, 1, S, 0, 16), None, [pool]) as c:
        cases = [(1, 4, False), (2, 3, True)]   # (tag, T, use the router GEMV)
        for tag, T, use_router in cases:
            x, lg = inputs(tag, T)
            want = torch.empty_like(x)
            got = torch.empty_like(x)
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            ft.ft_moe_layer_forward(c.h, 0, x, T, wr if use_router else None, None if use_router else lg, want,
                                    ft.FT_ROUTE_RENORM)
            ft.ft_moe_layer_forward_noalloc(H, I, E, K, S, pool, x, T, wr if use_router else None,
                                            None if use_router else lg, got, ft.FT_ROUTE_RENORM, status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            assert_close(bf16_bits(got), bits_to_f64(bf16_bits(want)))
            r = olayer.moe_layer(bf16_bits(x), lambda e: host[e * stride:(e + 1) * stride], H, I, E, K,
                                 logits=None if use_router else lg.cpu().numpy(),
                                 router_w=wr_host if use_router else None,
                                 shared_blob=host[E * stride:(E + 1) * stride])
            assert_close(bf16_bits(got), r["out_f64"])


def test_noalloc_rejects_calls_beyond_its_scratch():
    pool = synth.gpu.layer_pool(256, 128, 16, SEED, 0)
    x = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((17, 16), dtype=torch.float32, device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(ft.FtError) as e:        # T above the decode limit
        ft.ft_moe_layer_forward_noalloc(256, 128, 16, 2, 0, pool, x, 17, None, lg, out, 1)
    assert e.value.status == ft.FT_ERR_INVALID
    # 16 tokens x top-16 over intermediate 8192 needs ~8.5 MB of activations
    with pytest.raises(ft.FtError) as e:
        ft.ft_moe_layer_forward_noalloc(256, 8192, 16, 16, 0, pool, x, 16, None, lg, out, 1)
    assert e.value.status == ft.FT_ERR_INVALID
    assert "maximum" in str(e.value)
