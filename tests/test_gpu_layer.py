"""GPU parity of ft_moe_layer_forward (decode path) against the oracle, on the
shapes of the tiny layer and the 35B-class, DeepSeek-V4-Flash-class and
GLM-class layers, with resident expert pools."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu


def run_layer(H, I, E, k, S, T, seed, use_router, renorm=True, trace=True, max_tokens=16):
    pool = synth.gpu.layer_pool(H, I, E + S, seed, 0)
    xb = synth.activations_bf16(seed, 1, T, H)
    wr = synth.router_weights(seed, 0, E, H) if use_router else None
    if use_router:
        lg = None
    elif trace:
        sets = np.stack([synth.zipf_trace(seed, 0, 3, E, k, 1.1, 0.6, stream=t)[-1] for t in range(T)])
        lg = synth.logits_for_sets(seed, 2, sets, E)
    else:
        lg = np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)
    desc = ft.make_desc(H, I, E, k, 1, S, 0, max_tokens)
    with Ctx(desc, None, [pool]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_layer_forward(c.h, 0, x, T, torch.from_numpy(wr).cuda() if use_router else None,
                                torch.from_numpy(lg).cuda() if lg is not None else None, out,
                                (ft.FT_ROUTE_RENORM if renorm else 0) | ft.FT_ACT_BF16)
        ft.ft_sync_status(c.h)
        got = bf16_bits(out)
        ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
        w = torch.empty(T * k, dtype=torch.float32, device="cuda")
        ft.ft_last_routing(c.h, ids, w, T * k)
        torch.cuda.synchronize()
        got_ids, got_w = ids.cpu().numpy().reshape(T, k), w.cpu().numpy().reshape(T, k)
    blobs = {}

    def blob_of(e):
        if e not in blobs:
            blobs[e] = synth.expert_blob(seed, 0, e, H, I)
        return blobs[e]
    r = olayer.moe_layer(xb, blob_of, H, I, E, k, logits=lg, router_w=wr, renorm=renorm,
                         shared_blob=blob_of(E) if S else None)
    assert (got_ids == r["ids"]).all()
    assert np.allclose(got_w, r["w"], rtol=2e-6, atol=1e-9)
    return got, r


@pytest.mark.parametrize("T", [1, 2, 3, 8])
@pytest.mark.parametrize("use_router", [True, False])
def test_tiny_layer(T, use_router):
    got, r = run_layer(256, 128, 16, 2, 0, T, 1001, use_router, trace=False)
    assert_close(got, r["out_f64"])


def test_tiny_layer_no_renorm():
    got, r = run_layer(256, 128, 16, 2, 0, 8, 1001, True, renorm=False)
    assert_close(got, r["out_f64"])


@pytest.mark.parametrize("T", [1, 4, 16])
def test_35b_class_layer(T):
    got, r = run_layer(2048, 512, 256, 8, 1, T, 1002, False)
    assert_close(got, r["out_f64"])


@pytest.mark.parametrize("T", [1, 3])
def test_dsv4_class_layer(T):
    got, r = run_layer(4096, 2048, 256, 6, 0, T, 1003, False)
    assert_close(got, r["out_f64"])


def test_dsv4_class_layer_router_gemv():
    got, r = run_layer(4096, 2048, 256, 6, 0, 2, 1003, True)
    assert_close(got, r["out_f64"])


def test_glm_class_layer():
    got, r = run_layer(6144, 2048, 256, 8, 0, 1, 1005, False)
    assert_close(got, r["out_f64"])


def test_deterministic_repeat():
    a, _ = run_layer(2048, 512, 256, 8, 1, 4, 1002, False)
    b, _ = run_layer(2048, 512, 256, 8, 1, 4, 1002, False)
    assert (a == b).all()


def test_zero_tokens_and_limits():
    pool = synth.gpu.layer_pool(256, 128, 16, 1, 0)
    with Ctx(ft.make_desc(256, 128, 16, 2, 1, 0, 0, 4), None, [pool]) as c:
        x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
        out = torch.zeros_like(x)
        lg = torch.zeros((4, 16), dtype=torch.float32, device="cuda")
        ft.ft_moe_layer_forward(c.h, 0, x, 0, None, lg, out, 1)     # T = 0 is a no-op
        with pytest.raises(ft.FtError):
            ft.ft_moe_layer_forward(c.h, 0, x, 5, None, lg, out, 1)  # above max_tokens
        with pytest.raises(ft.FtError):
            ft.ft_moe_layer_forward(c.h, 1, x, 1, None, lg, out, 1)  # no such layer
        with pytest.raises(ft.FtError):
            ft.ft_moe_layer_forward(c.h, 0, x, 1, None, lg, x, 1)    # out aliases x


def test_fused_routing_ties_and_no_renorm():
    """Exact ties in the logits resolve to the lower id inside the fused kernels."""
    H, I, E, k, T, seed = 2048, 512, 256, 8, 4, 77
    pool = synth.gpu.layer_pool(H, I, E, seed, 0)
    lg = np.random.default_rng(1).standard_normal((T, E)).astype(np.float32)
    lg[:, 10:30] = 2.5                  # 20 tied experts above the rest
    lg[1, :] = 0.0                      # a fully tied row
    lg[2, 7] = -0.0
    xb = synth.activations_bf16(seed, 1, T, H)
    with Ctx(ft.make_desc(H, I, E, k, 1, 0, 0, 16), None, [pool]) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        for renorm in (1, 0):
            ft.ft_moe_layer_forward(c.h, 0, x, T, None, torch.from_numpy(lg).cuda(), out, renorm)
            ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
            w = torch.empty(T * k, dtype=torch.float32, device="cuda")
            ft.ft_last_routing(c.h, ids, w, T * k)
            torch.cuda.synchronize()
            want, _ = olayer.routing.topk(lg, k)
            assert (ids.cpu().numpy().reshape(T, k) == want).all()
            ww = olayer.routing.softmax_weights(lg, want, bool(renorm))
            assert np.allclose(w.cpu().numpy().reshape(T, k), ww, rtol=2e-6, atol=1e-9)


STACK_SHAPES = {
    # name: H, I, E, k, S, seed
    "tiny": (256, 128, 16, 2, 0, 1001),
    "35b": (2048, 512, 256, 8, 1, 1002),
    "no_shared": (1024, 512, 64, 4, 0, 1004),
    "narrow_down": (1024, 768, 64, 4, 1, 1005),   # down tile of 256 threads
    "dsv4": (4096, 2048, 256, 6, 0, 1003),
}


def stack_case(name, T, L):
    H, I, E, k, S, seed = STACK_SHAPES[name]
    pools = [synth.gpu.layer_pool(H, I, E + S, seed, l) for l in range(L)]
    lgs = []
    for l in range(L):
        sets = np.stack([synth.zipf_trace(seed, l, 3, E, k, 1.1, 0.6, stream=t)[-1] for t in range(T)])
        lgs.append(synth.logits_for_sets(seed, 10 + l, sets, E))
    return (H, I, E, k, S, seed), pools, lgs


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 2), ("35b", 1), ("35b", 2), ("35b", 4), ("35b", 16),
                                    ("no_shared", 1), ("no_shared", 2), ("no_shared", 16), ("narrow_down", 1),
                                    ("narrow_down", 2), ("narrow_down", 3), ("dsv4", 1), ("dsv4", 2)])
@pytest.mark.parametrize("flags", [1, 1 | ft.FT_STACK_COUNTERS, 1 | ft.FT_STACK_LAYERWISE],
                         ids=["default", "counters", "layerwise"])
def test_stack_forward_matches_layer_by_layer(name, T, flags):
    """Every stack mode equals the same layers run one ft_moe_layer_forward at
    a time, bit for bit: the dataflow kernel (the default for one or two
    tokens), the counter-synchronised persistent kernel, and two kernels per
    layer."""
    L = 3
    (H, I, E, k, S, seed), pools, lgs = stack_case(name, T, L)
    lg_all = torch.from_numpy(np.stack(lgs)).cuda()
    xb = synth.activations_bf16(seed, 1, T, H)
    with Ctx(ft.make_desc(H, I, E, k, L, S, 0, 16), None, pools) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, out, flags)
        ft.ft_sync_status(c.h)
        cur = x
        inputs = []
        for l in range(L):
            inputs.append(bf16_bits(cur))
            nxt = torch.empty_like(x)
            ft.ft_moe_layer_forward(c.h, l, cur, T, None, lg_all[l], nxt, 1)
            cur = nxt
        torch.cuda.synchronize()
        assert (bf16_bits(out) == bf16_bits(cur)).all()
        # the routing the stack leaves behind is the last layer's
        ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
        w = torch.empty(T * k, dtype=torch.float32, device="cuda")
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, out, flags)
        ft.ft_last_routing(c.h, ids, w, T * k)
        torch.cuda.synchronize()
        want, _ = olayer.routing.topk(lgs[-1], k)
        assert (ids.cpu().numpy().reshape(T, k) == want).all()
    # layer-local parity of the last layer against the oracle
    blobs = {}

    def blob_of(e):
        if e not in blobs:
            blobs[e] = synth.expert_blob(seed, L - 1, e, H, I)
        return blobs[e]
    r = olayer.moe_layer(inputs[-1], blob_of, H, I, E, k, logits=lgs[-1], shared_blob=blob_of(E) if S else None)
    assert_close(bf16_bits(out), r["out_f64"])


def test_stack_forward_repeated_and_sub_stacks():
    """Back-to-back persistent launches reuse the counters (zeroed by the
    routing kernel): 40 layers at once equal the same layers run as two
    sub-stacks, and a second identical call gives identical bits."""
    L, T = 40, 2
    (H, I, E, k, S, seed), pools, lgs = stack_case("35b", T, L)
    lg_all = torch.from_numpy(np.stack(lgs)).cuda()
    xb = synth.activations_bf16(seed, 1, T, H)
    with Ctx(ft.make_desc(H, I, E, k, L, S, 0, 16), None, pools) as c:
        x = x_dev(xb)
        a = torch.empty_like(x)
        b = torch.empty_like(x)
        mid = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, a, 1)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, b, 1)
        ft.ft_sync_status(c.h)
        torch.cuda.synchronize()
        assert (bf16_bits(a) == bf16_bits(b)).all()
        ft.ft_moe_stack_forward(c.h, 0, 17, x, T, lg_all[:17].contiguous(), mid, 1)
        ft.ft_moe_stack_forward(c.h, 17, L - 17, mid, T, lg_all[17:].contiguous(), b, 1)
        ft.ft_sync_status(c.h)
        torch.cuda.synchronize()
        assert (bf16_bits(a) == bf16_bits(b)).all()
        for other in (ft.FT_STACK_LAYERWISE, ft.FT_STACK_COUNTERS):
            ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, b, 1 | other)
            ft.ft_sync_status(c.h)
            torch.cuda.synchronize()
            assert (bf16_bits(a) == bf16_bits(b)).all()
