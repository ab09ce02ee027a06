"""Parity at the full size of the decode benchmark's workload: the 35B-A3B-class
stack (hidden 2048, 256 routed experts top-8 + 1 shared, intermediate 512, 40
layers, Zipf(1.1) traces with 0.6 adjacent reuse) at batch 1 and 4, run as the
benchmark runs it: one ft_moe_stack_forward (the routing kernel and the
persistent kernel).  Its output equals the same 40 layers run one
ft_moe_layer_forward at a time, bit for bit, and sampled layers match the oracle
layer-locally, each on the exact bf16 input it saw."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import layer as olayer

from _gpu import Ctx, assert_close, bf16_bits, x_dev

pytestmark = pytest.mark.gpu

H, I, E, K, S, L, SEED = 2048, 512, 256, 8, 1, 40, 1002


@pytest.mark.parametrize("T", [1, 2, 4])
def test_35b_class_stack_at_full_size(T):
    pools = [synth.gpu.layer_pool(H, I, E + S, SEED, layer) for layer in range(L)]
    lgs = []
    for layer in range(L):
        sets = np.stack([synth.zipf_trace(SEED, layer, 3, E, K, 1.1, 0.6, stream=t)[-1] for t in range(T)])
        lgs.append(synth.logits_for_sets(SEED, 10 + layer, sets, E))
    lg_all = torch.from_numpy(np.stack(lgs)).cuda()
    xb = synth.activations_bf16(SEED, 1, T, H)
    with Ctx(ft.make_desc(H, I, E, K, L, S, 0, 16), None, pools) as c:
        x = x_dev(xb)
        out = torch.empty_like(x)
        ft.ft_moe_stack_forward(c.h, 0, L, x, T, lg_all, out, ft.FT_ROUTE_RENORM)
        ft.ft_sync_status(c.h)
        cur, inputs = x, []
        for layer in range(L):
            inputs.append(bf16_bits(cur))
            nxt = torch.empty_like(x)
            ft.ft_moe_layer_forward(c.h, layer, cur, T, None, lg_all[layer], nxt, ft.FT_ROUTE_RENORM)
            cur = nxt
        ft.ft_sync_status(c.h)
        torch.cuda.synchronize()
        final = bf16_bits(cur)
        assert (bf16_bits(out) == final).all()
    del pools
    torch.cuda.empty_cache()
    outputs = inputs[1:] + [final]
    for layer in (0, L // 2, L - 1):
        blobs = {}

        def blob_of(e):
            if e not in blobs:
                blobs[e] = synth.expert_blob(SEED, layer, e, H, I)
            return blobs[e]
        r = olayer.moe_layer(inputs[layer], blob_of, H, I, E, K, logits=lgs[layer], shared_blob=blob_of(E))
        assert_close(outputs[layer], r["out_f64"])
