"""The oracle still reproduces the committed tiny-layer fixture."""
import json
import os

import numpy as np

import synth
from oracle import layer

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_layer_fixture():
    with open(os.path.join(HERE, "golden", "tiny_layer.json")) as f:
        g = json.load(f)
    c = g["config"]
    H, I, E, K, T, S = c["hidden"], c["inter"], c["experts"], c["top_k"], c["tokens"], c["seed"]
    blobs = {e: synth.expert_blob(S, 0, e, H, I) for e in range(E)}
    xb = synth.activations_bf16(S, 0, T, H)
    wr = synth.router_weights(S, 0, E, H)
    for mode, mx in (("decode", False), ("mxfp4", True)):
        r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, K, router_w=wr, mxfp4=mx)
        assert r["logits"].view(np.uint32).tolist() == g[mode]["logits_f32_bits"]
        assert r["ids"].tolist() == g[mode]["ids"]
        assert np.allclose(r["w"], np.array(g[mode]["w"]), rtol=0, atol=0)
        assert r["out_bits"].tolist() == g[mode]["out_bf16_bits"]
