"""Writes tests/golden/tiny_layer.json: the oracle's result for the tiny MoE
layer (hidden 256, 16 experts, top-2, intermediate 128, 8 tokens, seed 1001),
in decode mode and in MXFP4-activation mode.  Calls only ``oracle`` and the
seeded input module ``synth``.  The file pins the oracle against accidental
change; rerun this script only with a commit that names why the oracle moved.

    python tests/golden/make_tiny.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from oracle import layer  # noqa: E402

H, I, E, K, T, SEED = 256, 128, 16, 2, 8, 1001


def main():
    blobs = {e: synth.expert_blob(SEED, 0, e, H, I) for e in range(E)}
    xb = synth.activations_bf16(SEED, 0, T, H)
    wr = synth.router_weights(SEED, 0, E, H)
    out = {"config": dict(hidden=H, inter=I, experts=E, top_k=K, tokens=T, seed=SEED,
                          x="synth.activations_bf16(seed, 0, T, H)",
                          router="synth.router_weights(seed, 0, E, H)",
                          blobs="synth.expert_blob(seed, 0, e, H, I)")}
    for mode, mx in (("decode", False), ("mxfp4", True)):
        r = layer.moe_layer(xb, blobs.__getitem__, H, I, E, K, router_w=wr, mxfp4=mx)
        out[mode] = dict(logits_f32_bits=r["logits"].view(np.uint32).tolist(),
                         ids=r["ids"].tolist(), w=r["w"].tolist(),
                         out_bf16_bits=r["out_bits"].tolist())
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_layer.json"), "w") as f:
        json.dump(out, f, separators=(",", ":"))


if __name__ == "__main__":
    main()
