"""SwiGLU expert FFN and the weighted combine of one MoE layer, in fp64.

Test infrastructure only (see the package header).

Pages: experts are computed on the GPU from weights fetched over PCIe or held
in VRAM (jansverre.net page, section "Hvorfor er båndbredden viktigere enn
antall kjerner?"), and the outputs of however the selected experts are split
are summed at the end with no simplified expert, no changed router and no
approximation (same section).  The expert type (SwiGLU: h = silu(Wg x) * (Wu x),
y = Wd h) and the output rounding (one bf16 rounding of the fp64 sum) are the
readings used here.

Modes:
* ``mxfp4=False`` (decode): x is the bf16 input as is; h stays unrounded.
* ``mxfp4=True`` (prefill): x and h are quantised per 32 values along their
  contraction axis by the OCP MX rule before each product.

* ``nvfp4=True`` (prefill with NVFP4 experts): x and h are quantised to NVFP4
  (``formats.nvfp4_quantize_rows``) before each product, each with one
  per-tensor scale: x's over all T tokens, h's over every h row of the layer
  (all routed pairs and the shared expert's rows), so every expert's h is
  computed before any of them is quantised.

Weight formats (``weights``): "mxfp4" (the default), or "nvfp4" / "bf16"
(``formats``); MXFP4 activations go with MXFP4 weights, NVFP4 activations with
NVFP4 weights.
"""
from __future__ import annotations

import numpy as np

from . import formats, fp4, routing


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_ffn(blob: np.ndarray, hidden: int, inter: int, x: np.ndarray, mxfp4: bool = False,
               weights: str = "mxfp4") -> np.ndarray:
    """y [m, H] = Wd (silu(Wg x) * (Wu x)) for the rows of x [m, H] (fp64)."""
    if mxfp4 and weights != "mxfp4":
        raise ValueError("MXFP4 activations are defined for MXFP4 weights only")
    wg = formats.weight_matrix(blob, "wg", hidden, inter, weights)
    wu = formats.weight_matrix(blob, "wu", hidden, inter, weights)
    wd = formats.weight_matrix(blob, "wd", hidden, inter, weights)
    x = np.asarray(x, dtype=np.float64)
    if mxfp4:
        x = fp4.dequant_rows(*fp4.quantize_rows(x))
    g = x @ wg.T
    u = x @ wu.T
    h = silu(g) * u
    if mxfp4:
        h = fp4.dequant_rows(*fp4.quantize_rows(h))
    return h @ wd.T


def _nvfp4_expert_outputs(x, groups, hidden, inter):
    """NVFP4-activation expert outputs: groups = [(blob, rows of x)], returns
    [y rows] in the same order; both per-tensor scales span all groups."""
    cx, bx, sx = formats.nvfp4_quantize_rows(x)
    xq = formats.nvfp4_dequant_rows(cx, bx, sx)
    hs = []
    for blob, rows in groups:
        wg = formats.weight_matrix(blob, "wg", hidden, inter, "nvfp4")
        wu = formats.weight_matrix(blob, "wu", hidden, inter, "nvfp4")
        xr = xq[rows]
        hs.append(silu(xr @ wg.T) * (xr @ wu.T))
    amax = max((float(np.abs(h).max()) for h in hs if h.size), default=0.0)
    sh = formats.nvfp4_global_scale(np.float32(amax))
    ys = []
    for (blob, rows), h in zip(groups, hs):
        wd = formats.weight_matrix(blob, "wd", hidden, inter, "nvfp4")
        hq = formats.nvfp4_dequant_rows(*formats.nvfp4_quantize_rows(h, sh))
        ys.append(hq @ wd.T)
    return ys


def moe_layer(x_bits: np.ndarray, blob_of, hidden: int, inter: int, n_experts: int, top_k: int,
              logits: np.ndarray | None = None, router_w: np.ndarray | None = None,
              renorm: bool = True, mxfp4: bool = False, shared_blob=None, weights: str = "mxfp4",
              nvfp4: bool = False) -> dict:
    """One MoE layer on T tokens.

    x_bits   bf16 bits [T, H]
    blob_of  callable expert id -> blob (uint8)
    logits   fp32 [T, E] (used as given) or None to compute x . Wr^T
    shared_blob  blob of an always-on shared expert (weight 1) or None
    weights  format of every blob ("mxfp4", "nvfp4", "bf16")

    Returns dict with logits, ids, w (fp64), offs/perm/inv, out_f64 and
    out_bits (bf16 of out_f64).
    """
    x = fp4.bf16_to_f64(x_bits)
    T = x.shape[0]
    if logits is None:
        logits = routing.router_logits(x, router_w)
    ids, bad = routing.topk(logits, top_k)
    w = routing.softmax_weights(logits, ids, renorm)
    offs, perm, inv = routing.permutation(ids, n_experts)
    out = np.zeros((T, hidden), dtype=np.float64)
    y = {}
    experts = [int(e) for e in np.unique(ids)]
    rows_of = {e: np.nonzero((ids == e).any(axis=1))[0] for e in experts}
    y_shared = None
    if nvfp4:
        if weights != "nvfp4" or mxfp4:
            raise ValueError("NVFP4 activations are defined for NVFP4 weights only")
        groups = [(blob_of(e), rows_of[e]) for e in experts]
        if shared_blob is not None:
            groups.append((shared_blob, np.arange(T)))
        ys = _nvfp4_expert_outputs(x, groups, hidden, inter)
        y = {e: (rows_of[e], ys[i]) for i, e in enumerate(experts)}
        if shared_blob is not None:
            y_shared = ys[-1]
    else:
        for e in experts:
            y[e] = (rows_of[e], expert_ffn(blob_of(e), hidden, inter, x[rows_of[e]], mxfp4, weights))
    for t in range(T):
        acc = 0.0
        for j in range(top_k):
            rows, ye = y[int(ids[t, j])]
            acc = acc + w[t, j] * ye[int(np.nonzero(rows == t)[0][0])]
        if shared_blob is not None:
            acc = acc + (y_shared[t] if y_shared is not None
                         else expert_ffn(shared_blob, hidden, inter, x[t:t + 1], mxfp4, weights)[0])
        out[t] = acc
    return dict(logits=np.asarray(logits, dtype=np.float32), ids=ids, nonfinite=bad, w=w,
                offs=offs, perm=perm, inv=inv, out_f64=out, out_bits=fp4.round_bf16(out))
