"""Router logits, softmax top-k routing and the token permutation.

Test infrastructure only (see the package header).

The pages state that a gate picks a few experts per token and layer
(aiforradalom.hu page, section "A Mixture-of-Experts (MoE) kihívásai és a
FreeToken megoldásai": DeepSeek-V4-Flash activates 6 of 256 experts per layer;
world.tibi.club page, section "Ce este un model MoE?": a gate decides which
experts run).  They define no formula; the readings used here:

* logits = x . Wr^T, with the summation order fixed (``router_logits``) so that
  any implementation that follows the same order gets the same fp32 bits;
* top-k on the fp32 logits by (value descending, expert id ascending), -0 equal
  to +0, NaN below -inf;
* weights = softmax over all experts at the chosen ids, renormalised over the k
  chosen (or raw softmax when renormalisation is off);
* permutation = stable sort of the (token, rank) pairs by expert id.
"""
from __future__ import annotations

import math

import numpy as np

LANES = 32      # partial sums of a logit
VEC = 4         # consecutive elements per lane per step


def router_logits(x: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """fp32 logits [T, E] of x [T, H] (bf16 values as fp64) and Wr [E, H] fp32.

    Each product bf16 * fp32 is exact in fp64.  The sum runs in fp64 in a fixed
    order: element k goes to partial sum number (k // 4) mod 32; each partial
    sum adds its elements in ascending k; the 32 partial sums are then combined
    pairwise by the butterfly with distances 16, 8, 4, 2, 1 (position p takes
    its value plus the value at p xor d); the result at position 0 is rounded
    once to fp32.  H must be a multiple of 128.
    """
    x = np.asarray(x, dtype=np.float64)
    wr = np.asarray(wr, dtype=np.float32).astype(np.float64)
    T, H = x.shape
    E = wr.shape[0]
    assert H % (LANES * VEC) == 0
    C = H // (LANES * VEC)
    out = np.empty((T, E), dtype=np.float32)
    for t in range(T):
        prod = (wr * x[t][None, :]).reshape(E, C, LANES, VEC)   # exact products
        part = np.zeros((E, LANES))
        for c in range(C):
            for v in range(VEC):
                part = part + prod[:, c, :, v]
        for d in (16, 8, 4, 2, 1):
            part = part + part[:, np.arange(LANES) ^ d]
        out[t] = part[:, 0].astype(np.float32)
    return out


def topk(logits: np.ndarray, k: int) -> tuple[np.ndarray, bool]:
    """Ids [T, k] in rank order and a flag that is True when any logit is NaN
    or +inf, or a row has no finite logit."""
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int32)
    bad = False
    for t in range(T):
        row = [float(v) for v in lg[t]]
        if any(math.isnan(v) or v == math.inf for v in row) or not any(math.isfinite(v) for v in row):
            bad = True

        def key(e):
            v = row[e]
            if math.isnan(v):
                return (1, 0.0, e)
            return (0, -v, e)
        order = sorted(range(E), key=key)
        ids[t] = order[:k]
    return ids, bad


def softmax_weights(logits: np.ndarray, ids: np.ndarray, renorm: bool = True) -> np.ndarray:
    """fp64 weights [T, k]: p = softmax(logits row) at the chosen ids,
    divided by their sum when ``renorm``."""
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, k = ids.shape
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        m = np.max(lg[t])
        p = np.exp(lg[t] - m)
        p = p / p.sum()
        sel = p[ids[t]]
        w[t] = sel / sel.sum() if renorm else sel
    return w


def permutation(ids: np.ndarray, E: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(offs [E+1], perm [T*k], inv [T*k]) of the pairs f = t*k + j sorted
    stably by expert id: perm[pos] = f, inv[f] = pos, and the pairs of expert e
    occupy positions offs[e] .. offs[e+1]-1 in ascending (token, rank)."""
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    perm = np.array(sorted(range(flat.size), key=lambda f: (flat[f], f)), dtype=np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(flat.size, dtype=np.int32)
    offs = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offs[e + 1] = offs[e] + int(np.sum(flat == e))
    return offs, perm, inv
