"""ctypes binding of the C++ oracle (oracle/ft_oracle.cpp -> liboracle.so).

Test infrastructure only (see the package header).  The same functions as the
numpy modules of this package, under the same names, computed by the plain C++
restatement; the numpy modules serve as its cross-check.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None
P = C.c_void_p


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        sig = {
            "fto_threads": (C.c_int, []),
            "fto_e2m1_table": (None, [P]),
            "fto_ue8m0_table": (None, [P]),
            "fto_e4m3_table": (None, [P]),
            "fto_scale_index": (C.c_int64, [C.c_int64, C.c_int64, C.c_int64]),
            "fto_layout": (None, [C.c_int, C.c_int, C.c_int, P]),
            "fto_weight_matrix": (None, [P, C.c_int, C.c_int, C.c_int, C.c_int, P]),
            "fto_quantize_rows": (None, [P, C.c_int64, C.c_int, P, P]),
            "fto_round_bf16": (None, [P, C.c_int64, P]),
            "fto_nvfp4_quantize_rows": (C.c_float, [P, C.c_int64, C.c_int, C.c_float, P, P]),
            "fto_router_logits": (None, [P, P, C.c_int, C.c_int, C.c_int, P]),
            "fto_topk": (C.c_int, [P, C.c_int, C.c_int, C.c_int, P]),
            "fto_softmax_weights": (None, [P, P, C.c_int, C.c_int, C.c_int, C.c_int, P]),
            "fto_permutation": (None, [P, C.c_int, C.c_int, P, P, P]),
            "fto_expert_ffn": (None, [P, C.c_int, C.c_int, P, C.c_int, C.c_int, C.c_int, P]),
            "fto_moe_layer": (C.c_int, [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P, P, P, C.c_int, C.c_int,
                                        C.c_int, C.c_int, P, P, P, P]),
            "fto_lru_new": (P, [C.c_int64]),
            "fto_lru_free": (None, [P]),
            "fto_lru_step": (C.c_int64, [P, C.c_int, P, C.c_int, P, C.c_int64]),
            "fto_lru_resize": (C.c_int64, [P, C.c_int64, P, C.c_int64]),
            "fto_lru_lookup": (C.c_int, [P, C.c_int, C.c_int]),
            "fto_lru_set_prefetch": (None, [P, C.c_int, C.c_int, C.c_int]),
            "fto_lru_prefetch_counts": (None, [P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


FORMATS = {"mxfp4": 0, "nvfp4": 1, "bf16": 2}


def _p(a):
    return a.ctypes.data_as(P) if a is not None else None


def threads() -> int:
    """OpenMP threads available to the oracle (the host's cores unless limited)."""
    return lib().fto_threads()


def e2m1_table() -> np.ndarray:
    out = np.empty(16)
    lib().fto_e2m1_table(_p(out))
    return out


def ue8m0_table() -> np.ndarray:
    out = np.empty(256)
    lib().fto_ue8m0_table(_p(out))
    return out


def e4m3_table() -> np.ndarray:
    out = np.empty(256)
    lib().fto_e4m3_table(_p(out))
    return out


def scale_index(row: int, kblock: int, n_kblocks: int) -> int:
    return lib().fto_scale_index(row, kblock, n_kblocks)


def layout(hidden: int, inter: int, weights: str = "mxfp4") -> dict:
    out = np.empty(9, np.int64)
    lib().fto_layout(hidden, inter, FORMATS[weights], _p(out))
    d = dict(zip(("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "used", "stride", "tensor_scales"), map(int, out)))
    if weights == "mxfp4":
        d.pop("tensor_scales")
    return d


def weight_matrix(blob: np.ndarray, which: str, hidden: int, inter: int, weights: str = "mxfp4") -> np.ndarray:
    mat = ("wg", "wu", "wd").index(which)
    rows, K = (inter, hidden) if mat < 2 else (hidden, inter)
    out = np.empty((rows, K))
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    lib().fto_weight_matrix(_p(b), hidden, inter, mat, FORMATS[weights], _p(out))
    return out


def dequant_matrix(blob, which, hidden, inter):
    return weight_matrix(blob, which, hidden, inter, "mxfp4")


def quantize_rows(v: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    v = np.ascontiguousarray(v, dtype=np.float64)
    R, K = v.shape
    codes = np.empty((R, K), np.uint8)
    scales = np.empty((R, K // 32), np.uint8)
    lib().fto_quantize_rows(_p(v), R, K, _p(codes), _p(scales))
    return codes, scales


def nvfp4_quantize_rows(v: np.ndarray, s=None) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """As ``oracle.formats.nvfp4_quantize_rows``: codes [R, K], E4M3 scale
    bytes [R, K/16] and the per-tensor scale."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    R, K = v.shape
    codes = np.empty((R, K), np.uint8)
    scales = np.empty((R, K // 16), np.uint8)
    st = lib().fto_nvfp4_quantize_rows(_p(v), R, K, -1.0 if s is None else float(s), _p(codes), _p(scales))
    return codes, scales, np.float32(st)


def round_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().fto_round_bf16(_p(v), v.size, _p(out))
    return out


def router_logits(x_bits: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """fp32 logits [T, E] of bf16 bits x [T, H] and fp32 Wr [E, H]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w = np.ascontiguousarray(wr, dtype=np.float32)
    T, H = x.shape
    E = w.shape[0]
    out = np.empty((T, E), np.float32)
    lib().fto_router_logits(_p(x), _p(w), T, H, E, _p(out))
    return out


def topk(logits: np.ndarray, k: int) -> tuple[np.ndarray, bool]:
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    bad = lib().fto_topk(_p(lg), T, E, k, _p(ids))
    return ids, bool(bad)


def softmax_weights(logits: np.ndarray, ids: np.ndarray, renorm: bool = True) -> np.ndarray:
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, E = lg.shape
    k = ids.shape[1]
    w = np.empty((T, k))
    lib().fto_softmax_weights(_p(lg), _p(ids), T, E, k, 1 if renorm else 0, _p(w))
    return w


def permutation(ids: np.ndarray, E: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    flat = np.ascontiguousarray(np.asarray(ids).reshape(-1), dtype=np.int32)
    P_ = flat.size
    offs = np.empty(E + 1, np.int32)
    perm = np.empty(P_, np.int32)
    inv = np.empty(P_, np.int32)
    lib().fto_permutation(_p(flat), P_, E, _p(offs), _p(perm), _p(inv))
    return offs, perm, inv


def expert_ffn(blob, hidden, inter, x, mxfp4=False, weights="mxfp4") -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    m = x.shape[0]
    y = np.empty((m, hidden))
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    lib().fto_expert_ffn(_p(b), hidden, inter, _p(x), m, 1 if mxfp4 else 0, FORMATS[weights], _p(y))
    return y


def moe_layer(x_bits, blob_of, hidden, inter, n_experts, top_k, logits=None, router_w=None, renorm=True,
              mxfp4=False, shared_blob=None, weights="mxfp4", threads=1, nvfp4=False) -> dict:
    """One MoE layer on T tokens, as ``oracle.layer.moe_layer`` (blob_of is
    called for the selected experts only).  Returns dict with ids, w, out_f64,
    out_bits and nonfinite."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T = x.shape[0]
    H, E, k = hidden, n_experts, top_k
    if logits is not None:
        lg = np.ascontiguousarray(logits, dtype=np.float32)
    else:
        lg = router_logits(x, router_w)
    ids_pre, _ = topk(lg, k)
    keep = {int(e): np.ascontiguousarray(blob_of(int(e)), dtype=np.uint8) for e in np.unique(ids_pre)}
    ptrs = (P * E)()
    for e, b in keep.items():
        ptrs[e] = b.ctypes.data
    sb = np.ascontiguousarray(shared_blob, dtype=np.uint8) if shared_blob is not None else None
    out = np.empty((T, H))
    bits = np.empty((T, H), np.uint16)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k))
    bad = lib().fto_moe_layer(_p(x), T, H, inter, E, k, ptrs, _p(sb), _p(lg), None, 1 if renorm else 0,
                              2 if nvfp4 else (1 if mxfp4 else 0), FORMATS[weights], threads, _p(out), _p(bits),
                              _p(ids), _p(w))
    return dict(ids=ids, w=w, out_f64=out, out_bits=bits, nonfinite=bool(bad), logits=lg)


class LRUCache:
    """The global LRU of ``oracle.lru.LRUCache``, from the C++ oracle."""

    def __init__(self, capacity: int):
        self.h = lib().fto_lru_new(int(capacity))

    def __del__(self):
        if getattr(self, "h", None):
            lib().fto_lru_free(self.h)
            self.h = None

    @staticmethod
    def _events(buf, n):
        return [tuple(int(v) for v in buf[i]) for i in range(n)]

    def step(self, layer, experts) -> list[tuple]:
        e = np.ascontiguousarray(np.asarray(experts).reshape(-1), dtype=np.int32)
        buf = np.empty((3 * e.size + 4 + 2 * 16, 5), np.int32)
        n = lib().fto_lru_step(self.h, int(layer), _p(e), e.size, _p(buf), buf.shape[0])
        if n < 0:
            raise RuntimeError("more experts in one step than cache slots")
        return self._events(buf, n)

    def resize(self, capacity: int) -> list[tuple]:
        cap = 1 << 16
        buf = np.empty((cap, 5), np.int32)
        n = lib().fto_lru_resize(self.h, int(capacity), _p(buf), cap)
        assert n <= cap
        return self._events(buf, n)

    def lookup(self, layer: int, expert: int) -> int:
        return lib().fto_lru_lookup(self.h, int(layer), int(expert))


class PrefetchingLRUCache(LRUCache):
    """``oracle.lru.PrefetchingLRUCache`` from the C++ oracle."""

    def __init__(self, capacity: int, n_layers: int, n_experts: int, per_layer: int):
        super().__init__(capacity)
        lib().fto_lru_set_prefetch(self.h, n_layers, n_experts, per_layer)

    def _counts(self):
        out = np.zeros(2, np.int64)
        lib().fto_lru_prefetch_counts(self.h, _p(out))
        return int(out[0]), int(out[1])

    @property
    def prefetches(self) -> int:
        return self._counts()[0]

    @property
    def prefetch_hits(self) -> int:
        return self._counts()[1]
