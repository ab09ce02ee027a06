"""Python binding of libftmoe.so: one FreeToken-style MoE layer forward pass
with a GPU LRU expert cache over a pinned host expert pool, for B200 (sm_100a).

Argument marshalling only.  Every step of the hot path runs in the CUDA
library; the functions here take torch tensors (device memory, streams) or raw
pointers and call the C ABI declared in ``include/ft_moe.h`` under the same
names.  There is no CPU fallback: if the library is missing, the first call
raises.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libftmoe.so")

FT_OK, FT_ERR_INVALID, FT_ERR_CUDA, FT_ERR_NO_SPACE, FT_ERR_TIMEOUT, FT_ERR_NOT_FOUND, FT_ERR_NONFINITE, \
    FT_ERR_STATE = range(8)
STATUS_NAMES = {0: "FT_OK", 1: "FT_ERR_INVALID", 2: "FT_ERR_CUDA", 3: "FT_ERR_NO_SPACE", 4: "FT_ERR_TIMEOUT",
                5: "FT_ERR_NOT_FOUND", 6: "FT_ERR_NONFINITE", 7: "FT_ERR_STATE"}
FT_ROUTE_RENORM = 1
FT_ACT_BF16 = 0
FT_ACT_MXFP4 = 2
FT_STACK_LAYERWISE = 4
FT_STACK_COUNTERS = 8
FT_CACHE_SERIAL = 16
FT_ACT_NVFP4 = 32
FT_EV_HIT, FT_EV_MISS, FT_EV_EVICT, FT_EV_MOVE, FT_EV_PREFETCH = range(5)

EXPORTS = ("ft_blob_stride", "ft_blob_layout", "ft_last_error", "ft_create", "ft_destroy", "ft_sync_status",
           "ft_router_logits", "ft_moe_route", "ft_moe_permute", "ft_quantize_mxfp4", "ft_quantize_nvfp4", "ft_moe_layer_forward",
           "ft_expert_cache_lookup", "ft_expert_cache_insert", "ft_expert_cache_resize", "ft_cache_trace",
           "ft_cache_stats_get", "ft_prefetch_layer", "ft_debug_dequant", "ft_kernel_timing_enable",
           "ft_kernel_timing_read", "ft_moe_layer_forward_noalloc", "ft_moe_stack_forward", "ft_last_routing",
           "ft_debug_device_wait", "ft_debug_host_wait_limit", "ft_debug_fail_copy", "ft_decode_geometry",
           "ft_debug_stack_epoch", "ft_flow_geometry", "ft_fp4_mma_probe", "ft_blob_layout_format",
           "ft_cache_prefetch", "ft_debug_stack_timeline")
FT_NOALLOC_SCRATCH_BYTES = 8 << 20
KERNELS = ("router_logits", "topk", "permute", "gate_up", "down_combine", "quant_x", "gemm_gate_up", "gemm_down",
           "combine", "dec_stack", "quant_h")


class FtError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class ModelDesc(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("n_layers", C.c_int32), ("n_shared", C.c_int32), ("cache_budget_bytes", C.c_int64),
                ("max_tokens", C.c_int32), ("weight_format", C.c_int32)]


class CacheEvent(C.Structure):
    _fields_ = [("kind", C.c_int32), ("layer", C.c_int32), ("expert", C.c_int32), ("slot", C.c_int32),
                ("from_slot", C.c_int32)]


class CacheStats(C.Structure):
    _fields_ = [("hits", C.c_int64), ("misses", C.c_int64), ("evictions", C.c_int64), ("moves", C.c_int64),
                ("h2d_bytes", C.c_int64), ("h2d_ms", C.c_double), ("hit_ms", C.c_double),
                ("overlap_ms", C.c_double), ("capacity_slots", C.c_int64),
                ("used_slots", C.c_int64), ("mapped_bytes", C.c_int64), ("prefetches", C.c_int64),
                ("prefetch_hits", C.c_int64), ("prefetch_bytes", C.c_int64)]


_lib = None
P = C.c_void_p
I32 = C.c_int32
I64 = C.c_int64
U32 = C.c_uint32
ST = C.c_int


def lib() -> C.CDLL:
    """The loaded libftmoe.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m expert_offloaded_serving_b200.build` "
                           "(no CPU fallback exists)")
    L = C.CDLL(LIB_PATH)
    sig = {
        "ft_blob_stride": (I64, [I32, I32]),
        "ft_blob_layout": (ST, [I32, I32, C.POINTER(I64)]),
        "ft_last_error": (C.c_char_p, []),
        "ft_create": (ST, [C.POINTER(ModelDesc), P, P, C.POINTER(P)]),
        "ft_destroy": (ST, [P]),
        "ft_sync_status": (ST, [P, P]),
        "ft_router_logits": (ST, [P, P, I64, I32, P, I32, P, P]),
        "ft_moe_route": (ST, [P, P, I64, I32, I32, U32, P, P, P]),
        "ft_moe_permute": (ST, [P, P, I64, I32, I32, P, P, P, P]),
        "ft_quantize_mxfp4": (ST, [P, P, I64, I32, P, P, P]),
        "ft_quantize_nvfp4": (ST, [P, P, I64, I32, P, P, P, P]),
        "ft_moe_layer_forward": (ST, [P, I32, P, I64, P, P, P, U32, P]),
        "ft_expert_cache_lookup": (ST, [P, I32, I32, C.POINTER(I32)]),
        "ft_expert_cache_insert": (ST, [P, I32, I32, C.POINTER(I32), C.POINTER(I64), P]),
        "ft_expert_cache_resize": (ST, [P, I64]),
        "ft_cache_trace": (ST, [P, C.POINTER(CacheEvent), I64, C.POINTER(I64)]),
        "ft_cache_stats_get": (ST, [P, C.POINTER(CacheStats), I32]),
        "ft_prefetch_layer": (ST, [P, I32, P]),
        "ft_debug_dequant": (ST, [P, P, I32, P, P]),
        "ft_kernel_timing_enable": (ST, [P, I32]),
        "ft_kernel_timing_read": (ST, [P, C.POINTER(C.c_double), C.POINTER(I64), I32]),
        "ft_moe_layer_forward_noalloc": (ST, [I32, I32, I32, I32, I32, P, P, I64, P, P, P, U32, P, P]),
        "ft_moe_stack_forward": (ST, [P, I32, I32, P, I64, P, P, U32, P]),
        "ft_last_routing": (ST, [P, P, P, I64, P]),
        "ft_debug_device_wait": (ST, [P, I64, P]),
        "ft_debug_host_wait_limit": (ST, [P, C.c_double]),
        "ft_debug_fail_copy": (ST, [P, I64]),
        "ft_debug_stack_epoch": (ST, [P, U32, I32]),
        "ft_flow_geometry": (ST, [I32, I32, I32, I32, I32, I32, I32, I32, C.POINTER(I64)]),
        "ft_blob_layout_format": (ST, [I32, I32, I32, C.POINTER(I64)]),
        "ft_cache_prefetch": (ST, [P, I32]),
        "ft_debug_stack_timeline": (ST, [P, P, I64]),
        "ft_fp4_mma_probe": (ST, [I64, P, P, C.POINTER(I32), P]),
        "ft_decode_geometry": (ST, [I32, I32, I32, C.POINTER(I64)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _ptr(t, size: int | None = None) -> int | None:
    """Device/host pointer of a torch tensor, a numpy array (host), an int, or
    None.  The ABI takes
    dense row-major buffers, so a strided view is refused rather than read
    with the wrong layout; `size` is the element size in bytes the argument
    holds (2 for bf16 activations, 4 for fp32 / int32, 1 for codes), checked
    on tensors."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "__array_interface__") and not hasattr(t, "is_contiguous"):  # a numpy host buffer
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError(f"array of shape {t.shape} is not C-contiguous; the C ABI takes dense row-major buffers")
        if size is not None and t.itemsize != size:
            raise ValueError(f"array of dtype {t.dtype} has {t.itemsize}-byte elements where the C ABI "
                             f"takes {size}-byte ones")
        return t.ctypes.data
    if not t.is_contiguous():
        raise ValueError(f"tensor of shape {tuple(t.shape)} and strides {t.stride()} is not contiguous; "
                         "the C ABI takes dense row-major buffers")
    if size is not None and t.element_size() != size:
        raise ValueError(f"tensor of dtype {t.dtype} has {t.element_size()}-byte elements where the C ABI "
                         f"takes {size}-byte ones")
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int) -> None:
    if st != FT_OK:
        raise FtError(st, lib().ft_last_error().decode(errors="replace"))


# ---------------------------------------------------------------------------
# C ABI, same names
# ---------------------------------------------------------------------------

def ft_blob_stride(hidden: int, inter: int) -> int:
    return lib().ft_blob_stride(hidden, inter)


def ft_blob_layout(hidden: int, inter: int) -> dict:
    out = (I64 * 8)()
    _check(lib().ft_blob_layout(hidden, inter, out))
    return dict(zip(("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "used", "stride"), list(out)))


FT_FMT_MXFP4, FT_FMT_NVFP4, FT_FMT_BF16 = 0, 1, 2


def ft_blob_layout_format(hidden: int, inter: int, fmt: int) -> dict:
    out = (I64 * 9)()
    _check(lib().ft_blob_layout_format(hidden, inter, fmt, out))
    return dict(zip(("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "used", "stride", "ts"), list(out)))


# Buffers a context borrows (its host and resident pools), held here from
# ft_create until ft_destroy: the library keeps their addresses, so a tensor
# the caller dropped must not return to torch's allocator meanwhile.
_borrowed: dict[int, tuple] = {}


def ft_create(desc: ModelDesc, host_layers=None, resident_layers=None) -> int:
    """Returns the context handle.  host_layers / resident_layers: sequences of
    per-layer pointers (tensors, numpy arrays, ints or None) or None; the
    objects are held until ft_destroy of the handle."""
    L = desc.n_layers

    def arr(seq):
        if seq is None:
            return None
        a = (P * L)()
        for i in range(L):
            a[i] = _ptr(seq[i]) if seq[i] is not None else None
        return a
    h, r = arr(host_layers), arr(resident_layers)
    out = P()
    _check(lib().ft_create(C.byref(desc), C.cast(h, P) if h is not None else None,
                           C.cast(r, P) if r is not None else None, C.byref(out)))
    _borrowed[out.value] = (None if host_layers is None else list(host_layers),
                            None if resident_layers is None else list(resident_layers))
    return out.value


def ft_destroy(ctx: int) -> None:
    try:
        _check(lib().ft_destroy(ctx))
    finally:
        _borrowed.pop(ctx, None)


def ft_sync_status(ctx: int, stream=None) -> None:
    _check(lib().ft_sync_status(ctx, _stream(stream)))


def ft_router_logits(ctx, x, T, H, wr, E, logits, stream=None) -> None:
    _check(lib().ft_router_logits(ctx, _ptr(x, 2), T, H, _ptr(wr, 4), E, _ptr(logits, 4), _stream(stream)))


def ft_moe_route(ctx, logits, T, E, k, flags, ids, w, stream=None) -> None:
    _check(lib().ft_moe_route(ctx, _ptr(logits, 4), T, E, k, flags, _ptr(ids, 4), _ptr(w, 4), _stream(stream)))


def ft_moe_permute(ctx, ids, T, k, E, offs, perm, inv, stream=None) -> None:
    _check(lib().ft_moe_permute(ctx, _ptr(ids, 4), T, k, E, _ptr(offs, 4), _ptr(perm, 4), _ptr(inv, 4),
                                _stream(stream)))


def ft_quantize_mxfp4(ctx, x, R, K, codes, scales, stream=None) -> None:
    _check(lib().ft_quantize_mxfp4(ctx, _ptr(x, 4), R, K, _ptr(codes, 1), _ptr(scales, 1), _stream(stream)))


def ft_quantize_nvfp4(ctx, x, R, K, codes, scales, tensor_scale, stream=None) -> None:
    _check(lib().ft_quantize_nvfp4(ctx, _ptr(x, 4), R, K, _ptr(codes, 1), _ptr(scales, 1), _ptr(tensor_scale, 4),
                                   _stream(stream)))


def ft_moe_layer_forward(ctx, layer, x, T, router_w, logits_override, out, flags, stream=None) -> None:
    _check(lib().ft_moe_layer_forward(ctx, layer, _ptr(x, 2), T, _ptr(router_w, 4), _ptr(logits_override, 4),
                                      _ptr(out, 2), flags, _stream(stream)))


def ft_moe_stack_forward(ctx, first_layer, n_layers, x, T, logits, out, flags, stream=None) -> None:
    _check(lib().ft_moe_stack_forward(ctx, first_layer, n_layers, _ptr(x, 2), T, _ptr(logits, 4), _ptr(out, 2),
                                      flags, _stream(stream)))


def ft_last_routing(ctx, ids, w, n, stream=None) -> None:
    _check(lib().ft_last_routing(ctx, _ptr(ids, 4), _ptr(w, 4), n, _stream(stream)))


def ft_expert_cache_lookup(ctx, layer, expert) -> int:
    slot = I32()
    _check(lib().ft_expert_cache_lookup(ctx, layer, expert, C.byref(slot)))
    return slot.value


def ft_expert_cache_insert(ctx, layer, expert, stream=None) -> tuple[int, int]:
    slot, ev = I32(), I64()
    _check(lib().ft_expert_cache_insert(ctx, layer, expert, C.byref(slot), C.byref(ev), _stream(stream)))
    return slot.value, ev.value


def ft_expert_cache_resize(ctx, new_budget_bytes: int) -> None:
    _check(lib().ft_expert_cache_resize(ctx, new_budget_bytes))


def ft_cache_trace(ctx, cap: int = 1 << 20) -> list[tuple]:
    buf = (CacheEvent * cap)()
    n = I64()
    _check(lib().ft_cache_trace(ctx, buf, cap, C.byref(n)))
    return [(buf[i].kind, buf[i].layer, buf[i].expert, buf[i].slot, buf[i].from_slot) for i in range(n.value)]


def ft_debug_stack_timeline(ctx, buf=None) -> None:
    _check(lib().ft_debug_stack_timeline(ctx, _ptr(buf, 8), buf.numel() if buf is not None else 0))


def ft_cache_prefetch(ctx, per_layer: int) -> None:
    _check(lib().ft_cache_prefetch(ctx, per_layer))


def ft_cache_stats_get(ctx, reset: bool = False) -> dict:
    s = CacheStats()
    _check(lib().ft_cache_stats_get(ctx, C.byref(s), 1 if reset else 0))
    return {f: getattr(s, f) for f, _ in CacheStats._fields_}


def ft_prefetch_layer(ctx, layer, compute_stream=None) -> None:
    _check(lib().ft_prefetch_layer(ctx, layer, _stream(compute_stream)))


def ft_debug_dequant(ctx, blob, mat, out, stream=None) -> None:
    _check(lib().ft_debug_dequant(ctx, _ptr(blob), mat, _ptr(out), _stream(stream)))


def ft_debug_device_wait(ctx, timeout_us: int, stream=None) -> None:
    _check(lib().ft_debug_device_wait(ctx, timeout_us, _stream(stream)))


def ft_debug_host_wait_limit(ctx, seconds: float) -> None:
    _check(lib().ft_debug_host_wait_limit(ctx, seconds))


def ft_debug_fail_copy(ctx, n: int) -> None:
    _check(lib().ft_debug_fail_copy(ctx, n))


def ft_fp4_mma_probe(iters: int, sink, status, stream=None) -> int:
    """Launch the FP4 tensor-peak probe; returns the CTAs launched.  FLOPs =
    CTAs * iters * 4 * 2 * 128 * 128 * 64."""
    g = I32()
    _check(lib().ft_fp4_mma_probe(iters, _ptr(sink, 4), _ptr(status, 4), C.byref(g), _stream(stream)))
    return g.value


def ft_flow_geometry(hidden, inter, T, top_k, n_shared, n_experts, n_layers, weight_format=0) -> dict:
    out = (I64 * 3)()
    _check(lib().ft_flow_geometry(hidden, inter, T, top_k, n_shared, n_experts, n_layers, weight_format, out))
    return {"ok": bool(out[0]), "rows_cap": out[1], "smem": out[2]}


def ft_debug_stack_epoch(ctx, epoch: int, poison_layer: int = -1) -> None:
    _check(lib().ft_debug_stack_epoch(ctx, epoch & 0xFFFFFFFF, poison_layer))


GEOMETRY_FIELDS = ("K", "chunks", "lpr", "rpw", "parts", "rsets", "groups", "R", "smem", "taken")


def ft_decode_geometry(hidden: int, inter: int, n_layers: int = 1) -> dict:
    out = (I64 * 24)()
    _check(lib().ft_decode_geometry(hidden, inter, n_layers, out))
    tile = lambda o: {k: int(out[o + i]) for i, k in enumerate(GEOMETRY_FIELDS)}
    return {"gate_up": tile(0), "down": tile(10), "threads": int(out[20]), "smem_limit": int(out[21]),
            "stack": bool(out[22]), "sync_stride": int(out[23])}


def ft_kernel_timing_enable(ctx, on: bool) -> None:
    _check(lib().ft_kernel_timing_enable(ctx, 1 if on else 0))


def ft_kernel_timing_read(ctx) -> dict:
    n = len(KERNELS)
    ms = (C.c_double * n)()
    cnt = (I64 * n)()
    _check(lib().ft_kernel_timing_read(ctx, ms, cnt, n))
    return {KERNELS[i]: (ms[i], cnt[i]) for i in range(n)}


def ft_moe_layer_forward_noalloc(hidden, inter, n_experts, top_k, n_shared, layer_pool, x, T, router_w,
                                 logits_override, out, flags, status=None, stream=None) -> None:
    """Decode forward that allocates no device memory (scratch in a static
    device array shared by all calls; see ft_moe.h)."""
    _check(lib().ft_moe_layer_forward_noalloc(hidden, inter, n_experts, top_k, n_shared, _ptr(layer_pool),
                                              _ptr(x, 2), T, _ptr(router_w, 4), _ptr(logits_override, 4),
                                              _ptr(out, 2), flags, _ptr(status, 4), _stream(stream)))


def make_desc(hidden, inter, n_experts, top_k, n_layers=1, n_shared=0, cache_budget_bytes=0,
              max_tokens=16, weight_format=0) -> ModelDesc:
    return ModelDesc(hidden, inter, n_experts, top_k, n_layers, n_shared, cache_budget_bytes, max_tokens,
                     weight_format)
