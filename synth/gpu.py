"""ctypes binding of synth/libftsynth.so: fills expert blobs in device memory
with the same bytes as ``synth.gen.expert_blob`` (same counter-based draws)."""
from __future__ import annotations

import ctypes as C
import os

from .gen import blob_regions, bf16_blob_regions, nvfp4_blob_regions

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libftsynth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_PATH):
            raise RuntimeError(f"{_PATH} missing: run `python -m expert_offloaded_serving_b200.build`")
        _lib = C.CDLL(_PATH)
        _lib.ftsynth_fill_blobs.restype = C.c_int
        _lib.ftsynth_fill_blobs.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_uint64, C.c_int32,
                                           C.c_int32, C.c_int32, C.c_void_p]
        _lib.ftsynth_fill_blobs_bf16.restype = C.c_int
        _lib.ftsynth_fill_blobs_bf16.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_uint64, C.c_int32, C.c_int32,
                                                C.c_int32, C.c_void_p]
        _lib.ftsynth_fill_blobs_nvfp4.restype = C.c_int
        _lib.ftsynth_fill_blobs_nvfp4.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_uint64, C.c_int32,
                                                 C.c_int32, C.c_int32, C.c_void_p]
    return _lib


def fill_blobs(dst_ptr: int, hidden: int, inter: int, seed: int, layer: int, expert0: int, n: int,
               stream: int | None = None) -> None:
    """Write blobs of experts expert0 .. expert0+n-1 of `layer` at dst_ptr + i*stride (device)."""
    r = blob_regions(hidden, inter)
    rc = _load().ftsynth_fill_blobs(dst_ptr, r["stride"], r["codes_end"], r["used"], seed & 0xFFFFFFFFFFFFFFFF,
                                    layer, expert0, n, stream)
    if rc != 0:
        raise RuntimeError(f"ftsynth_fill_blobs failed with CUDA error {rc}")


FORMATS = ("mxfp4", "nvfp4", "bf16")


def fill_blobs_format(dst_ptr: int, hidden: int, inter: int, fmt: str, seed: int, layer: int, expert0: int, n: int,
                      stream: int | None = None) -> None:
    """As fill_blobs, for the blobs of ``synth.gen`` in format fmt (same bytes
    as expert_blob / expert_blob_nvfp4 / expert_blob_bf16)."""
    if fmt == "mxfp4":
        return fill_blobs(dst_ptr, hidden, inter, seed, layer, expert0, n, stream)
    s = seed & 0xFFFFFFFFFFFFFFFF
    if fmt == "bf16":
        r = bf16_blob_regions(hidden, inter)
        rc = _load().ftsynth_fill_blobs_bf16(dst_ptr, r["stride"], r["used"], s, layer, expert0, n, stream)
    elif fmt == "nvfp4":
        r = nvfp4_blob_regions(hidden, inter)
        rc = _load().ftsynth_fill_blobs_nvfp4(dst_ptr, r["stride"], r["codes_end"], r["tensor_scales"], s, layer,
                                              expert0, n, stream)
    else:
        raise ValueError(fmt)
    if rc != 0:
        raise RuntimeError(f"blob filler failed with CUDA error {rc}")


def blob_stride_format(hidden: int, inter: int, fmt: str) -> int:
    return {"mxfp4": blob_regions, "nvfp4": nvfp4_blob_regions, "bf16": bf16_blob_regions}[fmt](hidden, inter)["stride"]


def layer_pool(hidden: int, inter: int, n_blobs: int, seed: int, layer: int, device="cuda", fmt: str = "mxfp4"):
    """A device uint8 tensor holding one layer's n_blobs blobs (format fmt)."""
    import torch
    stride = blob_stride_format(hidden, inter, fmt)
    t = torch.empty(n_blobs * stride, dtype=torch.uint8, device=device)
    fill_blobs_format(t.data_ptr(), hidden, inter, fmt, seed, layer, 0, n_blobs,
                      torch.cuda.current_stream().cuda_stream)
    return t
