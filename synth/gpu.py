"""ctypes binding of synth/libftsynth.so: fills expert blobs in device memory
with the same bytes as ``synth.gen.expert_blob`` (same counter-based draws)."""
from __future__ import annotations

import ctypes as C
import os

from .gen import blob_regions

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
    return _lib


def fill_blobs(dst_ptr: int, hidden: int, inter: int, seed: int, layer: int, expert0: int, n: int,
               stream: int | None = None) -> None:
    """Write blobs of experts expert0 .. expert0+n-1 of `layer` at dst_ptr + i*stride (device)."""
    r = blob_regions(hidden, inter)
    rc = _load().ftsynth_fill_blobs(dst_ptr, r["stride"], r["codes_end"], r["used"], seed & 0xFFFFFFFFFFFFFFFF,
                                    layer, expert0, n, stream)
    if rc != 0:
        raise RuntimeError(f"ftsynth_fill_blobs failed with CUDA error {rc}")


def layer_pool(hidden: int, inter: int, n_blobs: int, seed: int, layer: int, device="cuda"):
    """A device uint8 tensor holding one layer's n_blobs blobs."""
    import torch
    stride = blob_regions(hidden, inter)["stride"]
    t = torch.empty(n_blobs * stride, dtype=torch.uint8, device=device)
    fill_blobs(t.data_ptr(), hidden, inter, seed, layer, 0, n_blobs, torch.cuda.current_stream().cuda_stream)
    return t
