"""Helpers for the GPU parity tests (not collected by pytest)."""
from __future__ import annotations

import numpy as np
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu

# layer-output tolerance: fp32 accumulation, one bf16 rounding
MAX_ABS = 2e-2
REL_L2 = 2e-3


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def assert_close(got_bits: np.ndarray, want: np.ndarray):
    g = bits_to_f64(got_bits)
    want = np.asarray(want, np.float64)
    err = np.abs(g - want)
    rel = np.linalg.norm(g - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= MAX_ABS, f"max abs {err.max():.3e}"
    assert rel <= REL_L2, f"rel L2 {rel:.3e}"
    return err.max(), rel


def assert_close_scaled(got_bits: np.ndarray, want: np.ndarray):
    """The layer tolerance on outputs divided by their largest magnitude, for
    inputs whose outputs span many binades (wide-range block scales): max
    |got - want| <= MAX_ABS * max |want| and relative L2 <= REL_L2.  Every
    output must be finite."""
    g = bits_to_f64(got_bits)
    want = np.asarray(want, np.float64)
    assert np.isfinite(g).all() and np.isfinite(want).all()
    scale = np.abs(want).max()
    assert scale > 0
    err = np.abs(g - want) / scale
    rel = np.linalg.norm(g - want) / np.linalg.norm(want)
    assert err.max() <= MAX_ABS, f"max abs / max |want| {err.max():.3e}"
    assert rel <= REL_L2, f"rel L2 {rel:.3e}"
    return err.max(), rel


class Ctx:
    def __init__(self, desc, host_layers=None, resident_layers=None):
        self.desc = desc
        self.h = ft.ft_create(desc, host_layers, resident_layers)

    def close(self):
        if self.h:
            ft.ft_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def x_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).cuda().view(torch.bfloat16)


def layer_blobs_np(seed, layer, H, I, experts):
    return {int(e): synth.expert_blob(seed, layer, int(e), H, I) for e in experts}
