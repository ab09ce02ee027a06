"""The C ABI library loads without a GPU and exports every declared symbol;
its host-side format helpers agree with the oracle's reading of the format."""
import ctypes
import os
import re

import pytest

import expert_offloaded_serving_b200 as ft
from oracle import fp4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ft_moe.h")).read()
    return sorted(set(re.findall(r"^FT_API\s+[\w\s\*]*?\b(ft_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(ft.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(ft.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(L, name), name


@pytest.mark.parametrize("H,I", [(256, 128), (2048, 512), (4096, 2048), (6144, 2048), (32, 32), (512, 96)])
def test_blob_layout_matches_oracle(H, I):
    got = ft.ft_blob_layout(H, I)
    want = fp4.layout(H, I)
    for k in ("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "used", "stride"):
        assert got[k] == want[k], k
    assert ft.ft_blob_stride(H, I) == want["stride"]


def test_blob_layout_rejects_bad_shape():
    with pytest.raises(ft.FtError):
        ft.ft_blob_layout(100, 128)
    assert ft.ft_blob_stride(0, 128) == -1


def test_create_rejects_bad_desc_without_touching_the_gpu():
    with pytest.raises(ft.FtError) as e:
        ft.ft_create(ft.make_desc(100, 128, 16, 2))
    assert e.value.status == ft.FT_ERR_INVALID
    with pytest.raises(ft.FtError):
        ft.ft_create(ft.make_desc(256, 128, 16, 17))
