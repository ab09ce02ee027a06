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


def test_every_declaration_is_documented():
    """Each entry point of the header has its own comment above it, or is
    named in an earlier comment block that documents it with its neighbours
    (meaning of the arguments, layouts, ownership, errors live there)."""
    src = open(os.path.join(ROOT, "include", "ft_moe.h")).read()
    comments = [m for m in re.finditer(r"/\*.*?\*/", src, flags=re.S)]
    prev = 0
    for m in re.finditer(r"^FT_API\s+[\w\s\*]*?\b(ft_\w+)\s*\(", src, flags=re.M):
        name = m.group(1)
        own = [c for c in comments if prev <= c.start() and c.end() <= m.start() and len(c.group(0)) > 40]
        named = [c for c in comments if c.end() <= m.start() and name in c.group(0)]
        assert own or named, name
        prev = src.index(";", m.end()) + 1
