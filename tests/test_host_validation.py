"""Argument checks of the C ABI that run before any CUDA call, so they are
tested without a GPU: every refusal of ft_create's descriptor check and of the
allocation-free forward (fake, never dereferenced pointers stand in for
device buffers)."""
import pytest

import expert_offloaded_serving_b200 as ft

# stand-ins for device pointers: the calls refuse before touching them
POOL, X, OUT, LG, WR = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000


@pytest.mark.parametrize("desc,what", [
    (dict(hidden=100), "hidden"),
    (dict(hidden=0), "hidden"),
    (dict(inter=96), "inter"),
    (dict(n_experts=0), "n_experts"),
    (dict(n_experts=1025), "n_experts"),
    (dict(top_k=0), "top_k"),
    (dict(top_k=17), "top_k"),
    (dict(n_experts=4, top_k=5), "top_k"),
    (dict(n_layers=0), "n_layers"),
    (dict(n_shared=2), "n_shared"),
    (dict(cache_budget_bytes=-1), "budget"),
    (dict(max_tokens=0), "max_tokens"),
    (dict(weight_format=3), "weight_format"),
    (dict(weight_format=-1), "weight_format"),
])
def test_create_refuses_each_bad_descriptor_field(desc, what):
    base = dict(hidden=256, inter=128, n_experts=16, top_k=2, n_layers=1, n_shared=0, cache_budget_bytes=0,
                max_tokens=16)
    desc = dict(desc)
    fmt = desc.pop("weight_format", 0)
    base.update(desc)
    d = ft.make_desc(**base)
    d.weight_format = fmt
    with pytest.raises(ft.FtError) as e:
        ft.ft_create(d)
    assert e.value.status == ft.FT_ERR_INVALID
    assert what in str(e.value)


def noalloc(**kw):
    a = dict(hidden=256, inter=128, n_experts=16, top_k=2, n_shared=0, layer_pool=POOL, x=X, T=1, router_w=None,
             logits_override=LG, out=OUT, flags=ft.FT_ROUTE_RENORM)
    a.update(kw)
    ft.ft_moe_layer_forward_noalloc(a["hidden"], a["inter"], a["n_experts"], a["top_k"], a["n_shared"],
                                    a["layer_pool"], a["x"], a["T"], a["router_w"], a["logits_override"], a["out"],
                                    a["flags"], None, 0)  # stream 0: never used, the call refuses first


@pytest.mark.parametrize("kw,what", [
    (dict(layer_pool=None), "NULL"),
    (dict(out=None), "NULL"),
    (dict(x=None), "NULL"),
    (dict(hidden=200), "multiples of 128"),
    (dict(inter=0), "multiples of 128"),
    # the split-K GEMV spreads a row over min(32, K/32) lanes: that count must
    # be a power of two and divide K/32 (K = 384 gives 12 lanes, K = 1152 gives
    # 36 chunks over 32 lanes)
    (dict(hidden=384), "multiple of 1024"),
    (dict(hidden=1152), "multiple of 1024"),
    (dict(inter=384), "multiple of 1024"),
    (dict(inter=1152), "multiple of 1024"),
    (dict(hidden=15360), "at most 14336"),
    (dict(n_experts=2000), "expert counts"),
    (dict(top_k=17), "expert counts"),
    (dict(n_shared=2), "expert counts"),
    (dict(T=17), "T outside"),
    (dict(T=-1), "T outside"),
    (dict(flags=ft.FT_ACT_MXFP4), "decode"),
    (dict(logits_override=None, router_w=None), "router_w or logits_override"),
    (dict(out=X), "alias"),
    # (16*8 + 16) rows of h at inter 16384 in fp32: 9.4 MB > 8 MiB of scratch
    (dict(hidden=1024, inter=16384, top_k=8, n_shared=1, T=16), "maximum"),
])
def test_noalloc_refuses_before_touching_the_device(kw, what):
    with pytest.raises(ft.FtError) as e:
        noalloc(**kw)
    assert e.value.status == ft.FT_ERR_INVALID
    assert what in str(e.value)


def test_noalloc_with_no_tokens_is_a_no_op():
    noalloc(T=0)
    noalloc(T=0, x=None)


def test_binding_refuses_strided_views():
    """The binding passes data pointers: a transposed or sliced-with-step view
    would be read as if dense, so it is refused before the library is called."""
    import torch
    x = torch.zeros(8, 4, dtype=torch.bfloat16).t()
    with pytest.raises(ValueError, match="not contiguous"):
        ft.ft_moe_layer_forward(0, 0, x, 4, None, torch.zeros(4, 16), torch.zeros(4, 8), 1, 0)
    with pytest.raises(ValueError, match="not contiguous"):
        ft.ft_moe_route(0, torch.zeros(4, 32)[:, ::2], 4, 16, 2, 1, torch.zeros(4, 2, dtype=torch.int32),
                        torch.zeros(4, 2), 0)


def test_binding_refuses_wrong_element_sizes():
    """fp32 where bf16 activations go, or int64 ids, would be misread: refused."""
    import torch
    with pytest.raises(ValueError, match="2-byte"):
        ft.ft_moe_layer_forward(0, 0, torch.zeros(4, 8), 4, None, torch.zeros(4, 16), torch.zeros(4, 8), 1, 0)
    with pytest.raises(ValueError, match="4-byte"):
        ft.ft_moe_route(0, torch.zeros(4, 16), 4, 16, 2, 1, torch.zeros(4, 2, dtype=torch.int64), torch.zeros(4, 2),
                        0)


def test_binding_takes_numpy_host_buffers():
    """Host pools may be numpy arrays (pageable memory the context pins): the
    binding passes their data pointer, and refuses strided ones like tensors."""
    import numpy as np
    a = np.zeros(64, np.uint8)
    assert ft._ptr(a) == a.ctypes.data
    f = np.zeros(4, np.float32)
    assert ft._ptr(f, 4) == f.ctypes.data
    with pytest.raises(ValueError, match="not C-contiguous"):
        ft._ptr(np.zeros((4, 4), np.uint8)[:, ::2])
    with pytest.raises(ValueError, match="4-byte"):
        ft._ptr(np.zeros(4, np.float64), 4)


def test_binding_holds_borrowed_pools_until_destroy(monkeypatch):
    """The context keeps the addresses of its host and resident pools, so the
    binding holds the objects from ft_create to ft_destroy: a pool passed
    inline and dropped by the caller must not go back to the allocator (and
    be reused under the context) meanwhile.  A fake library stands in for the
    C calls."""
    import gc
    import weakref

    import numpy as np

    class FakeLib:
        def ft_create(self, desc, host, res, out):
            out._obj.value = 0x7000
            return ft.FT_OK

        def ft_destroy(self, ctx):
            return ft.FT_OK

    monkeypatch.setattr(ft, "lib", lambda: FakeLib())
    host, res = np.zeros(64, np.uint8), np.zeros(64, np.uint8)
    wh, wr = weakref.ref(host), weakref.ref(res)
    d = ft.make_desc(256, 128, 16, 2, 1, 0, 0, 16)
    h = ft.ft_create(d, [host], [res])
    del host, res
    gc.collect()
    assert wh() is not None and wr() is not None
    ft.ft_destroy(h)
    gc.collect()
    assert wh() is None and wr() is None


@pytest.mark.parametrize("kw", [dict(layer_pool=POOL + 8), dict(x=X + 2), dict(out=OUT + 4), dict(logits_override=LG + 8),
                                dict(router_w=WR + 4, logits_override=None)])
def test_noalloc_refuses_misaligned_buffers(kw):
    """Buffers the kernels access with vector loads and stores must start on a
    16-byte boundary; others are refused before any launch."""
    with pytest.raises(ft.FtError) as e:
        noalloc(**kw)
    assert e.value.status == ft.FT_ERR_INVALID and "16-byte" in str(e.value)
