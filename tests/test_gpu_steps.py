"""GPU parity of the single hot-path steps against the oracle, through the
C ABI: seeded inputs, blob filler, dequantisation, router logits, top-k,
permutation, MXFP4 quantiser."""
import numpy as np
import pytest
import torch

import expert_offloaded_serving_b200 as ft
import synth
import synth.gpu
from oracle import fp4, routing

from _gpu import Ctx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    c = Ctx(ft.make_desc(4096, 2048, 256, 8, max_tokens=4096))
    yield c.h
    c.close()


@pytest.mark.parametrize("H,I", [(256, 128), (2048, 512), (4096, 2048)])
def test_gpu_blob_filler_matches_numpy_generator(H, I):
    stride = synth.blob_stride(H, I)
    t = torch.empty(3 * stride, dtype=torch.uint8, device="cuda")
    synth.gpu.fill_blobs(t.data_ptr(), H, I, 77, 5, 10, 3)
    torch.cuda.synchronize()
    got = t.cpu().numpy()
    for i in range(3):
        assert (got[i * stride:(i + 1) * stride] == synth.expert_blob(77, 5, 10 + i, H, I)).all()


@pytest.mark.parametrize("H,I", [(256, 128), (2048, 512), (4096, 2048)])
def test_gpu_dequant_bit_exact(H, I):
    c = Ctx(ft.make_desc(H, I, 16, 2))
    try:
        blob = synth.expert_blob(3, 0, 1, H, I)
        # plant extreme scale bytes (0 and 254) and every code in the first atom rows
        off = fp4.layout(H, I)
        blob[off["wg_sf"]:off["wg_sf"] + 64] = np.arange(64, dtype=np.uint8) * 4 % 255
        blob[off["wd_sf"]] = 0
        blob[off["wd_sf"] + 1] = 254
        d = torch.from_numpy(blob).cuda()
        for mat, name, shape in ((0, "wg", (I, H)), (1, "wu", (I, H)), (2, "wd", (H, I))):
            out = torch.empty(shape, dtype=torch.float32, device="cuda")
            ft.ft_debug_dequant(c.h, d, mat, out)
            want = fp4.dequant_matrix(blob, name, H, I).astype(np.float32)
            got = out.cpu().numpy()
            assert (got.view(np.uint32) == want.view(np.uint32)).all(), name
    finally:
        c.close()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 8, 33, 63, 64, 300])
@pytest.mark.parametrize("H,E", [(256, 16), (2048, 256), (4096, 256)])
def test_gpu_router_logits_bit_exact(ctx, T, H, E):
    xb = synth.activations_bf16(11, T, T, H)
    wr = synth.router_weights(11, T, E, H)
    x = torch.from_numpy(xb.view(np.int16)).cuda()
    w = torch.from_numpy(wr).cuda()
    out = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ft.ft_router_logits(ctx, x, T, H, w, E, out)
    want = routing.router_logits(fp4.bf16_to_f64(xb), wr)
    assert (out.cpu().numpy().view(np.uint32) == want.view(np.uint32)).all()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 8, 33, 4096])
@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (256, 6), (1024, 16)])
@pytest.mark.parametrize("renorm", [True, False])
def test_gpu_topk(ctx, T, E, k, renorm):
    rng = np.random.default_rng(T * 1000 + E + k)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[::3, ::7] = 0.75                      # exact ties
    lg[1::5, 2] = -0.0
    lg[1::5, 3] = 0.0
    lg[::11, 5] = -np.inf
    d = torch.from_numpy(lg).cuda()
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ft.ft_moe_route(ctx, d, T, E, k, ft.FT_ROUTE_RENORM if renorm else 0, ids, w)
    ft.ft_sync_status(ctx)
    want_ids, bad = routing.topk(lg, k)
    assert (ids.cpu().numpy() == want_ids).all()
    want_w = routing.softmax_weights(lg, want_ids, renorm)
    assert np.allclose(w.cpu().numpy(), want_w, rtol=2e-6, atol=1e-9)


def test_gpu_topk_nonfinite_sets_status(ctx):
    lg = np.zeros((4, 16), np.float32)
    lg[2, 3] = np.nan
    d = torch.from_numpy(lg).cuda()
    ids = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 2), dtype=torch.float32, device="cuda")
    ft.ft_moe_route(ctx, d, 4, 16, 2, 1, ids, w)
    with pytest.raises(ft.FtError) as e:
        ft.ft_sync_status(ctx)
    assert e.value.status == ft.FT_ERR_NONFINITE
    # NaN ranks last: row 2 still picks ids 0, 1
    assert ids.cpu().numpy()[2].tolist() == [0, 1]
    ft.ft_sync_status(ctx)  # cleared


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 8, 33, 4096])
@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (256, 6)])
def test_gpu_permutation_bit_exact(ctx, T, E, k):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    d = torch.from_numpy(ids).cuda()
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ft.ft_moe_permute(ctx, d, T, k, E, offs, perm, inv)
    ft.ft_sync_status(ctx)
    o, p, i = routing.permutation(ids, E)
    assert (offs.cpu().numpy() == o).all()
    assert (perm.cpu().numpy() == p).all()
    assert (inv.cpu().numpy() == i).all()


def test_gpu_permutation_bad_id(ctx):
    ids = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32, device="cuda")
    offs = torch.empty(17, dtype=torch.int32, device="cuda")
    perm = torch.empty(4, dtype=torch.int32, device="cuda")
    inv = torch.empty(4, dtype=torch.int32, device="cuda")
    ft.ft_moe_permute(ctx, ids, 2, 2, 16, offs, perm, inv)
    with pytest.raises(ft.FtError) as e:
        ft.ft_sync_status(ctx)
    assert e.value.status == ft.FT_ERR_INVALID


@pytest.mark.parametrize("R,K", [(1, 128), (37, 256), (300, 4096)])
def test_gpu_quantiser_bit_exact(ctx, R, K):
    rng = np.random.default_rng(R + K)
    x = (rng.standard_normal((R, K)) * np.exp(rng.uniform(-8, 8, (R, 1)))).astype(np.float32)
    # planted blocks: zeros, grid midpoints (ties), saturation, negative values rounding to zero
    x[0, :32] = 0.0
    x[0, 32:64] = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4) * np.float32(0.5)
    x[0, 64:96] = np.float32(-0.01)
    x[0, 64] = np.float32(4.0)
    if R > 2:
        x[1, :32] = (np.arange(32, dtype=np.float32) - 16) * np.float32(1e-40)   # subnormal block
    d = torch.from_numpy(x).cuda()
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
    nsf = fp4._pad(R, 128) * fp4._pad(K // 32, 4)
    scales = torch.zeros(nsf, dtype=torch.uint8, device="cuda")
    ft.ft_quantize_mxfp4(ctx, d, R, K, codes, scales)
    want_codes, want_sc = fp4.quantize_rows(x.astype(np.float64))
    assert (codes.cpu().numpy() == fp4.pack_codes(want_codes)).all()
    sc = scales.cpu().numpy()
    r = np.arange(R)[:, None]
    b = np.arange(K // 32)[None, :]
    assert (sc[fp4.scale_index(r, b, K // 32)] == want_sc).all()


def test_misaligned_buffers_are_refused():
    """A buffer that does not start on a 16-byte boundary (here a view two
    bytes into an allocation) is refused on the host with FT_ERR_INVALID
    before any launch: the forward, the stacked forward, the router logits,
    and a resident pool at context creation."""
    H, I, E, k, T = 256, 128, 16, 2, 4
    big = torch.zeros(T * H + 16, dtype=torch.bfloat16, device="cuda")
    xm = big[1:1 + T * H].view(T, H)                          # 2 bytes past the allocation's start
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    pool = synth.gpu.layer_pool(H, I, E, 77, 0)
    with Ctx(ft.make_desc(H, I, E, k, 1, 0, 0, 16), None, [pool]) as c:
        calls = [lambda: ft.ft_moe_layer_forward(c.h, 0, xm, T, None, lg, out, ft.FT_ROUTE_RENORM),
                 lambda: ft.ft_moe_stack_forward(c.h, 0, 1, xm, T, lg, out, ft.FT_ROUTE_RENORM),
                 lambda: ft.ft_router_logits(c.h, xm, T, H, torch.zeros((E, H), device="cuda"), E, lg)]
        for call in calls:
            with pytest.raises(ft.FtError) as e:
                call()
            assert e.value.status == ft.FT_ERR_INVALID and "16-byte" in str(e.value)
        ft.ft_sync_status(c.h)
    with pytest.raises(ft.FtError) as e:
        ft.ft_create(ft.make_desc(H, I, E, k, 1, 0, 0, 16), None, [pool[8:]])
    assert e.value.status == ft.FT_ERR_INVALID and "16-byte" in str(e.value)
