"""Tile geometry of the decode GEMV kernels (host logic, no GPU): for every
shape the kernels take, the tile fits shared memory, covers K and the rows
exactly, and keeps the row loop's trip count equal for all lanes of a warp
(the xor-shuffle reductions need the whole warp); shapes past the limits are
refused."""
import pytest

import expert_offloaded_serving_b200 as ft

SIZES = [128, 256, 384, 512, 640, 768, 1024, 1536, 2048, 2560, 3072, 4096, 5120, 6144, 7168, 8192, 12288, 16384]
OPT_IN_SMEM = 227 * 1024


def is_pow2(v):
    return v > 0 and (v & (v - 1)) == 0


def check_tile(t, K, rows, threads, limit):
    warps = threads // 32
    assert t["K"] == K and t["chunks"] == K // 32
    assert is_pow2(t["lpr"]) and t["lpr"] <= 32 and t["lpr"] * t["rpw"] == 32
    assert t["lpr"] >= min(t["chunks"], 32)            # a lane group spans all chunks it can
    assert t["parts"] * t["lpr"] >= t["chunks"] > (t["parts"] - 1) * t["lpr"]
    assert 1 <= t["rsets"] and t["rsets"] * t["parts"] <= warps
    assert t["groups"] == t["rsets"] * t["rpw"]
    assert is_pow2(t["R"]) and 8 <= t["R"] <= 128 and rows % t["R"] == 0
    assert t["smem"] <= 128 + limit <= OPT_IN_SMEM
    # several lane groups share a warp only with one K part, and then R is a
    # multiple of the groups per warp: every lane of a warp runs the same rows loop
    if t["rpw"] > 1:
        assert t["parts"] == 1 and t["R"] % t["rpw"] == 0


@pytest.mark.parametrize("H", SIZES)
@pytest.mark.parametrize("I", [128, 512, 768, 1536, 2048, 4096])
def test_tiles_of_every_supported_shape(H, I):
    g = ft.ft_decode_geometry(H, I, 40)
    assert g["threads"] == 512
    assert g["gate_up"]["taken"] and g["down"]["taken"]
    check_tile(g["gate_up"], H, I, g["threads"], g["smem_limit"])
    check_tile(g["down"], I, H, g["threads"], g["smem_limit"])
    if g["stack"]:
        assert g["sync_stride"] == 2 + H // g["down"]["R"]


def test_35b_class_tiles_and_stack():
    g = ft.ft_decode_geometry(2048, 512, 40)
    assert (g["gate_up"]["R"], g["gate_up"]["lpr"], g["gate_up"]["parts"]) == (32, 32, 2)
    assert (g["down"]["R"], g["down"]["lpr"], g["down"]["rpw"]) == (128, 16, 2)
    # 9 units (8 routed + shared) x I/R = 144 gate/up tiles and x H/R = 144 down
    # tiles: one of each per CTA on 148 SMs
    assert 9 * 512 // g["gate_up"]["R"] == 144 and 9 * 2048 // g["down"]["R"] == 144
    assert g["stack"] and g["sync_stride"] == 18


def test_limits_are_refused():
    g = ft.ft_decode_geometry(16384 + 128, 512, 1)        # K past 16384 chunks-per-warp coverage
    assert not g["gate_up"]["taken"]
    g = ft.ft_decode_geometry(2048, 512, 100000)           # the per-layer tile table outgrows shared memory
    assert not g["stack"] and g["sync_stride"] == 0
    with pytest.raises(ft.FtError) as e:
        ft.ft_decode_geometry(2000, 512, 1)
    assert e.value.status == ft.FT_ERR_INVALID


@pytest.mark.parametrize("shape", [(2048, 512, 256, 8, 1, 40), (4096, 2048, 256, 6, 0, 43), (6144, 2048, 256, 8, 0, 8),
                                   (256, 128, 16, 2, 0, 4), (1024, 512, 64, 4, 0, 3), (1024, 768, 64, 4, 1, 3),
                                   (256, 256, 16, 4, 1, 3)])
@pytest.mark.parametrize("T", [1, 2])
def test_dataflow_kernel_geometry(shape, T):
    """The dataflow stack kernel takes the workload shapes at one and two
    tokens: its CTA fits the opt-in shared memory, and a down tile has room
    for two rows of every unit a layer can have (rb >= 2, even)."""
    H, I, E, k, S, L = shape
    g = ft.ft_flow_geometry(H, I, T, k, S, E, L)
    assert g["ok"] and g["smem"] <= OPT_IN_SMEM
    units = min(E, T * k) + S
    assert g["rows_cap"] % 2 == 0 and g["rows_cap"] >= 2 * units


def test_dataflow_kernel_limits():
    """Three or more tokens, or more than 127 layers (the tag holds the layer
    in 7 bits), go to the other kernels."""
    assert not ft.ft_flow_geometry(2048, 512, 3, 8, 1, 256, 40)["ok"]
    assert not ft.ft_flow_geometry(2048, 512, 1, 8, 1, 256, 128)["ok"]
    assert ft.ft_flow_geometry(2048, 512, 1, 8, 1, 256, 127)["ok"]


@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("T", [1, 2])
def test_dataflow_kernel_geometry_other_formats(fmt, T):
    """NVFP4 and BF16 experts at the 35B-class shape (the formats' decode
    benchmark) fit the dataflow kernel at one and two tokens."""
    g = ft.ft_flow_geometry(2048, 512, T, 8, 1, 256, 40, fmt)
    assert g["ok"] and g["smem"] <= OPT_IN_SMEM


def test_blob_layout_formats():
    """Blob sizes of the three formats at the 35B-class shape, from the
    definitions: MXFP4 3HI(1/2 + 1/32); NVFP4 3HI(1/2 + 1/16) + 16 bytes of
    matrix scales, padded to 256; BF16 6HI."""
    H, I = 2048, 512
    mx = ft.ft_blob_layout_format(H, I, 0)
    nv = ft.ft_blob_layout_format(H, I, 1)
    bf = ft.ft_blob_layout_format(H, I, 2)
    assert mx["stride"] == 3 * H * I * 17 // 32 and mx["ts"] == -1
    assert nv["ts"] == 3 * H * I * 9 // 16 and nv["used"] == nv["ts"] + 16 and nv["stride"] == nv["used"] + 240
    assert bf["used"] == bf["stride"] == 6 * H * I
    import synth
    assert synth.nvfp4_blob_regions(H, I)["stride"] == nv["stride"]
    assert synth.bf16_blob_regions(H, I)["stride"] == bf["stride"]
