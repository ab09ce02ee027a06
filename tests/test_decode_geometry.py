"""Tile geometry of the decode GEMV kernels (host logic, no GPU): for every
shape the kernels take, the tile fits shared memory, covers K and the rows
exactly in whole 16-row tensor-core tasks, and its staged rows fall in
distinct shared-memory banks; shapes past the limits are refused."""
import pytest

import expert_offloaded_serving_b200 as ft

SIZES = [128, 256, 384, 512, 640, 768, 1024, 1536, 2048, 2560, 3072, 4096, 5120, 6144, 7168, 8192, 12288, 16384]
OPT_IN_SMEM = 227 * 1024


def is_pow2(v):
    return v > 0 and (v & (v - 1)) == 0


def check_tile(t, K, rows, nmat, threads, limit):
    assert t["K"] == K and t["chunks"] == K // 32
    # K parts of 8 blocks of 32 when K allows, else of 4; they cover K exactly
    assert t["pblk"] == (8 if K % 256 == 0 else 4) and t["parts"] * t["pblk"] == t["chunks"]
    assert is_pow2(t["R"]) and 8 <= t["R"] <= 128 and rows % t["R"] == 0
    assert (nmat * t["R"]) % 16 == 0 and t["tasks"] == nmat * t["R"] // 16 * t["parts"]
    # a staged row holds the row's codes; consecutive rows start 64 bytes apart
    # modulo 128 (the 16-byte loads of 8 rows hit distinct banks); an odd count
    # of scale words per row
    assert t["rstride"] >= K // 2 and t["rstride"] % 128 == 64 and t["rstride"] % 16 == 0
    assert t["sstride"] % 2 == 1 and t["sstride"] >= K // 128
    assert t["smem"] <= 128 + limit <= OPT_IN_SMEM


@pytest.mark.parametrize("H", SIZES)
@pytest.mark.parametrize("I", [128, 512, 768, 1536, 2048, 4096])
def test_tiles_of_every_supported_shape(H, I):
    g = ft.ft_decode_geometry(H, I, 40)
    assert g["threads"] == 512
    assert g["gate_up"]["taken"] and g["down"]["taken"]
    check_tile(g["gate_up"], H, I, 2, g["threads"], g["smem_limit"])
    check_tile(g["down"], I, H, 1, g["threads"], g["smem_limit"])
    if g["stack"]:
        assert g["sync_stride"] == 2 + H // g["down"]["R"]


def test_35b_class_tiles_and_stack():
    g = ft.ft_decode_geometry(2048, 512, 40)
    assert (g["gate_up"]["R"], g["gate_up"]["parts"], g["gate_up"]["tasks"]) == (32, 8, 32)
    assert (g["down"]["R"], g["down"]["parts"], g["down"]["tasks"]) == (128, 2, 16)
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


FLOW_SHAPES = [(2048, 512, 256, 8, 1, 40), (4096, 2048, 256, 6, 0, 43), (6144, 2048, 256, 8, 0, 8),
               (256, 128, 16, 2, 0, 4), (1024, 512, 64, 4, 0, 3), (1024, 768, 64, 4, 1, 3), (256, 256, 16, 4, 1, 3)]
# shapes whose down tile (16 rows of every unit over the full intermediate
# size) and gate/up tile together outgrow a CTA's shared memory: the
# counter-synchronised persistent kernel takes their stacks
FLOW_TOO_BIG = {((4096, 2048, 256, 6, 0, 43), 2), ((6144, 2048, 256, 8, 0, 8), 1), ((6144, 2048, 256, 8, 0, 8), 2)}


@pytest.mark.parametrize("shape", FLOW_SHAPES)
@pytest.mark.parametrize("T", [1, 2])
def test_dataflow_kernel_geometry(shape, T):
    """The dataflow stack kernel takes the workload shapes at one and two
    tokens where they fit: its CTA fits the opt-in shared memory, a down tile
    has room for one 16-row tensor-core task of every unit a layer can have,
    and the gate/up tile whole tasks (8 rows of each matrix at least).  The
    rest go to the counter-synchronised kernel."""
    H, I, E, k, S, L = shape
    g = ft.ft_flow_geometry(H, I, T, k, S, E, L)
    if (shape, T) in FLOW_TOO_BIG:
        assert not g["ok"] and ft.ft_decode_geometry(H, I, L)["stack"]
        return
    assert g["ok"] and g["smem"] <= OPT_IN_SMEM
    units = min(E, T * k) + S
    assert g["rows_cap"] % 16 == 0 and g["rows_cap"] >= 16 * units
    assert g["a_rows"] >= 8 and I % g["a_rows"] == 0


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
