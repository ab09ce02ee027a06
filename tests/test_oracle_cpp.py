"""Pins of the C++ oracle (oracle/ft_oracle.cpp through oracle/cpp.py): the
same closed forms, tables, worked example, brute force and invariants that pin
the numpy oracle, plus a cross-check of every function against the numpy
oracle on seeded inputs (bit-exact wherever both compute exactly, else within
fp64 rounding)."""
import math

import numpy as np
import pytest

import synth
from oracle import cpp, formats, fp4, layer, lru, routing

OCP_E2M1_POSITIVE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_and_ue8m0_tables_match_the_spec():
    t = cpp.e2m1_table()
    for c in range(8):
        assert t[c] == OCP_E2M1_POSITIVE[c] and t[c + 8] == -OCP_E2M1_POSITIVE[c]
    assert math.copysign(1.0, t[8]) < 0
    u = cpp.ue8m0_table()
    for e in range(255):
        assert u[e] == 2.0 ** (e - 127)
    assert math.isnan(u[255])


def test_e4m3_table_closed_form():
    t = cpp.e4m3_table()
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            assert math.isnan(t[b])
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        assert t[b] == (-mag if s else mag)
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9


def test_scale_index_hand_values():
    cases = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (64, 0): 8, (96, 0): 12,
             (0, 1): 1, (0, 3): 3, (0, 4): 512, (33, 5): 512 + 16 + 4 + 1,
             (127, 7): 512 + 31 * 16 + 3 * 4 + 3, (128, 0): 1024, (130, 5): 1536 + 32 + 1}
    for (r, kb), want in cases.items():
        assert cpp.scale_index(r, kb, 8) == want


@pytest.mark.parametrize("H,I,stride", [(256, 128, 52224), (2048, 512, 1671168), (4096, 2048, 13369344),
                                        (6144, 2048, 20054016)])
def test_layout_sizes(H, I, stride):
    off = cpp.layout(H, I)
    assert off["stride"] == off["used"] == stride == 3 * H * I * 17 // 32
    r = synth.blob_regions(H, I)
    for k in ("wg", "wu", "wd", "wg_sf", "wu_sf", "wd_sf", "stride"):
        assert r[k] == off[k]
    nv = cpp.layout(H, I, "nvfp4")
    for k, v in formats.nvfp4_layout(H, I).items():
        assert nv[k] == v


def test_dequant_exhaustive_codes_times_scales():
    """Every (code, scale byte) pair placed by the pinned index, against the
    closed form sign * magnitude * 2^(e - 127)."""
    H, I = 512, 256
    off = cpp.layout(H, I)
    blob = np.zeros(off["stride"], np.uint8)
    codes = np.zeros((I, H), np.uint8)
    scales = np.zeros((I, H // 32), np.int64)
    cell = 0
    for r in range(I):
        for b in range(H // 32):
            scales[r, b] = cell % 255
            codes[r, 32 * b:32 * b + 32] = (np.arange(32) + cell) % 16
            cell += 1
    blob[off["wg"]:off["wg"] + I * H // 2] = (codes[:, 0::2] | (codes[:, 1::2] << 4)).reshape(-1)
    for r in range(I):
        for b in range(H // 32):
            blob[off["wg_sf"] + cpp.scale_index(r, b, H // 32)] = scales[r, b]
    got = cpp.dequant_matrix(blob, "wg", H, I)
    seen = set()
    for r in range(I):
        for k in range(0, H, 3):
            c, e = int(codes[r, k]), int(scales[r, k // 32])
            want = (-1.0 if c & 8 else 1.0) * OCP_E2M1_POSITIVE[c & 7] * 2.0 ** (e - 127)
            assert got[r, k] == want and math.copysign(1.0, got[r, k]) == math.copysign(1.0, want)
            seen.add((c, e))
    assert len(seen) == 16 * 255


@pytest.mark.parametrize("weights,gen", [("mxfp4", synth.expert_blob), ("nvfp4", synth.expert_blob_nvfp4),
                                         ("bf16", synth.expert_blob_bf16)])
def test_weight_matrices_equal_the_numpy_oracle(weights, gen):
    H, I = 256, 128
    blob = gen(77, 1, 3, H, I)
    for which in ("wg", "wu", "wd"):
        a = cpp.weight_matrix(blob, which, H, I, weights)
        b = formats.weight_matrix(blob, which, H, I, weights)
        assert (a.view(np.uint64) == b.view(np.uint64)).all(), which


def test_quantiser_ties_saturation_sign_and_idempotence():
    # grid midpoints tie to the even code; values above 6 saturate; a negative
    # value that rounds to zero keeps its sign (code 8)
    blk = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4) * 0.5
    codes, sc = cpp.quantize_rows(blk[None, :])
    assert sc[0, 0] == 127 - 1 + 0           # amax 3.0 -> floor(log2 3) - 2 = -1
    vals = cpp.e2m1_table()[codes[0, :8]] * 2.0 ** -1
    assert list(vals) == [0.0, 0.5, 0.5, 1.0, 1.0, 2.0, 2.0, 3.0]
    neg = np.full((1, 32), -0.01)
    neg[0, 0] = 4.0
    c2, _ = cpp.quantize_rows(neg)
    assert (c2[0, 1:] == 8).all()
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, 256)) * np.exp(rng.uniform(-30, 30, (16, 1)))
    c3, s3 = cpp.quantize_rows(x)
    deq = cpp.e2m1_table()[c3] * np.repeat(cpp.ue8m0_table()[s3], 32, axis=1)
    c4, s4 = cpp.quantize_rows(deq)
    assert (c4 == c3).all() and (s4 == s3).all()


def test_quantiser_equals_the_numpy_oracle():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 512)) * np.exp(rng.uniform(-60, 60, (64, 1)))
    x[0, :32] = 0.0
    x[1, :32] = (np.arange(32) - 16) * 1e-40
    a = cpp.quantize_rows(x)
    b = fp4.quantize_rows(x)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


def test_nvfp4_quantiser_equals_the_numpy_oracle():
    """The two-level NVFP4 activation quantiser, bit for bit: codes, E4M3
    scale bytes and the per-tensor scale, on rows spanning 10^+-7, zero,
    negative-zero and underflowing blocks, the hand-worked block of the numpy
    oracle's pin, a given scale, and a tensor below 2^-100."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((48, 256)) * np.exp(rng.uniform(-16, 16, (48, 1)))).astype(np.float32)
    x[0, :16] = 0.0
    x[0, 16:32] = -0.0
    x[1, :16] *= np.float32(1e-12)
    worked = np.zeros((1, 64), np.float32)
    worked[0, 0:3] = [2688.0, 224.0, -672.0]
    worked[0, 16:25] = [12.0, 3.0, -1.5, 5.0, 7.0, 0.4, -0.6, -0.0, 1.0]
    for v, s in ((x, None), (worked, None), (x, np.float32(0.125)), (np.full((2, 32), 1e-31, np.float32), None)):
        a = cpp.nvfp4_quantize_rows(v, s)
        b = formats.nvfp4_quantize_rows(v, s)
        assert (a[0] == b[0]).all() and (a[1] == b[1]).all() and a[2] == b[2]


def test_nvfp4_layer_equals_the_numpy_oracle():
    H, I, E, k, T, seed = 256, 128, 16, 4, 12, 1102
    blobs = {e: synth.expert_blob_nvfp4(seed, 0, e, H, I) for e in range(E + 1)}
    xb = synth.activations_bf16(seed, 0, T, H)
    wr = synth.router_weights(seed, 0, E, H)
    kw = dict(router_w=wr, shared_blob=blobs[E], weights="nvfp4", nvfp4=True)
    a = cpp.moe_layer(xb, blobs.__getitem__, H, I, E, k, threads=4, **kw)
    b = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, **kw)
    assert (a["ids"] == b["ids"]).all()
    assert np.allclose(a["out_f64"], b["out_f64"], rtol=1e-12, atol=1e-15)


def test_round_bf16_equals_the_numpy_oracle():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * np.exp(rng.uniform(-90, 90, 20000)),
                        [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** 128, -(2.0 ** 127) * 1.999,
                         1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -9, np.nan, np.inf]])
    assert (cpp.round_bf16(v) == fp4.round_bf16(v)).all()


@pytest.mark.parametrize("T,H,E", [(1, 256, 16), (5, 2048, 256), (3, 4096, 64)])
def test_router_logits_bit_exact_with_the_numpy_oracle(T, H, E):
    xb = synth.activations_bf16(11, T, T, H)
    wr = synth.router_weights(11, T, E, H)
    a = cpp.router_logits(xb, wr)
    b = routing.router_logits(fp4.bf16_to_f64(xb), wr)
    assert (a.view(np.uint32) == b.view(np.uint32)).all()


def test_topk_against_brute_force_with_ties_nan_and_signed_zero():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((200, 64)).astype(np.float32)
    lg[::3, ::7] = 0.75
    lg[1::5, 2] = -0.0
    lg[1::5, 3] = 0.0
    lg[::11, 5] = -np.inf
    ids, bad = cpp.topk(lg, 8)
    assert not bad
    for t in range(200):
        order = sorted(range(64), key=lambda e: (-float(lg[t, e]), e))
        assert list(ids[t]) == order[:8]
    lg[7, 9] = np.nan
    ids, bad = cpp.topk(lg, 64)
    assert bad and ids[7, -1] == 9
    w_ids, w_bad = routing.topk(lg, 64)
    assert (ids == w_ids).all() and w_bad


@pytest.mark.parametrize("renorm", [True, False])
def test_softmax_weights_closed_form(renorm):
    lg = np.array([[0.0, math.log(3.0), -1.0, 2.0]], np.float32)
    ids = np.array([[3, 1]], np.int32)
    w = cpp.softmax_weights(lg, ids, renorm)
    p = np.exp(lg[0].astype(np.float64))
    p /= p.sum()
    want = p[[3, 1]] / (p[3] + p[1]) if renorm else p[[3, 1]]
    assert np.allclose(w[0], want, rtol=1e-15, atol=0)
    rng = np.random.default_rng(5)
    lg2 = rng.standard_normal((50, 256)).astype(np.float32)
    ids2, _ = cpp.topk(lg2, 6)
    assert np.allclose(cpp.softmax_weights(lg2, ids2, renorm), routing.softmax_weights(lg2, ids2, renorm),
                       rtol=1e-14, atol=1e-300)


def test_permutation_stable_sort_and_numpy():
    rng = np.random.default_rng(6)
    ids = np.stack([rng.choice(32, 4, replace=False) for _ in range(40)]).astype(np.int32)
    offs, perm, inv = cpp.permutation(ids, 32)
    flat = ids.reshape(-1)
    assert (perm[inv] == np.arange(flat.size)).all() and offs[-1] == flat.size
    assert (np.diff(flat[perm]) >= 0).all()
    for e in range(32):
        seg = perm[offs[e]:offs[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()
    for a, b in zip((offs, perm, inv), routing.permutation(ids, 32)):
        assert (a == b).all()


def _worked_blob(H, I, g, u, d):
    off = cpp.layout(H, I)
    b = np.zeros(off["stride"], np.uint8)
    for which, rows, K, (code, col, sb) in (("wg", I, H, g), ("wu", I, H, u), ("wd", H, I, d)):
        c = np.zeros((rows, K), np.uint8)
        c[:, col] = code
        b[off[which]:off[which] + rows * K // 2] = (c[:, 0::2] | (c[:, 1::2] << 4)).reshape(-1)
        for r in range(rows):
            for kb in range(K // 32):
                b[off[which + "_sf"] + cpp.scale_index(r, kb, K // 32)] = sb
    return b


def test_worked_two_expert_example():
    """H = I = 32, experts built so that the output has a closed form (the
    hand computation is written out in the numpy oracle's layer pins):
    decode 0.5403734107238539 (bf16 0.5390625); MXFP4 mode 0.46875 exactly."""
    H = I = 32
    blobs = [_worked_blob(H, I, (2, 0, 127), (4, 0, 127), (1, 0, 127)),
             _worked_blob(H, I, (4, 1, 127), (2, 1, 127), (6, 0, 126))]
    x = np.zeros((1, H))
    x[0, 0], x[0, 1] = 1.0, -1.0
    xb = cpp.round_bf16(x)
    lg = np.array([[0.0, math.log(3.0)]], np.float32)
    w1 = math.exp(float(lg[0, 1])) / (1 + math.exp(float(lg[0, 1])))
    y0 = 0.5 * 2.0 / (1.0 + math.exp(-1.0))
    y1 = 2.0 * 2.0 / (1.0 + math.exp(2.0))
    r = cpp.moe_layer(xb, lambda e: blobs[e], H, I, 2, 2, logits=lg)
    assert list(r["ids"][0]) == [1, 0]
    assert np.allclose(r["out_f64"], (1 - w1) * y0 + w1 * y1, rtol=1e-14, atol=0)
    assert (fp4.bf16_to_f64(r["out_bits"]) == 0.5390625).all()
    r = cpp.moe_layer(xb, lambda e: blobs[e], H, I, 2, 2, logits=lg, mxfp4=True)
    assert np.allclose(r["out_f64"], (1 - w1) * 0.75 + w1 * 0.375, rtol=1e-14, atol=0)
    assert (fp4.bf16_to_f64(r["out_bits"]) == 0.46875).all()


@pytest.mark.parametrize("mxfp4", [False, True])
@pytest.mark.parametrize("weights", ["mxfp4", "nvfp4", "bf16"])
def test_layer_equals_the_numpy_oracle(mxfp4, weights):
    if mxfp4 and weights != "mxfp4":
        pytest.skip("MXFP4 activations are defined for MXFP4 weights only")
    H, I, E, k, T, seed = 256, 128, 16, 4, 6, 1101
    gen = {"mxfp4": synth.expert_blob, "nvfp4": synth.expert_blob_nvfp4, "bf16": synth.expert_blob_bf16}[weights]
    blobs = {e: gen(seed, 0, e, H, I) for e in range(E + 1)}
    xb = synth.activations_bf16(seed, 0, T, H)
    wr = synth.router_weights(seed, 0, E, H)
    a = cpp.moe_layer(xb, blobs.__getitem__, H, I, E, k, router_w=wr, mxfp4=mxfp4, shared_blob=blobs[E],
                      weights=weights)
    b = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, router_w=wr, mxfp4=mxfp4, shared_blob=blobs[E],
                        weights=weights)
    assert (a["ids"] == b["ids"]).all()
    assert np.allclose(a["w"], b["w"], rtol=1e-14, atol=0)
    assert np.allclose(a["out_f64"], b["out_f64"], rtol=1e-12, atol=1e-15)
    # the two sum the expert dot products in different orders: bf16 bits agree
    # except where the fp64 result sits within that difference of a rounding boundary
    diff = a["out_bits"] != b["out_bits"]
    assert diff.mean() < 1e-3


def test_layer_parallel_equals_serial_and_tiny_fixture():
    """OpenMP over experts changes no bit (each expert is computed alone, the
    combine order is fixed), and the 35B-class shape matches numpy."""
    H, I, E, k, T, seed = 2048, 512, 64, 8, 2, 1102
    blobs = {e: synth.expert_blob(seed, 0, e, H, I) for e in range(E + 1)}
    xb = synth.activations_bf16(seed, 0, T, H)
    sets = np.stack([synth.zipf_trace(seed, 0, 3, E, k, 1.1, 0.6, stream=t)[-1] for t in range(T)])
    lg = synth.logits_for_sets(seed, 0, sets, E)
    a = cpp.moe_layer(xb, blobs.__getitem__, H, I, E, k, logits=lg, shared_blob=blobs[E], threads=1)
    b = cpp.moe_layer(xb, blobs.__getitem__, H, I, E, k, logits=lg, shared_blob=blobs[E], threads=4)
    assert (a["out_f64"].view(np.uint64) == b["out_f64"].view(np.uint64)).all()
    c = layer.moe_layer(xb, blobs.__getitem__, H, I, E, k, logits=lg, shared_blob=blobs[E])
    assert np.allclose(a["out_f64"], c["out_f64"], rtol=1e-12, atol=1e-15)


def test_lru_equals_the_numpy_oracle_on_random_traces_with_resizes():
    rng = np.random.default_rng(7)
    a, b = cpp.LRUCache(12), lru.LRUCache(12)
    for step in range(400):
        if step == 150:
            assert a.resize(5) == b.resize(5)
        if step == 260:
            assert a.resize(12) == b.resize(12)
        if step % 37 == 5:
            layer_ = int(rng.integers(4))
            e = int(rng.integers(16))
            assert a.lookup(layer_, e) == b.lookup(layer_, e)
            continue
        layer_ = step % 4
        experts = rng.choice(16, int(rng.integers(1, 5)), replace=True)
        assert a.step(layer_, experts) == b.step(layer_, experts), step


def test_lru_hit_rate_one_when_everything_fits():
    c = cpp.LRUCache(64)
    rng = np.random.default_rng(8)
    keys = [(int(rng.integers(4)), rng.choice(16, 3, replace=False)) for _ in range(50)]
    for layer_, e in keys:
        c.step(layer_, e)
    for layer_, e in keys:
        assert all(ev[0] == lru.HIT for ev in c.step(layer_, e))
    with pytest.raises(RuntimeError):
        cpp.LRUCache(2).step(0, [1, 2, 3])


@pytest.mark.parametrize("per_layer", [0, 1, 2])
def test_prefetching_lru_equals_the_numpy_oracle(per_layer):
    rng = np.random.default_rng(12 + per_layer)
    a = cpp.PrefetchingLRUCache(10, 4, 16, per_layer)
    b = lru.PrefetchingLRUCache(10, 4, 16, per_layer)
    for step in range(400):
        if step == 150:
            assert a.resize(5) == b.resize(5)
        if step == 260:
            assert a.resize(10) == b.resize(10)
        experts = rng.choice(16, int(rng.integers(1, 4)), replace=False)
        assert a.step(step % 4, experts) == b.step(step % 4, experts), step
    assert (a.prefetches, a.prefetch_hits) == (b.prefetches, b.prefetch_hits)


def test_nvfp4_quantiser_equals_the_numpy_oracle_on_generated_tensors():
    """The C++ and numpy NVFP4 quantisers agree bit for bit (codes, scale
    bytes, per-tensor scale) on generated tensors mixing every magnitude of
    fp32, zeros and signed zeros."""
    from hypothesis import given, settings, strategies as st

    vals = st.one_of(st.floats(width=32, allow_nan=False, allow_infinity=False, min_value=-2.0 ** 99,
                               max_value=2.0 ** 99),
                     st.sampled_from([0.0, -0.0, 1e-40, -1e-40, 2688.0, 6.0, 0.25, 1e-31]))

    @settings(max_examples=200, deadline=None, derandomize=True)
    @given(st.lists(vals, min_size=64, max_size=64))
    def check(row):
        x = np.asarray(row, np.float32).reshape(2, 32)
        a = cpp.nvfp4_quantize_rows(x)
        b = formats.nvfp4_quantize_rows(x)
        assert (a[0] == b[0]).all() and (a[1] == b[1]).all() and a[2] == b[2]
    check()


def test_mxfp4_quantiser_equals_the_numpy_oracle_on_generated_rows():
    """The C++ and numpy MXFP4 quantisers agree (codes and UE8M0 bytes) on
    generated rows mixing every fp64 magnitude from subnormal to 1e300, zeros,
    signed zeros and the e2m1 grid's midpoints."""
    from hypothesis import given, settings, strategies as st

    vals = st.one_of(st.floats(allow_nan=False, allow_infinity=False, min_value=-1e300, max_value=1e300),
                     st.sampled_from([0.0, -0.0, 5e-324, 0.25, 0.75, 2.5, 5.0, 6.0, -3.5]))

    @settings(max_examples=200, deadline=None, derandomize=True)
    @given(st.lists(vals, min_size=64, max_size=64))
    def check(row):
        x = np.asarray(row, np.float64).reshape(2, 32)
        a = cpp.quantize_rows(x)
        b = fp4.quantize_rows(x)
        assert (a[0] == b[0]).all() and (a[1] == b[1]).all()
    check()
