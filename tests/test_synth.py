"""The seeded input module: determinism, region boundaries, distributions."""
import numpy as np

import synth


def test_blob_deterministic_and_keyed():
    a = synth.expert_blob(7, 3, 5, 256, 128)
    b = synth.expert_blob(7, 3, 5, 256, 128)
    c = synth.expert_blob(7, 3, 6, 256, 128)
    assert (a == b).all() and not (a == c).all()
    r = synth.blob_regions(256, 128)
    assert (a[r["used"]:] == 0).all()


def test_code_and_scale_histograms():
    r = synth.blob_regions(2048, 512)
    blob = synth.expert_blob(11, 0, 0, 2048, 512)
    codes = blob[:r["codes_end"]]
    nib = np.concatenate([codes & 15, codes >> 4])
    mag = np.bincount(nib & 7, minlength=8) / nib.size
    assert np.allclose(mag, np.array(synth.MAG_COUNTS) / 128, atol=0.005)
    assert abs((nib >> 3).mean() - 0.5) < 0.005
    sc = blob[r["codes_end"]:r["used"]]
    assert set(np.unique(sc)) == {119, 120, 121}
    assert abs((sc == 120).mean() - 0.5) < 0.01


def test_trace_overlap_and_distinct():
    tr = synth.zipf_trace(1, 0, 200, 256, 8, 1.1, 0.6)
    assert all(len(set(row)) == 8 for row in tr)
    keep = np.mean([len(set(tr[t]) & set(tr[t - 1])) / 8 for t in range(1, 200)])
    assert 0.55 < keep < 0.75     # rho plus chance re-draws of popular experts
    lg = synth.logits_for_sets(1, 0, tr[:10], 256)
    top = np.argsort(-lg, axis=1, kind="stable")[:, :8]
    assert (top == tr[:10]).all()


def test_bf16_blob_deterministic_keyed_and_shaped():
    a = synth.expert_blob_bf16(7, 3, 5, 2048, 512)
    assert (a == synth.expert_blob_bf16(7, 3, 5, 2048, 512)).all()
    assert not (a == synth.expert_blob_bf16(7, 3, 6, 2048, 512)).all()
    bits = a[:synth.bf16_blob_regions(2048, 512)["used"]].view("<u2")
    binade = ((bits >> 7) & 0xFF).astype(np.int64) - synth.BF16_EXP_LOW
    assert binade.min() >= 0 and binade.max() < len(synth.BF16_BINADE_COUNTS)
    assert np.allclose(np.bincount(binade, minlength=11) / bits.size, np.array(synth.BF16_BINADE_COUNTS) / 256,
                       atol=0.002)
    assert abs((bits >> 15).mean() - 0.5) < 0.005
    v = (bits.astype(np.uint32) << 16).view(np.float32)
    assert 0.018 < v.std() < 0.026          # about N(0, 0.02)


def test_nvfp4_blob_regions_and_bytes():
    r = synth.nvfp4_blob_regions(2048, 512)
    a = synth.expert_blob_nvfp4(7, 3, 5, 2048, 512)
    assert (a == synth.expert_blob_nvfp4(7, 3, 5, 2048, 512)).all()
    # the code region is the MXFP4 generator's, byte for byte
    assert (a[:r["codes_end"]] == synth.code_bytes(7, 3, 5, r["codes_end"])).all()
    sc = a[r["codes_end"]:r["tensor_scales"]]
    assert set(np.unique(sc)) == set(synth.NVFP4_SCALE_BYTES)
    ts = a[r["tensor_scales"]:r["tensor_scales"] + 12].view("<f4")
    assert list(ts) == list(np.float32(synth.NVFP4_TENSOR_SCALES))
    assert (a[r["tensor_scales"] + 12:] == 0).all()


def test_wide_nvfp4_blob_covers_every_e4m3_byte():
    """The wide NVFP4 blob: each wide matrix's scale bytes take every value
    0x00 .. 0x7e and nothing above (no NaN byte 0x7f); all 16 codes occur;
    the matrix scales are the ones asked for; the draws are deterministic."""
    import numpy as np
    import synth
    H, I = 256, 128
    b = synth.expert_blob_nvfp4_wide(9, 1, 2, H, I, tensor_scales=(0.5, 0.25, 0.125))
    r = synth.nvfp4_blob_regions(H, I)
    for a, z in ((r["wg_sf"], r["wu_sf"]), (r["wu_sf"], r["wd_sf"]), (r["wd_sf"], r["tensor_scales"])):
        assert set(np.unique(b[a:z])) == set(range(0x7F))
    codes = b[:r["codes_end"]]
    assert set(np.unique(np.concatenate([codes & 15, codes >> 4]))) == set(range(16))
    assert list(b[r["tensor_scales"]:r["tensor_scales"] + 12].view("<f4")) == [0.5, 0.25, 0.125]
    assert (b == synth.expert_blob_nvfp4_wide(9, 1, 2, H, I, tensor_scales=(0.5, 0.25, 0.125))).all()


def test_wide_bf16_blob_covers_every_finite_exponent():
    """The wide BF16 blob: every biased exponent 0 .. 254 (zeros and
    subnormals included) in both signs, no infinity or NaN; deterministic."""
    import numpy as np
    import synth
    H, I = 256, 128
    b = synth.expert_blob_bf16_wide(9, 1, 2, H, I)
    v = b[:6 * H * I].view("<u2")
    e = (v >> 7) & 0xFF
    assert set(np.unique(e)) == set(range(255))
    assert 0.45 < ((v >> 15) & 1).mean() < 0.55
    assert (b == synth.expert_blob_bf16_wide(9, 1, 2, H, I)).all()
