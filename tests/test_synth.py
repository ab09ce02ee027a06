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
