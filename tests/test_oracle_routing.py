"""Pins of the oracle's routing: fixed-order logits, top-k, weights, permutation."""
import math

import numpy as np
import pytest
import scipy.special

from oracle import routing


def test_router_logits_close_to_exact_sum():
    rng = np.random.default_rng(0)
    T, E, H = 3, 16, 512
    x = rng.standard_normal((T, H)).astype(np.float32)
    x = (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)  # bf16 values
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    got = routing.router_logits(x, wr)
    for t in range(T):
        for e in range(E):
            exact = math.fsum(float(x[t, k]) * float(wr[e, k]) for k in range(H))
            want = np.float32(exact)
            assert abs(float(got[t, e]) - float(want)) <= float(np.spacing(np.abs(want)))


def test_router_logits_order_is_the_stated_one():
    """Products placed so that only the stated order gives 0: lane 0 adds
    2^53 then 1 (absorbed by ties-to-even) then -2^53; a plain left-to-right
    sum over k would give 1 instead."""
    H = 256
    x = np.zeros((1, H))
    wr = np.zeros((1, H), np.float32)
    x[0, 0], wr[0, 0] = 2.0 ** 26, 2.0 ** 27     # product 2^53, lane 0, step 0
    x[0, 1], wr[0, 1] = 1.0, 1.0                 # product 1, lane 0, step 0
    x[0, 128], wr[0, 128] = -(2.0 ** 26), 2.0 ** 27   # -2^53, lane 0, chunk 1
    assert routing.router_logits(x, wr)[0, 0] == 0.0
    # butterfly: lane 0 = 2^53, lane 16 = 1, lane 8 = -2^53 -> (2^53 + 1) + (-2^53) = 0,
    # whereas a sequential sum over lanes 0..31 would give 1
    x2 = np.zeros((1, H))
    wr2 = np.zeros((1, H), np.float32)
    x2[0, 0], wr2[0, 0] = 2.0 ** 26, 2.0 ** 27
    x2[0, 16 * 4], wr2[0, 16 * 4] = 1.0, 1.0
    x2[0, 8 * 4], wr2[0, 8 * 4] = -(2.0 ** 26), 2.0 ** 27
    assert routing.router_logits(x2, wr2)[0, 0] == 0.0
    assert math.fsum([2.0 ** 53, -(2.0 ** 53), 1.0]) == 1.0


def brute_topk(lg, k):
    T, E = lg.shape
    out = np.empty((T, k), np.int64)
    for t in range(T):
        v = lg[t].astype(np.float64)
        key = np.where(np.isnan(v), -np.inf, v)
        nanflag = np.isnan(v).astype(np.int64)
        order = np.lexsort((np.arange(E), -key, nanflag))   # last key is primary
        out[t] = order[:k]
    return out


@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (256, 6), (7, 7)])
def test_topk_matches_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 10 + k)
    lg = rng.standard_normal((50, E)).astype(np.float32)
    lg[::3, ::5] = 1.25                 # many exact ties
    lg[1::4, 3] = -0.0
    lg[1::4, 4] = 0.0
    lg[2, :] = 0.5                      # whole row tied
    lg[5, 1] = -np.inf
    ids, bad = routing.topk(lg, k)
    assert not bad
    assert (ids == brute_topk(lg, k)).all()
    # ties resolve toward the lower id
    assert list(routing.topk(np.full((1, E), 0.5, np.float32), k)[0][0]) == list(range(k))


def test_topk_nan_flag_and_rank():
    lg = np.array([[1.0, np.nan, -np.inf, 0.5]], np.float32)
    ids, bad = routing.topk(lg, 4)
    assert bad
    assert list(ids[0]) == [0, 3, 2, 1]
    assert routing.topk(np.array([[1.0, np.inf]], np.float32), 1)[1]
    assert routing.topk(np.array([[-np.inf, -np.inf]], np.float32), 1)[1]


def test_softmax_weights():
    rng = np.random.default_rng(1)
    lg = rng.standard_normal((20, 32)).astype(np.float32) * 3
    ids, _ = routing.topk(lg, 4)
    w_raw = routing.softmax_weights(lg, ids, renorm=False)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    assert np.allclose(w_raw, np.take_along_axis(p, ids, 1), rtol=1e-14, atol=0)
    w = routing.softmax_weights(lg, ids, renorm=True)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)
    # renormalised weights equal a softmax over the chosen logits alone
    sel = np.take_along_axis(lg.astype(np.float64), ids, 1)
    assert np.allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-13)
    # k = E: renormalisation changes nothing
    idsE, _ = routing.topk(lg, 32)
    assert np.allclose(routing.softmax_weights(lg, idsE, True), routing.softmax_weights(lg, idsE, False))
    # the worked-example weights: logits (0, ln 3) -> (1/4, 3/4)
    w2 = routing.softmax_weights(np.array([[0.0, math.log(3)]], np.float32), np.array([[1, 0]]))
    assert np.allclose(w2[0], [0.75, 0.25], rtol=1e-7)


@pytest.mark.parametrize("T,E,k", [(1, 16, 2), (8, 16, 2), (33, 256, 8), (300, 64, 6)])
def test_permutation_invariants(T, E, k):
    rng = np.random.default_rng(T)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offs, perm, inv = routing.permutation(ids, E)
    flat = ids.reshape(-1)
    assert (perm == np.argsort(flat, kind="stable")).all()
    assert (perm[inv] == np.arange(T * k)).all()
    assert offs[0] == 0 and offs[E] == T * k
    assert (np.diff(offs) == np.bincount(flat, minlength=E)).all()
    for e in range(E):
        seg = perm[offs[e]:offs[e + 1]]
        assert (flat[seg] == e).all()
        assert (np.diff(seg // k) > 0).all()      # tokens ascending, each once
