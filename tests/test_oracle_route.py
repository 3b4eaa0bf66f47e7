"""Pins for the oracle's router logits, top-k selection, gates and permute.

References used here are independent of the oracle: numpy/BLAS matmul,
numpy lexsort and Python's sorted(), scipy's softmax, brute-force counting.
"""
import numpy as np
import pytest
import scipy.special

import workloads as W


def _brute_topk(l, k):
    """Sort by (value desc, id asc), NaN last, with numpy's lexsort."""
    T, E = l.shape
    ids = np.empty((T, k), np.int64)
    for t in range(T):
        v = l[t]
        key_nan = np.isnan(v)
        vv = np.where(key_nan, 0.0, v)
        order = np.lexsort((np.arange(E), -vv, key_nan))
        ids[t] = order[:k]
    return ids


def test_router_logits_against_blas(oracle_lib):
    rng = np.random.default_rng(1)
    T, H, E = 5, 256, 24
    x = W.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wr = W.f32_to_bf16_bits((rng.standard_normal((E, H)) * 0.1).astype(np.float32))
    bias = rng.standard_normal(E).astype(np.float32)
    got = oracle_lib.router_logits(x, "bf16", wr, "bf16", bias)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    wf = W.bf16_bits_to_f32(wr).astype(np.float64)
    ref = xf @ wf.T + bias.astype(np.float64)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)
    # f32 inputs
    xf32 = rng.standard_normal((T, H)).astype(np.float32)
    wf32 = rng.standard_normal((E, H)).astype(np.float32)
    got = oracle_lib.router_logits(xf32, "f32", wf32, "f32")
    assert np.allclose(got, xf32.astype(np.float64) @ wf32.astype(np.float64).T, rtol=1e-13, atol=1e-12)


@pytest.mark.parametrize("E,k", [(16, 2), (512, 10), (37, 37), (24576, 10)])
def test_topk_brute_force(oracle_lib, E, k):
    rng = np.random.default_rng(E + k)
    T = 6 if E < 1000 else 2
    l = rng.standard_normal((T, E))
    ids, w, st = oracle_lib.topk(l, k)
    assert st == 0
    assert np.array_equal(ids, _brute_topk(l, k))
    # invariants: k distinct ids in range, descending logits, gates sum to 1 and do not increase
    for t in range(T):
        assert len(set(ids[t])) == k and ids[t].min() >= 0 and ids[t].max() < E
        sel = l[t, ids[t]]
        assert np.all(np.diff(sel) <= 0)
        assert abs(w[t].sum() - 1.0) <= 1e-12
        assert np.all(np.diff(w[t]) <= 1e-15)
        # gate = full softmax renormalised over the selected experts
        full = scipy.special.softmax(l[t])
        assert np.allclose(w[t], full[ids[t]] / full[ids[t]].sum(), rtol=1e-12)


def test_topk_ties_go_to_lower_id(oracle_lib):
    l = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.0],
                  [5.0, 5.0, 5.0, 5.0, 5.0, 5.0],
                  [0.0, -0.0, 0.0, -1.0, -0.0, 2.0]])
    ids, w, st = oracle_lib.topk(l, 3)
    assert st == 0
    assert ids[0].tolist() == [1, 2, 4]
    assert ids[1].tolist() == [0, 1, 2]
    assert ids[2].tolist() == [5, 0, 1]        # -0.0 == +0.0: ties by id
    assert np.allclose(w[1], 1 / 3, rtol=0, atol=1e-15)
    # integer-valued logits given as float32 take the same path
    ids32, _, _ = oracle_lib.topk(l.astype(np.float32), 3)
    assert np.array_equal(ids32, ids)


def test_topk_nonfinite(oracle_lib):
    nan, inf = np.nan, np.inf
    l = np.array([[nan, 1.0, -inf, 0.5, nan]])
    ids, w, st = oracle_lib.topk(l, 3)
    assert st == 0
    assert ids[0].tolist() == [1, 3, 2]          # NaN ranks below -inf
    assert w[0, 2] == 0.0                         # -inf gets gate 0
    ids, w, st = oracle_lib.topk(l, 4)
    assert st == -1 and ids[0].tolist() == [1, 3, 2, 0]   # a NaN had to be selected
    ids, w, st = oracle_lib.topk(np.array([[1.0, inf, 0.0]]), 2)
    assert st == -1                               # +inf selected


def test_topk_k_equals_E_is_full_softmax(oracle_lib):
    rng = np.random.default_rng(9)
    l = rng.standard_normal((3, 12)) * 4
    ids, w, st = oracle_lib.topk(l, 12)
    for t in range(3):
        full = scipy.special.softmax(l[t])
        assert np.allclose(w[t], full[ids[t]], rtol=1e-13, atol=1e-16)


def _brute_permute(ids, E):
    T, k = ids.shape
    pairs = sorted(((int(ids[t, j]), t, j) for t in range(T) for j in range(k)))
    perm_src = np.array([t for (_, t, _) in pairs], np.int32)
    perm_dst = np.empty((T, k), np.int32)
    for r, (_, t, j) in enumerate(pairs):
        perm_dst[t, j] = r
    counts = np.bincount(ids.ravel(), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    active = np.flatnonzero(counts)
    return offsets, perm_src, perm_dst, active


@pytest.mark.parametrize("T,k,E", [(8, 2, 16), (1, 10, 512), (37, 10, 512), (300, 3, 7), (5, 10, 24576)])
def test_permute_brute_force(oracle_lib, T, k, E):
    rng = np.random.default_rng(T * 100 + k)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    p = oracle_lib.permute(ids, E)
    offsets, perm_src, perm_dst, active = _brute_permute(ids, E)
    assert np.array_equal(p["offsets"], offsets)
    assert np.array_equal(p["perm_src"], perm_src)
    assert np.array_equal(p["perm_dst"], perm_dst)
    assert p["active"][0] == len(active) and np.array_equal(p["active"][1:], active)
    # invariants: bijection, rows of an expert contiguous and ascending in token
    assert sorted(p["perm_dst"].ravel().tolist()) == list(range(T * k))
    for t in range(T):
        for j in range(k):
            r = p["perm_dst"][t, j]
            assert p["perm_src"][r] == t
            e = ids[t, j]
            assert p["offsets"][e] <= r < p["offsets"][e + 1]
    for e in active:
        seg = p["perm_src"][p["offsets"][e]:p["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_permute_rejects_bad_id(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.permute(np.array([[0, 16]], np.int32), 16)
    with pytest.raises(ValueError):
        oracle_lib.permute(np.array([[-1, 3]], np.int32), 16)
