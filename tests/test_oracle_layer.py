"""Pins for the oracle's expert FFN and the whole MoE step.

* a hand-built expert whose matrices are permutations turns the FFN into a
  closed form in the logistic function (checks orientation and the sign
  inside silu);
* torch's silu and matmul on the oracle's own dequantised matrices;
* a brute-force layer: every expert computed densely for every token, then
  the top-k picked with numpy and mixed -- no permute, no row bookkeeping;
* special cases: k = E (full softmax mixture), E = k = 1 (one SwiGLU FFN),
  a one-hot gate, the shared expert entering with weight 1, and a window of
  T tokens giving the same rows as T single-token steps (Strata article,
  section 2 item 3: the verify pass gives the same answer as plain decode).
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import workloads as W


def _perm_block_codes(bits, rows, cols, col_of_row, code_val):
    """codes/scales for a matrix with W[r, col_of_row[r]] = code_val - half, else 0 (d = 1)."""
    half = 1 << (bits - 1)
    q = np.full((rows, cols), half, np.int64)
    q[np.arange(rows), col_of_row] = code_val
    # pack by hand with the documented bit layout
    nb = cols // 32
    qb = q.reshape(rows, nb, 32)
    if bits == 4:
        codes = (qb[..., :16] | (qb[..., 16:] << 4)).astype(np.uint8)
    else:
        c = qb.reshape(rows, nb, 4, 8)
        codes = (c[:, :, 0] | (c[:, :, 1] << 2) | (c[:, :, 2] << 4) | (c[:, :, 3] << 6)).astype(np.uint8)
    scales = np.full((rows, nb), 0x3C00, np.uint16)       # fp16 1.0
    return codes.reshape(rows, -1), scales


def _hand_blob(bits, H, I, pg, pu, pd, cg, cu, cd):
    a = _perm_block_codes(bits, I, H, pg, cg)
    b = _perm_block_codes(bits, I, H, pu, cu)
    c = _perm_block_codes(bits, H, I, pd, cd)
    return np.concatenate([a[0].ravel(), b[0].ravel(), c[0].ravel(),
                           a[1].ravel().view(np.uint8), b[1].ravel().view(np.uint8),
                           c[1].ravel().view(np.uint8)])


@pytest.mark.parametrize("bits", [4, 2])
def test_ffn_closed_form_permutation_expert(oracle_lib, bits):
    H = I = 64
    rng = np.random.default_rng(2)
    pg, pu, pd = rng.permutation(I), rng.permutation(I), rng.permutation(H)
    half = 1 << (bits - 1)
    # Wg[i, pg[i]] = 1, Wu[i, pu[i]] = -1 (q4) / 1 (q2), Wd[h, pd[h]] = 1
    gu = -1 if bits == 4 else 1
    blob = _hand_blob(bits, H, I, pg, pu, pd, half + 1, half + gu, half + 1)
    x = np.array([(-1) ** c * (0.25 * (c % 9) + 0.1) for c in range(H)])
    y, h = oracle_lib.expert_ffn(bits, H, I, blob, x)
    for i in range(I):
        g = x[pg[i]]
        u = gu * x[pu[i]]
        assert h[i] == pytest.approx(g / (1.0 + math.exp(-g)) * u, rel=1e-15, abs=1e-300)
    for r in range(H):
        i = pd[r]
        g = x[pg[i]]
        assert y[r] == pytest.approx(g / (1.0 + math.exp(-g)) * gu * x[pu[i]], rel=1e-15, abs=1e-300)
    # the logistic function at 1 and -1: 1/(1+e^-1) and 1/(1+e)
    assert 1 / (1 + math.exp(-1.0)) == pytest.approx(0.7310585786300049, rel=1e-15)


@pytest.mark.parametrize("bits", [4, 2])
def test_ffn_against_torch_dense(oracle_lib, bits):
    rng = np.random.default_rng(7)
    H, I = 256, 128
    blob = W.random_expert_blob(rng, bits, H, I, 0.02)
    Wg, Wu, Wd = (torch.from_numpy(m) for m in oracle_lib.expert_weights(bits, H, I, blob))
    for s in range(3):
        x = rng.standard_normal(H)
        y, _ = oracle_lib.expert_ffn(bits, H, I, blob, x)
        xt = torch.from_numpy(x)
        ref = Wd @ (torch.nn.functional.silu(Wg @ xt) * (Wu @ xt))
        assert np.allclose(y, ref.numpy(), rtol=1e-11, atol=1e-14)


def _brute_layer(oracle_lib, layer, x, x_dtype, logits=None):
    """Dense brute force: all experts on all tokens, numpy top-k, mix."""
    E, k, H, I, bits = layer.E, layer.k, layer.H, layer.I, layer.bits
    xd = W.bf16_bits_to_f32(x).astype(np.float64) if x_dtype == "bf16" else x.astype(np.float64)
    T = xd.shape[0]
    if logits is None:
        wr = (W.bf16_bits_to_f32(layer.w_router) if layer.w_dtype == "bf16" else layer.w_router).astype(np.float64)
        logits = xd @ wr.T
        if layer.bias is not None:
            logits = logits + layer.bias.astype(np.float64)
    mats = [tuple(torch.from_numpy(m) for m in oracle_lib.expert_weights(bits, H, I, layer.blobs[e])) for e in range(E)]
    X = torch.from_numpy(xd)
    dense = torch.stack([(torch.nn.functional.silu(X @ g.T) * (X @ u.T)) @ d.T for (g, u, d) in mats])  # [E,T,H]
    y = np.zeros((T, H))
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t]))[:k]
        gate = scipy.special.softmax(logits[t])[order]
        gate = gate / gate.sum()
        y[t] = sum(gate[j] * dense[order[j], t].numpy() for j in range(k))
    if layer.shared is not None:
        g, u, d = (torch.from_numpy(m) for m in oracle_lib.expert_weights(bits, H, I, layer.shared))
        y += ((torch.nn.functional.silu(X @ g.T) * (X @ u.T)) @ d.T).numpy()
    return y


def test_layer_tiny_brute_force(oracle_lib):
    layer, x = W.tiny_case()
    out = oracle_lib.moe_layer(layer.bits, x, "f32", layer.blobs, k=layer.k, H=layer.H, I=layer.I,
                               E=layer.E, w_router=layer.w_router, w_dtype=layer.w_dtype)
    assert out["status"] == 0
    ref = _brute_layer(oracle_lib, layer, x, "f32")
    assert np.allclose(out["y"], ref, rtol=1e-11, atol=1e-13)


def test_layer_bf16_shared_bias_brute_force(oracle_lib):
    layer = W.make_layer(77, 2, 128, 64, 12, 3, shared=True, w_dtype="bf16",
                         bias=np.linspace(-1, 1, 12).astype(np.float32))
    x = W.make_tokens(78, 5, 128, "bf16")
    out = oracle_lib.moe_layer(2, x, "bf16", layer.blobs, k=3, H=128, I=64, E=12,
                               w_router=layer.w_router, w_dtype="bf16", bias=layer.bias,
                               shared_blob=layer.shared)
    ref = _brute_layer(oracle_lib, layer, x, "bf16")
    assert np.allclose(out["y"], ref, rtol=1e-11, atol=1e-13)


def test_layer_k_equals_E_is_dense_mixture(oracle_lib):
    layer = W.make_layer(5, 4, 128, 64, 6, 6, shared=False, w_dtype="f32")
    x = W.make_tokens(6, 3, 128, "f32")
    out = oracle_lib.moe_layer(4, x, "f32", layer.blobs, k=6, H=128, I=64, E=6,
                               w_router=layer.w_router, w_dtype="f32")
    logits = x.astype(np.float64) @ layer.w_router.astype(np.float64).T
    y = np.zeros((3, 128))
    for t in range(3):
        p = scipy.special.softmax(logits[t])
        for e in range(6):
            ye, _ = oracle_lib.expert_ffn(4, 128, 64, layer.blobs[e], x[t].astype(np.float64))
            y[t] += p[e] * ye
    assert np.allclose(out["y"], y, rtol=1e-12, atol=1e-14)


def test_layer_single_expert_is_one_ffn(oracle_lib):
    layer = W.make_layer(9, 4, 128, 64, 1, 1, shared=False, w_dtype="f32")
    x = W.make_tokens(10, 4, 128, "f32")
    out = oracle_lib.moe_layer(4, x, "f32", layer.blobs, k=1, H=128, I=64, E=1,
                               w_router=layer.w_router, w_dtype="f32")
    assert np.all(out["w"] == 1.0)
    for t in range(4):
        ye, _ = oracle_lib.expert_ffn(4, 128, 64, layer.blobs[0], x[t].astype(np.float64))
        assert np.array_equal(out["y"][t], ye)


def test_layer_one_hot_gate_and_shared(oracle_lib):
    layer = W.make_layer(12, 4, 128, 64, 8, 2, shared=True, w_dtype="f32")
    x = W.make_tokens(13, 2, 128, "f32")
    logits = np.full((2, 8), -2000.0, np.float32)
    logits[0, 5] = 0.0
    logits[1, 2] = 0.0
    out = oracle_lib.moe_layer(4, x, "f32", layer.blobs, k=2, H=128, I=64, E=8,
                               logits_in=logits, shared_blob=layer.shared)
    assert out["ids"][0, 0] == 5 and out["ids"][1, 0] == 2
    assert np.all(out["w"][:, 0] == 1.0) and np.all(out["w"][:, 1] == 0.0)
    for t, e in [(0, 5), (1, 2)]:
        ye, _ = oracle_lib.expert_ffn(4, 128, 64, layer.blobs[e], x[t].astype(np.float64))
        ys, _ = oracle_lib.expert_ffn(4, 128, 64, layer.shared, x[t].astype(np.float64))
        assert np.array_equal(out["y_shared"][t], ys)
        assert np.allclose(out["y"][t], ye + ys, rtol=1e-15, atol=0)


def test_window_equals_single_steps(oracle_lib):
    """A T-token verify window gives the same rows as T one-token steps."""
    layer = W.verify_layer(H=128, I=64, E=32, k=4)
    x = W.make_tokens(21, 9, 128, "bf16")
    kw = dict(k=4, H=128, I=64, E=32, w_router=layer.w_router, w_dtype="bf16",
              bias=layer.bias, shared_blob=layer.shared)
    win = oracle_lib.moe_layer(2, x, "bf16", layer.blobs, **kw)
    for t in range(9):
        one = oracle_lib.moe_layer(2, x[t:t + 1], "bf16", layer.blobs, **kw)
        assert np.array_equal(one["ids"][0], win["ids"][t])
        assert np.array_equal(one["y"][0], win["y"][t])


def test_combine_matches_layer(oracle_lib):
    layer, x = W.tiny_case()
    out = oracle_lib.moe_layer(layer.bits, x, "f32", layer.blobs, k=layer.k, H=layer.H, I=layer.I,
                               E=layer.E, w_router=layer.w_router, w_dtype="f32", want_yperm=True)
    y = oracle_lib.combine(out["y_perm"], out["perm_dst"], out["w"])
    assert np.array_equal(y, out["y"])
    # each y_perm row is that expert applied to that token
    for t in range(x.shape[0]):
        for j in range(layer.k):
            r = out["perm_dst"][t, j]
            ye, _ = oracle_lib.expert_ffn(4, layer.H, layer.I, layer.blobs[out["ids"][t, j]], x[t].astype(np.float64))
            assert np.array_equal(out["y_perm"][r], ye)


@pytest.mark.parametrize("bits", [4, 2])
def test_ffn_rows_is_the_single_row_ffn(oracle_lib, bits):
    """The batched row helper is a parallel map of the pinned one-token FFN:
    each of its rows equals that function's result bit for bit, whichever
    expert and token it pairs (including repeated experts and a reversed order)."""
    rng = np.random.default_rng(11 + bits)
    H, I = 128, 64
    blobs = [W.random_expert_blob(rng, bits, H, I, 0.02) for _ in range(3)]
    xs = rng.standard_normal((7, H))
    pick = [0, 2, 1, 1, 0, 2, 0]
    got = oracle_lib.expert_ffn_rows(bits, H, I, [blobs[e] for e in pick], xs)
    for i, e in enumerate(pick):
        y, _ = oracle_lib.expert_ffn(bits, H, I, blobs[e], xs[i])
        assert np.array_equal(got[i], y)
    rev = oracle_lib.expert_ffn_rows(bits, H, I, [blobs[e] for e in pick[::-1]], xs[::-1])
    assert np.array_equal(rev[::-1], got)
