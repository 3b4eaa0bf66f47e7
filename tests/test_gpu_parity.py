"""GPU parity: every kernel of the step against the fp64 oracle on the same
seeded inputs.  Integer results (expert ids, permutation, cache events) must
be bit-exact; floating outputs within 2e-3 x RMS of the oracle (the bar the
task sets, with fp32 accumulation).  All calls go through the C ABI."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import TOL, decisive_tokens, dev_x, logit_bound, rel_err, run_gpu, xd

pytestmark = pytest.mark.gpu

# The CUDA-core path computes sum_i (q_i - half) x_i as 128 * sum_i f_i x_i -
# (128 + half) * sum_i x_i with f_i = 1 + q_i/128 (a float built from the code
# bits).  The subtraction cancels the leading bits, so each 32-weight block
# carries an absolute error of about (128 + half) * 2^-24 * sqrt(32) * |x|;
# relative to RMS(y) that measures 1e-5 (4-bit) to 2e-4 (2-bit), ten times
# below the acceptance bar.  GEMV_TOL bounds it.
GEMV_TOL = 5e-4

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402


def _t(a, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype))).cuda()


def _layer_gpu(layer):
    return M.MoELayer(layer.bits, layer.H, layer.I, layer.E, layer.k, layer.blobs, layer.shared,
                      layer.w_router, layer.w_dtype, layer.bias)


# ------------------------------------------------------------------ top-k
def _logits_case(seed, T, E, kind):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        return rng.standard_normal((T, E)).astype(np.float32)
    if kind == "ints":          # many exact ties
        return rng.integers(-3, 4, size=(T, E)).astype(np.float32)
    if kind == "special":
        l = rng.standard_normal((T, E)).astype(np.float32)
        l[:, ::7] = np.nan
        l[:, 1::11] = -np.inf
        l[:, 2::13] = 0.0
        l[:, 3::13] = -0.0
        return l
    raise ValueError(kind)


@pytest.mark.parametrize("E,k", [(16, 2), (64, 10), (512, 10), (1000, 32), (24576, 10), (3000, 1)])
@pytest.mark.parametrize("kind", ["gauss", "ints", "special"])
def test_topk_bit_exact(E, k, kind):
    T = 33 if E <= 1024 else 5
    l = _logits_case(E * 7 + k, T, E, kind)
    ids_ref, w_ref, st = oracle.topk(l, k)
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    w = torch.empty(T * k, dtype=torch.float32, device="cuda")
    wsb = M.moe_route_ws_size(T, E, k)                 # E > 1024: the chunked top-k's candidates
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    M.moe_route_topk(None, 0, None, 0, _t(l), None, T, 0, E, k, ids, w, None, ws, wsb)
    err = M.moe_device_error(clear=True)
    assert np.array_equal(ids.cpu().numpy().reshape(T, k), ids_ref)
    if st == 0:
        assert err == 0
        assert np.allclose(w.cpu().numpy().reshape(T, k), w_ref, rtol=4e-6, atol=1e-7)
    else:
        assert err & M.DEVERR_NONFINITE


def test_topk_nan_selected_sets_error():
    l = np.full((2, 40), np.nan, np.float32)
    l[0, 3] = 1.0
    ids = torch.empty(8, dtype=torch.int32, device="cuda")
    w = torch.empty(8, dtype=torch.float32, device="cuda")
    M.moe_route_topk(None, 0, None, 0, _t(l), None, 2, 0, 40, 4, ids, w)
    assert M.moe_device_error(clear=True) & M.DEVERR_NONFINITE
    assert ids.cpu().numpy()[:4].tolist() == [3, 0, 1, 2]
    assert np.all(np.isnan(w.cpu().numpy()))


# ----------------------------------------------------------------- logits
@pytest.mark.parametrize("dt,T,E", [("bf16", 21, 48), ("f32", 21, 48), ("bf16", 300, 200), ("bf16", 64, 128)])
def test_router_logits_within_bound(dt, T, E):
    """bf16 chunks of 64+ tokens take the tensor-core router (ragged token and
    expert tiles here); the rest the CUDA-core one."""
    layer = W.make_layer(31, 4, 256, 128, E, 4, shared=False, w_dtype=dt, sigma_r=0.1,
                         bias=np.linspace(-0.5, 0.5, E).astype(np.float32))
    x = W.make_tokens(32, T, 256, dt)
    ref = oracle.router_logits(x, dt, layer.w_router, dt, layer.bias)
    g = _layer_gpu(layer)
    out = run_gpu(g, x, dt)
    eps = logit_bound(layer, x, dt)
    assert np.all(np.abs(out["logits"] - ref) <= eps)


@pytest.mark.parametrize("T", [40, 100])
def test_router_ties_from_duplicate_rows(T):
    """Duplicated router rows give bit-identical logits, so the lower id must win."""
    layer = W.make_layer(41, 4, 256, 128, 16, 3, shared=False, w_dtype="bf16")
    wr = layer.w_router.copy()
    wr[9] = wr[2]
    wr[12] = wr[5]
    layer.w_router = wr
    x = W.make_tokens(42, T, 256, "bf16")
    out = run_gpu(_layer_gpu(layer), x, "bf16")
    l = out["logits"]
    assert np.array_equal(l[:, 9], l[:, 2]) and np.array_equal(l[:, 12], l[:, 5])
    for t in range(T):
        ids = out["ids"][t].tolist()
        assert 9 not in ids or 2 in ids
        if 2 in ids and 9 in ids:
            assert ids.index(2) < ids.index(9)


# ---------------------------------------------------------------- permute
@pytest.mark.parametrize("T,k,E", [(1, 10, 512), (37, 10, 512), (500, 10, 512), (8192, 10, 512),
                                   (3, 10, 24576), (2000, 3, 7), (1, 1, 1), (4096, 1, 32768),
                                   (1, 10, 24576), (2, 16, 32768), (3, 11, 100)])
def test_permute_bit_exact(T, k, E):
    rng = np.random.default_rng(T + 13 * k + E)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    ref = oracle.permute(ids, E)
    n = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ps = torch.empty(n, dtype=torch.int32, device="cuda")
    pd = torch.empty(n, dtype=torch.int32, device="cuda")
    act = torch.empty(1 + min(n, E) + 3, dtype=torch.int32, device="cuda")
    wsb = M.moe_permute_ws_size(T, k, E)
    ws = torch.empty(max(16, wsb), dtype=torch.uint8, device="cuda")
    M.moe_permute(_t(ids), T, k, E, offsets, ps, pd, act, ws, wsb)
    assert M.moe_device_error(clear=True) == 0
    assert np.array_equal(offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(ps.cpu().numpy(), ref["perm_src"])
    assert np.array_equal(pd.cpu().numpy().reshape(T, k), ref["perm_dst"])
    a = act.cpu().numpy()
    assert np.array_equal(a[:1 + a[0]], ref["active"])


def test_permute_empty_and_bad_id():
    offsets = torch.full((17,), 7, dtype=torch.int32, device="cuda")
    act = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    M.moe_permute(None, 0, 2, 16, offsets, None, None, act)
    assert offsets.cpu().numpy().tolist() == [0] * 17 and act[0].item() == 0
    ids = _t(np.array([[1, 16]], np.int32))
    ps = torch.empty(2, dtype=torch.int32, device="cuda")
    pd = torch.empty(2, dtype=torch.int32, device="cuda")
    M.moe_permute(ids, 1, 2, 16, offsets, ps, pd, act)
    assert M.moe_device_error(clear=True) & M.DEVERR_BAD_EXPERT


# ---------------------------------------------------------------- combine
def test_combine_against_oracle():
    rng = np.random.default_rng(5)
    T, k, H = 37, 10, 512
    yp = rng.standard_normal((T * k, H)).astype(np.float32)
    pd = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    w = rng.random((T, k)).astype(np.float32)
    ys = rng.standard_normal((T, H)).astype(np.float32)
    ref = oracle.combine(yp.astype(np.float64), pd, w.astype(np.float64), ys.astype(np.float64))
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    M.moe_combine(_t(yp), _t(pd), _t(w), _t(ys), T, k, H, y)
    assert rel_err(y.cpu().numpy().reshape(T, H), ref) < 1e-6


# ------------------------------------------------------------ whole layer
def _check_undecided(gpu_logits, gpu_ids, k):
    """Tokens whose routing margin is within the logit error bound: their ids
    must be the top-k of the GPU's own fp32 logits (same precision on both
    sides)."""
    if gpu_ids.shape[0] == 0:
        return
    ids_ref, _, _ = oracle.topk(np.ascontiguousarray(gpu_logits, np.float32), k)
    assert np.array_equal(gpu_ids, ids_ref)


def _check_layer(out, ref, layer, x, x_dtype, tol=TOL):
    """ids/permutation bit-exact where the routing margin is decisive (the
    rest: the top-k of the GPU's own logits); y within tol."""
    eps = logit_bound(layer, x, x_dtype) if layer.w_router is not None else np.zeros_like(ref["logits"])
    dec = decisive_tokens(ref["logits"], eps, layer.k)
    assert out["err"] == 0
    assert np.array_equal(out["ids"][dec], ref["ids"][dec])
    _check_undecided(out["logits"][~dec], out["ids"][~dec], layer.k)
    if dec.all():
        assert np.array_equal(out["offsets"], ref["offsets"])
        assert np.array_equal(out["perm_src"], ref["perm_src"])
        assert np.array_equal(out["perm_dst"], ref["perm_dst"])
    e = rel_err(out["y"][dec], ref["y"][dec])
    assert e <= tol, f"max|y - y_oracle| = {e:.3e} x RMS"
    return e, int((~dec).sum())


def test_layer_tiny_gemv():
    layer, x = W.tiny_case()
    ref = oracle.moe_layer(4, x, "f32", layer.blobs, k=2, H=256, I=128, E=16, w_router=layer.w_router,
                           w_dtype="f32", want_yperm=True)
    out = run_gpu(_layer_gpu(layer), x, "f32", mode=M.MOE_MODE_GEMV)
    e, _ = _check_layer(out, ref, layer, x, "f32")
    assert e < GEMV_TOL
    assert rel_err(out["y_perm"], ref["y_perm"]) < GEMV_TOL


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("T", [1, 3, 16, 40])
def test_layer_small_gemv(bits, T):
    layer = W.make_layer(50 + bits, bits, 256, 128, 24, 4, shared=True, w_dtype="bf16")
    x = W.make_tokens(60 + T, T, 256, "bf16")
    ref = oracle.moe_layer(bits, x, "bf16", layer.blobs, k=4, H=256, I=128, E=24, w_router=layer.w_router,
                           w_dtype="bf16", shared_blob=layer.shared, want_yperm=True)
    out = run_gpu(_layer_gpu(layer), x, "bf16", mode=M.MOE_MODE_GEMV)
    e, _ = _check_layer(out, ref, layer, x, "bf16")
    assert e < GEMV_TOL
    assert rel_err(out["y_shared"], ref["y_shared"]) < GEMV_TOL


@pytest.mark.parametrize("mode", [M.MOE_MODE_GEMM, M.MOE_MODE_AUTO])
@pytest.mark.parametrize("bits,T", [(4, 300), (2, 300), (4, 17), (4, 1000)])
def test_layer_ragged_gemm(mode, bits, T):
    """Several tiles per expert with ragged tails (uneven per-expert counts)."""
    layer = W.make_layer(70 + bits, bits, 256, 256, 8, 2, shared=True, w_dtype="bf16")
    x = W.make_tokens(71 + T, T, 256, "bf16")
    ref = oracle.moe_layer(bits, x, "bf16", layer.blobs, k=2, H=256, I=256, E=8, w_router=layer.w_router,
                           w_dtype="bf16", shared_blob=layer.shared)
    out = run_gpu(_layer_gpu(layer), x, "bf16", mode=mode)
    _check_layer(out, ref, layer, x, "bf16")


@pytest.mark.parametrize("bits", [4, 2])
def test_layer_gemm_odd_hidden(bits):
    """H = 384: the down GEMM's last tile holds one 128-row matrix, not two."""
    layer = W.make_layer(80 + bits, bits, 384, 256, 8, 2, shared=True, w_dtype="bf16")
    x = W.make_tokens(81, 300, 384, "bf16")
    ref = oracle.moe_layer(bits, x, "bf16", layer.blobs, k=2, H=384, I=256, E=8, w_router=layer.w_router,
                           w_dtype="bf16", shared_blob=layer.shared)
    out = run_gpu(_layer_gpu(layer), x, "bf16", mode=M.MOE_MODE_GEMM)
    _check_layer(out, ref, layer, x, "bf16")


# ------------------------------------------------------ full-size layers
@pytest.fixture(scope="module")
def decode_layer():
    c = W.DECODE
    layer = W.make_layer(W.SEED["decode"], 4, c["H"], c["I"], c["E"], c["k"], shared=True, w_dtype="bf16")
    return layer, _layer_gpu(layer)


def _sampled_ref(layer, x, rows):
    return oracle.moe_layer(layer.bits, x[rows], "bf16", layer.blobs, k=layer.k, H=layer.H, I=layer.I, E=layer.E,
                            w_router=layer.w_router, w_dtype="bf16", bias=layer.bias, shared_blob=layer.shared)


@pytest.mark.parametrize("T", [1, 4])
def test_decode_full_size(decode_layer, T):
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["decode"] + 100 + T, T, layer.H, "bf16")
    out = run_gpu(g, x, "bf16")
    ref = _sampled_ref(layer, x, np.arange(T))
    e, _ = _check_layer(out, ref, layer, x, "bf16")
    assert e < GEMV_TOL


def _tile_edge_rows(n, tiles=(64, 256)):
    """Local row positions that start or end a token tile of either size, plus the last row."""
    pos = {0, n - 1}
    for t in tiles:
        for b in range(t, n, t):
            pos.update((b - 1, b))
    return sorted(p for p in pos if 0 <= p < n)


def _check_expert_rows(out, layer, x, tol=TOL):
    """y_perm rows at the first and last row of every active expert and at
    every token-tile edge, and y_shared at the shared expert's tile edges,
    each against the oracle's FFN of that expert on that token.  Covers every
    expert group and every tile tail of the grouped GEMM."""
    T, H, I = x.shape[0], layer.H, layer.I
    offs, ps = out["offsets"], out["perm_src"]
    xs = xd(x, "bf16")
    rows, blobs = [], []
    for e in range(layer.E):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        for p in (_tile_edge_rows(r1 - r0) if r1 > r0 else []):
            rows.append(r0 + p)
            blobs.append(layer.blobs[e])
    ref = oracle.expert_ffn_rows(layer.bits, H, I, blobs, xs[ps[rows]])
    got = out["y_perm"][rows]
    assert rel_err(got, ref) <= tol, f"y_perm rows: {rel_err(got, ref):.3e} x RMS over {len(rows)} rows"
    if layer.shared is not None:
        toks = _tile_edge_rows(T)
        ref_s = oracle.expert_ffn_rows(layer.bits, H, I, [layer.shared] * len(toks), xs[toks])
        assert rel_err(out["y_shared"][toks], ref_s) <= tol
    return len(rows)


@pytest.mark.parametrize("T", [512, 2048, 8192])
def test_prefill_full_size_sampled(decode_layer, T):
    """Prefill chunk in GEMM mode (the launch configuration the benchmark
    times) at full layer size: every expert's edge rows against the oracle,
    the combined output on sampled tokens, and the routing of every token."""
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["prefill"] + T, T, layer.H, "bf16")
    out = run_gpu(g, x, "bf16", mode=M.MOE_MODE_GEMM)
    assert out["err"] == 0
    n_rows = _check_expert_rows(out, layer, x)
    assert n_rows >= 2 * int(out["active"][0]) - 1
    rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, 6, replace=False)]))
    ref = _sampled_ref(layer, x, rows)
    eps = logit_bound(layer, x[rows], "bf16")
    dec = decisive_tokens(ref["logits"], eps, layer.k)
    assert np.array_equal(out["ids"][rows][dec], ref["ids"][dec])
    e = rel_err(out["y"][rows][dec], ref["y"][dec])
    assert e <= TOL, e
    # every token: the ids are the top-k of the GPU's own fp32 logits, and
    # the logits are within the fp32 error bound of the exact ones
    _check_undecided(out["logits"], out["ids"], layer.k)
    ref_l = oracle.router_logits(x[rows], "bf16", layer.w_router, "bf16", layer.bias)
    assert np.all(np.abs(out["logits"][rows] - ref_l) <= eps)
    # whole-chunk invariants: every row of the permutation is used once
    assert sorted(out["perm_dst"].ravel().tolist()) == list(range(T * layer.k))
    assert out["offsets"][-1] == T * layer.k
    assert np.array_equal(out["offsets"], oracle.permute(out["ids"], layer.E)["offsets"])


@pytest.mark.parametrize("bits", [4, 2])
def test_gemm_many_tiles_per_cta(bits):
    """A shape whose 256-token tiles number several per CTA in both GEMMs
    (gate/up: 8 experts x 16 token tiles x 4 row tiles + the shared expert's
    128 = 640 tiles; down: 320), so each CTA reuses its TMEM accumulator
    across tiles."""
    H, I, E, k, T = 512, 512, 8, 4, 8192
    layer = W.make_layer(90 + bits, bits, H, I, E, k, shared=True, w_dtype="bf16")
    x = W.make_tokens(91 + bits, T, H, "bf16")
    out = run_gpu(_layer_gpu(layer), x, "bf16", mode=M.MOE_MODE_GEMM)
    assert out["err"] == 0
    counts = np.diff(out["offsets"])
    assert counts.min() > 256 * 2                     # several 256-token tiles per expert
    _check_expert_rows(out, layer, x)
    rows = np.unique(np.concatenate([[0, 255, 256, T - 1], np.random.default_rng(bits).choice(T, 8, replace=False)]))
    ref = _sampled_ref(layer, x, rows)
    eps = logit_bound(layer, x[rows], "bf16")
    dec = decisive_tokens(ref["logits"], eps, k)
    assert np.array_equal(out["ids"][rows][dec], ref["ids"][dec])
    assert rel_err(out["y"][rows][dec], ref["y"][dec]) <= TOL
    _check_undecided(out["logits"], out["ids"], k)


@pytest.fixture(scope="module")
def verify_layer():
    layer = W.verify_layer()
    return layer, _layer_gpu(layer)


@pytest.mark.parametrize("T", [2, 3, 5, 9, 16])
def test_verify_windows_q2(verify_layer, T):
    layer, g = verify_layer
    x = W.make_tokens(W.SEED["verify"] + T, T, layer.H, "bf16")
    out = run_gpu(g, x, "bf16")
    ref = _sampled_ref(layer, x, np.arange(T))
    e, _ = _check_layer(out, ref, layer, x, "bf16")
    assert e < GEMV_TOL
    # the window gives the rows of T single-token steps (Strata article, section 2 item 3)
    for t in range(T):
        one = run_gpu(g, x[t:t + 1], "bf16")
        assert np.array_equal(one["ids"][0], out["ids"][t])
        assert rel_err(one["y"][0], out["y"][t]) < 1e-6


def test_null_blob_sets_error(decode_layer):
    layer, g = decode_layer
    x = W.make_tokens(5, 1, layer.H, "bf16")
    out = run_gpu(g, x, "bf16")
    e = int(out["ids"][0, 0])
    saved = g.table[e].item()
    g.table[e] = 0
    try:
        out = run_gpu(g, x, "bf16")
        assert out["err"] & M.DEVERR_NULL_BLOB
    finally:
        g.table[e] = saved
    assert run_gpu(g, x, "bf16")["err"] == 0


# ------------------------------------------------------ fused decode step
@pytest.fixture(params=["chain", "one_kernel"])
def decode_path(request):
    """Runs a test on both fused decode paths: the three-kernel chain (the
    default) and the one-kernel persistent step (test hook)."""
    M.moe_test_hook(M.MOE_HOOK_DECODE_ONE_KERNEL, 1 if request.param == "one_kernel" else 0)
    yield request.param
    M.moe_test_hook(M.MOE_HOOK_DECODE_ONE_KERNEL, 0)


@pytest.fixture
def one_kernel():
    M.moe_test_hook(M.MOE_HOOK_DECODE_ONE_KERNEL, 1)
    yield
    M.moe_test_hook(M.MOE_HOOK_DECODE_ONE_KERNEL, 0)


def _run_fused(g, x, x_dtype, logits_in=None):
    import quantized_expert_ffn_route_b200 as MM
    xdev = dev_x(x, x_dtype)
    li = None if logits_in is None else torch.from_numpy(np.ascontiguousarray(logits_in, np.float32)).cuda()
    b = g.forward_decode(xdev, MM.MOE_BF16 if x_dtype == "bf16" else MM.MOE_F32, logits_in=li)
    torch.cuda.synchronize()
    return dict(err=MM.moe_device_error(clear=True), ids=b["ids"][:g.k].cpu().numpy(),
                w=b["w"][:g.k].cpu().numpy(), logits=b["logits"].cpu().numpy(), y=b["y"].cpu().numpy())


def test_prepared_decode_matches_forward_decode(decode_path):
    """The prepared one-token call runs the same kernels on the same buffers."""
    layer = W.make_layer(430, 4, 256, 256, 24, 4, shared=True, w_dtype="bf16")
    x = W.make_tokens(431, 3, 256, "bf16")
    g = _layer_gpu(layer)
    xd = torch.empty(1, 256, dtype=torch.bfloat16, device="cuda")
    step = g.prepare_decode(xd, M.MOE_BF16)
    for t in range(3):
        xd.copy_(dev_x(x[t:t + 1], "bf16"))
        b = step()
        torch.cuda.synchronize()
        y1, ids1 = b["y"].clone(), b["ids"][:4].clone()
        f = _run_fused(g, x[t:t + 1], "bf16")
        assert f["err"] == 0
        assert np.array_equal(ids1.cpu().numpy(), f["ids"])
        assert np.array_equal(y1.cpu().numpy(), f["y"])


def test_fused_decode_full_size(decode_layer, decode_path):
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["decode"] + 500, 6, layer.H, "bf16")
    ref = _sampled_ref(layer, x, np.arange(6))
    eps = logit_bound(layer, x, "bf16")
    dec = decisive_tokens(ref["logits"], eps, layer.k)
    for t in range(6):
        f = _run_fused(g, x[t:t + 1], "bf16")
        assert f["err"] == 0
        assert np.all(np.abs(f["logits"] - ref["logits"][t]) <= eps[t])
        if dec[t]:
            assert np.array_equal(f["ids"], ref["ids"][t])
            assert rel_err(f["y"], ref["y"][t]) < GEMV_TOL
        # the gates are the softmax of the call's own selected logits (ids:
        # the top-k of those logits, as the oracle selects them in fp32)
        ids_own, w_own, _ = oracle.topk(f["logits"][None].astype(np.float32), layer.k)
        assert np.array_equal(f["ids"], ids_own[0])
        assert np.allclose(f["w"], w_own[0], rtol=4e-6, atol=1e-8)
        # same routing and outputs as the separate calls (their logits are
        # summed in another order: gates agree within the logit error bound)
        m = run_gpu(g, x[t:t + 1], "bf16", mode=M.MOE_MODE_GEMV)
        assert np.array_equal(f["ids"], m["ids"][0])
        assert np.allclose(f["w"], m["w"][0], rtol=4 * float(eps[t].max()) + 4e-6, atol=1e-8)
        assert rel_err(f["y"], m["y"][0]) < 1e-4   # two fp32 orders of the same cancellation, each ~2e-5


def test_fused_decode_q2_bias(verify_layer, decode_path):
    layer, g = verify_layer
    x = W.make_tokens(W.SEED["verify"] + 900, 3, layer.H, "bf16")
    ref = _sampled_ref(layer, x, np.arange(3))
    eps = logit_bound(layer, x, "bf16")
    dec = decisive_tokens(ref["logits"], eps, layer.k)
    for t in range(3):
        f = _run_fused(g, x[t:t + 1], "bf16")
        assert f["err"] == 0
        if dec[t]:
            assert np.array_equal(f["ids"], ref["ids"][t])
            assert rel_err(f["y"], ref["y"][t]) < GEMV_TOL


@pytest.mark.parametrize("bits,dt,shared,H,I", [(4, "f32", False, 256, 256), (2, "bf16", True, 256, 256),
                                               (4, "bf16", True, 256, 256), (4, "bf16", True, 256, 128),
                                               (2, "f32", False, 384, 256)])
def test_fused_decode_small(bits, dt, shared, H, I, decode_path):
    """H and I multiples of 256: the one-kernel step; I = 128 or H = 384
    (scale rows not 16-byte multiples): the three-kernel chain."""
    layer = W.make_layer(400 + bits, bits, H, I, 24, 4, shared=shared, w_dtype=dt)
    x = W.make_tokens(401 + bits, 3, H, dt)
    ref = oracle.moe_layer(bits, x, dt, layer.blobs, k=4, H=H, I=I, E=24, w_router=layer.w_router,
                           w_dtype=dt, shared_blob=layer.shared)
    g = _layer_gpu(layer)
    eps = logit_bound(layer, x, dt)
    dec = decisive_tokens(ref["logits"], eps, 4)
    for t in range(3):
        f = _run_fused(g, x[t:t + 1], dt)
        assert f["err"] == 0
        if dec[t]:
            assert np.array_equal(f["ids"], ref["ids"][t])
            assert rel_err(f["y"], ref["y"][t]) < GEMV_TOL


def test_fused_decode_logits_in(decode_path):
    """Router logits given directly (the paging path), with exact ties."""
    layer = W.make_layer(410, 2, 256, 256, 64, 6, shared=False, w_dtype="bf16")
    x = W.make_tokens(411, 2, 256, "bf16")
    rng = np.random.default_rng(412)
    li = rng.integers(-2, 3, size=(2, 64)).astype(np.float32)
    ref = oracle.moe_layer(2, x, "bf16", layer.blobs, k=6, H=256, I=256, E=64, logits_in=li)
    g = _layer_gpu(layer)
    for t in range(2):
        f = _run_fused(g, x[t:t + 1], "bf16", logits_in=li[t:t + 1])
        assert f["err"] == 0
        assert np.array_equal(f["ids"], ref["ids"][t])
        assert rel_err(f["y"], ref["y"][t]) < GEMV_TOL


def test_fused_decode_is_one_kernel_and_replays_from_a_graph(decode_layer, one_kernel):
    """At full size the one-kernel step is a single kernel launch; captured in
    a CUDA graph and replayed it gives the eager result bit for bit, call
    after call; its grid-barrier arrival count moves on by exactly two
    arrivals per CTA per call."""
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["decode"] + 700, 3, layer.H, "bf16")
    b = g.decode_buffers()

    def count():
        return int(b["ws"][256:264].cpu().numpy().view(np.uint64)[0])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    eager = []
    for t in range(3):
        n0, c0 = M.moe_kernel_launches(), count()
        f = _run_fused(g, x[t:t + 1], "bf16")
        assert f["err"] == 0 and M.moe_kernel_launches() - n0 == 1
        assert count() - c0 == 2 * sms
        eager.append(f)
    xd = torch.empty(1, layer.H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            g.forward_decode(xd, M.MOE_BF16, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    c0 = count()
    for t in (2, 0, 1):
        xd.copy_(dev_x(x[t:t + 1], "bf16"))
        graph.replay()
        torch.cuda.synchronize()
        assert M.moe_device_error(clear=True) == 0
        assert np.array_equal(b["ids"][:layer.k].cpu().numpy(), eager[t]["ids"])
        assert np.array_equal(b["y"].cpu().numpy(), eager[t]["y"])
    assert count() - c0 == 3 * 2 * sms


def test_fused_decode_chain_replays_from_a_graph_and_leaves_ws_ready(decode_layer):
    """The default path at full size is three kernels (route, gate/up, down)
    per call; replayed from a CUDA graph it gives the eager result bit for
    bit, and every call returns the route kernel's ticket count to zero."""
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["decode"] + 710, 3, layer.H, "bf16")
    b = g.decode_buffers()

    def tickets():
        return int(b["ws"][264:268].cpu().numpy().view(np.uint32)[0])
    eager = []
    for t in range(3):
        n0 = M.moe_kernel_launches()
        f = _run_fused(g, x[t:t + 1], "bf16")
        assert f["err"] == 0 and M.moe_kernel_launches() - n0 == 3
        assert tickets() == 0
        eager.append(f)
    xd_ = torch.empty(1, layer.H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            g.forward_decode(xd_, M.MOE_BF16, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for t in (2, 0, 1, 2):
        xd_.copy_(dev_x(x[t:t + 1], "bf16"))
        graph.replay()
        torch.cuda.synchronize()
        assert M.moe_device_error(clear=True) == 0
        assert np.array_equal(b["ids"][:layer.k].cpu().numpy(), eager[t]["ids"])
        assert np.array_equal(b["y"].cpu().numpy(), eager[t]["y"])
        assert tickets() == 0


def test_fused_decode_leaves_out_null_and_misaligned_blobs(decode_path):
    """A selected expert whose table entry is NULL (MOE_DEVERR_NULL_BLOB) or
    not 16-byte aligned (MOE_DEVERR_MISALIGNED) is left out: the ids and
    gates are unchanged, and y is the full step minus that slot's weighted
    expert output (the oracle's FFN of that expert)."""
    layer = W.make_layer(440, 4, 256, 256, 24, 4, shared=True, w_dtype="bf16")
    x = W.make_tokens(441, 1, 256, "bf16")
    g = _layer_gpu(layer)
    full = _run_fused(g, x, "bf16")
    assert full["err"] == 0
    j = 1
    e = int(full["ids"][j])
    saved = int(g.table[e].item())
    outs = {}
    for name, val, bit in (("null", 0, M.DEVERR_NULL_BLOB), ("misaligned", saved + 8, M.DEVERR_MISALIGNED)):
        g.table[e] = val
        try:
            r = _run_fused(g, x, "bf16")
        finally:
            g.table[e] = saved
        assert r["err"] == bit, (name, r["err"])
        assert np.array_equal(r["ids"], full["ids"]) and np.array_equal(r["w"], full["w"])
        outs[name] = r["y"]
    assert np.array_equal(outs["null"], outs["misaligned"])
    ffn_j = oracle.expert_ffn_rows(4, 256, 256, [layer.blobs[e]], xd(x, "bf16")[:1])[0]
    want = full["y"].astype(np.float64) - float(full["w"][j]) * ffn_j
    assert rel_err(outs["null"], want) <= TOL
    again = _run_fused(g, x, "bf16")                      # the table restored: the full step again
    assert again["err"] == 0 and np.array_equal(again["y"], full["y"])


def test_fused_decode_barrier_timeout_recovers(decode_layer, one_kernel):
    """A grid barrier that can never complete (the test hook makes it wait
    for one CTA more than the grid has) runs out after its 2 ms limit: the
    call sets MOE_DEVERR_TIMEOUT and returns; with the hook cleared and the
    workspace zeroed again, the next call is exact."""
    layer, g = decode_layer
    x = W.make_tokens(W.SEED["decode"] + 800, 1, layer.H, "bf16")
    good = _run_fused(g, x, "bf16")
    assert good["err"] == 0
    b = g.decode_buffers()
    M.moe_test_hook(M.MOE_HOOK_WAIT_LIMIT_NS, 2_000_000)
    M.moe_test_hook(M.MOE_HOOK_DECODE_EXTRA_ARRIVALS, 1)
    try:
        g.forward_decode(dev_x(x, "bf16"), M.MOE_BF16)
        torch.cuda.synchronize()
        err = M.moe_device_error(clear=True)
    finally:
        M.moe_test_hook(M.MOE_HOOK_DECODE_EXTRA_ARRIVALS, 0)
        M.moe_test_hook(M.MOE_HOOK_WAIT_LIMIT_NS, 0)
    assert err & M.MOE_DEVERR_TIMEOUT
    b["ws"].zero_()
    again = _run_fused(g, x, "bf16")
    assert again["err"] == 0
    assert np.array_equal(again["ids"], good["ids"]) and np.array_equal(again["y"], good["y"])


def test_gemm_wait_timeout_recovers():
    """The grouped GEMM's pipeline waits limited to two polls (test hook) run
    out: the call sets MOE_DEVERR_TIMEOUT, every role leaves its loop, TMEM is
    freed (the kernel returns), and the next call with the normal limit is
    exact."""
    layer = W.make_layer(72, 4, 256, 256, 8, 2, shared=True, w_dtype="bf16")
    x = W.make_tokens(73, 300, 256, "bf16")
    g = _layer_gpu(layer)
    M.moe_test_hook(M.MOE_HOOK_GEMM_SPIN, 2)
    try:
        out = run_gpu(g, x, "bf16", mode=M.MOE_MODE_GEMM)
    finally:
        M.moe_test_hook(M.MOE_HOOK_GEMM_SPIN, 0)
    assert out["err"] & M.MOE_DEVERR_TIMEOUT
    ref = oracle.moe_layer(4, x, "bf16", layer.blobs, k=2, H=256, I=256, E=8, w_router=layer.w_router,
                           w_dtype="bf16", shared_blob=layer.shared)
    for _ in range(2):
        out = run_gpu(g, x, "bf16", mode=M.MOE_MODE_GEMM)
        _check_layer(out, ref, layer, x, "bf16")


def test_decode_session_matches_forward_decode():
    """The decode session (x copied in, the step, y and ids copied out, one
    recorded graph per call) gives forward_decode's output bit for bit, token
    after token; it refuses the legacy default stream."""
    layer = W.make_layer(450, 4, 256, 256, 24, 4, shared=True, w_dtype="bf16")
    x = W.make_tokens(451, 5, 256, "bf16")
    g = _layer_gpu(layer)
    x_in = torch.empty(256, dtype=torch.bfloat16).pin_memory()
    y_out = torch.empty(256, dtype=torch.float32).pin_memory()
    ids_out = torch.empty(4, dtype=torch.int32).pin_memory()
    s = torch.cuda.Stream()
    x_in.copy_(torch.from_numpy(x[0].view(np.int16)).view(torch.bfloat16))   # creation runs one step on x_in
    sess = g.decode_session(x_in, M.MOE_BF16, y_out, s, ids_host=ids_out)
    torch.cuda.synchronize()
    assert M.moe_device_error(clear=True) == 0
    try:
        for t in range(5):
            x_in.copy_(torch.from_numpy(x[t].view(np.int16)).view(torch.bfloat16))
            n0 = M.moe_kernel_launches()
            sess.run()
            assert M.moe_kernel_launches() - n0 == 3
            ref = _run_fused(g, x[t:t + 1], "bf16")
            assert ref["err"] == 0 and M.moe_device_error() == 0
            assert np.array_equal(y_out.numpy(), ref["y"]) and np.array_equal(ids_out.numpy(), ref["ids"])
    finally:
        sess.close()
    with pytest.raises(M.MoEError) as ei:
        M.lib()                                               # the default stream cannot be captured
        g.decode_session(x_in, M.MOE_BF16, y_out, torch.cuda.default_stream())
    assert ei.value.status == M.MOE_EINVAL
