"""The allocation-free expert FFN entry point (moe_expert_ffn_noalloc).

It exists for callers that cannot allocate device memory when they run the
step -- engines held to a device-memory budget fixed at start-up, C hosts
without a device allocator of their own, and latency-critical loops where an
allocation could synchronise the device -- and takes its scratch from an
array built into the library.  This file is collected last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402

TOL = 2e-3   # the output tolerance of the parity tests (x RMS)


def _rel(a, b):
    rms = float(np.sqrt(np.mean(np.square(b))))
    return float(np.max(np.abs(a - b))) / rms


def _xd(x):
    return W.bf16_bits_to_f32(x).astype(np.float64)


def _setup(bits, H, I, E, k, T, seed):
    layer = W.make_layer(seed, bits, H, I, E, k, shared=True, w_dtype="bf16")
    x = W.make_tokens(seed + 10, T, H, "bf16")
    g = M.MoELayer(bits, H, I, E, k, layer.blobs, layer.shared, layer.w_router, "bf16")
    xdev = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    b = g.forward(xdev, M.MOE_BF16, mode=M.MOE_MODE_GEMV)         # routing + the workspace FFN
    torch.cuda.synchronize()
    return layer, x, g, xdev, b


def _noalloc(bits, g, b, xdev, T, k, H, I, E):
    yp = torch.full((T * k * H,), float("nan"), dtype=torch.float32, device="cuda")
    ys = torch.full((T * H,), float("nan"), dtype=torch.float32, device="cuda")
    M.moe_expert_ffn_noalloc(bits, g.table, b.offsets, b.active, b.perm_src, xdev, M.MOE_BF16, T, k, H, I, E,
                             g.shared, yp, ys)
    torch.cuda.synchronize()
    assert M.moe_device_error() == 0
    return yp.cpu().numpy().reshape(T * k, H), ys.cpu().numpy().reshape(T, H)


def _oracle_rows(layer, x, b, rows, T):
    """The oracle's FFN of each checked permuted row's expert on its token,
    and of the shared expert on every token."""
    offs = b.offsets[:layer.E + 1].cpu().numpy()
    ps = b.perm_src[:T * layer.k].cpu().numpy()
    expert_of = np.searchsorted(offs, rows, side="right") - 1
    xs = _xd(x)
    yp = oracle.expert_ffn_rows(layer.bits, layer.H, layer.I, [layer.blobs[e] for e in expert_of], xs[ps[rows]])
    ys = oracle.expert_ffn_rows(layer.bits, layer.H, layer.I, [layer.shared] * T, xs)
    return yp, ys


@pytest.mark.parametrize("bits,T", [(4, 1), (4, 8), (2, 5)])
def test_noalloc_matches_workspace_entry_point(bits, T):
    H, I, E, k = 256, 128, 16, 4
    layer, x, g, xdev, b = _setup(bits, H, I, E, k, T, 300 + bits + T)
    ref_perm = b.y_perm[:T * k * H].cpu().numpy().reshape(T * k, H)
    ref_shared = b.y_shared[:T * H].cpu().numpy().reshape(T, H)
    rows = np.arange(T * k)
    or_perm, or_shared = _oracle_rows(layer, x, b, rows, T)
    for call in range(2):                                      # two calls in a row share the scratch
        yp, ys = _noalloc(bits, g, b, xdev, T, k, H, I, E)
        assert _rel(yp, ref_perm) <= TOL and _rel(ys, ref_shared) <= TOL
        assert _rel(yp, or_perm) <= TOL and _rel(ys, or_shared) <= TOL


def test_noalloc_scratch_boundary_then_small_call():
    """T*(k+1)*I*4 equal to the built-in size is accepted and exact; one more
    token is rejected; a small call of another shape right after the large
    one (the scratch still holds the large call's values) is exact too."""
    cap = M.moe_expert_ffn_noalloc_max_bytes()
    assert cap == 8 << 20
    bits, H, I, E, k = 4, 128, 512, 8, 3
    T = cap // ((k + 1) * I * 4)
    assert T == 1024 and T * (k + 1) * I * 4 == cap
    layer, x, g, xdev, b = _setup(bits, H, I, E, k, T, 350)
    yp, ys = _noalloc(bits, g, b, xdev, T, k, H, I, E)
    assert _rel(yp, b.y_perm[:T * k * H].cpu().numpy().reshape(T * k, H)) <= TOL
    offs = b.offsets[:E + 1].cpu().numpy()
    rows = np.unique(np.concatenate([offs[:-1][np.diff(offs) > 0], offs[1:][np.diff(offs) > 0] - 1, [0, T * k - 1]]))
    or_perm, or_shared = _oracle_rows(layer, x, b, rows, T)
    assert _rel(yp[rows], or_perm) <= TOL and _rel(ys, or_shared) <= TOL
    with pytest.raises(M.MoEError) as ei:
        M.moe_expert_ffn_noalloc(bits, g.table, b.offsets, b.active, b.perm_src, xdev, M.MOE_BF16, T + 1, k, H, I,
                                 E, g.shared, b.y_perm, b.y_shared)
    assert ei.value.status == M.MOE_EINVAL and "scratch" in M.moe_last_error()
    # a small call of another shape after the large one
    layer2, x2, g2, xdev2, b2 = _setup(2, 256, 128, 16, 4, 1, 360)
    yp2, ys2 = _noalloc(2, g2, b2, xdev2, 1, 4, 256, 128, 16)
    or_perm2, or_shared2 = _oracle_rows(layer2, x2, b2, np.arange(4), 1)
    assert _rel(yp2, or_perm2) <= TOL and _rel(ys2, or_shared2) <= TOL


def test_noalloc_rejects_oversized_calls():
    # T*(k+1)*I*4 bytes of scratch: T = 1024, k = 10, I = 2048 (2-bit) needs 92 MB
    p = torch.zeros(64, dtype=torch.int64, device="cuda")
    with pytest.raises(M.MoEError) as ei:
        M.moe_expert_ffn_noalloc(2, p, p, p, p, p, M.MOE_BF16, 1024, 10, 2048, 2048, 512, None, p, None)
    assert ei.value.status == M.MOE_EINVAL
    assert "scratch" in M.moe_last_error()
