"""The allocation-free expert FFN entry point (moe_expert_ffn_noalloc).

It exists for callers that cannot allocate device memory when they run the
step -- code running inside CUDA-graph stream capture, engines with a memory
budget fixed at start-up, C hosts without a device allocator -- and takes its
scratch from an array built into the library.  This file is collected last so
that a run stopping at the first failure has already run every other test;
it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402

TOL = 2e-3   # the output tolerance of the parity tests (x RMS)


def _rel(a, b):
    rms = float(np.sqrt(np.mean(np.square(b))))
    return float(np.max(np.abs(a - b))) / rms


@pytest.mark.parametrize("bits,T", [(4, 1), (4, 8), (2, 5)])
def test_noalloc_matches_workspace_entry_point(bits, T):
    H, I, E, k = 256, 128, 16, 4
    layer = W.make_layer(300 + bits, bits, H, I, E, k, shared=True, w_dtype="bf16")
    x = W.make_tokens(310 + T, T, H, "bf16")
    g = M.MoELayer(bits, H, I, E, k, layer.blobs, layer.shared, layer.w_router, "bf16")
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    b = g.forward(xd, M.MOE_BF16, mode=M.MOE_MODE_GEMV)          # routing + reference FFN (with workspace)
    torch.cuda.synchronize()
    ref_perm = b.y_perm.clone()
    ref_shared = b.y_shared.clone()
    outs = []
    for call in range(2):                                      # two calls in a row share the scratch
        yp = torch.full_like(ref_perm, float("nan"))
        ys = torch.full_like(ref_shared, float("nan"))
        M.moe_expert_ffn_noalloc(bits, g.table, b.offsets, b.active, b.perm_src, xd, M.MOE_BF16, T, k, H, I, E,
                                 g.shared, yp, ys)
        torch.cuda.synchronize()
        assert M.moe_device_error() == 0
        n = T * k * H
        outs.append((yp[:n].cpu().numpy(), ys[:T * H].cpu().numpy()))
    for yp, ys in outs:
        assert _rel(yp, ref_perm[:T * k * H].cpu().numpy()) <= TOL
        assert _rel(ys, ref_shared[:T * H].cpu().numpy()) <= TOL


def test_noalloc_rejects_oversized_calls():
    cap = M.moe_expert_ffn_noalloc_max_bytes()
    assert cap == 8 << 20
    # T*(k+1)*I*4 bytes of scratch: T = 1024, k = 10, I = 2048 (2-bit) needs 92 MB
    p = torch.zeros(64, dtype=torch.int64, device="cuda")
    with pytest.raises(M.MoEError) as ei:
        M.moe_expert_ffn_noalloc(2, p, p, p, p, p, M.MOE_BF16, 1024, 10, 2048, 2048, 512, None, p, None)
    assert ei.value.status == M.MOE_EINVAL
    assert "scratch" in M.moe_last_error()
