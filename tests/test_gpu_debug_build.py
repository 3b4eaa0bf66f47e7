"""The MOE_DEBUG build (MOE_LIBRARY=debug): an out-of-range permutation entry
passed to the expert FFN is kept in range by every build, and reported in the
device error word (MOE_DEVERR_BAD_ROW) by the debug build only.  Each build
runs in its own process, since a process loads one of them."""
import json
import os
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parents[1]

SCRIPT = r'''
import json
import numpy as np
import torch
import quantized_expert_ffn_route_b200 as M
import workloads as W

T, H, I, E, k = 8, 256, 128, 16, 2
layer = W.make_layer(410, 4, H, I, E, k, shared=True, w_dtype="bf16")
x = W.make_tokens(411, T, H, "bf16")
g = M.MoELayer(4, H, I, E, k, layer.blobs, layer.shared, layer.w_router, "bf16")
xdev = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
out = {"flags": int(M.lib().moe_build_flags())}
for mode in (M.MOE_MODE_GEMV, M.MOE_MODE_GEMM):
    b = g.forward(xdev, M.MOE_BF16, mode=mode)
    torch.cuda.synchronize()
    clean = M.moe_device_error()
    bad = b.perm_src.clone()
    bad[3], bad[5] = T + 100, -7                      # two corrupt entries
    fixed = b.perm_src.clone()
    fixed[3], fixed[5] = 0, 0                          # what every build reads for them
    ys = []
    bits = []
    for ps in (bad, fixed):
        yp = torch.full_like(b.y_perm, float("nan"))
        M.moe_expert_ffn_q4(g.table, b.offsets, b.active, ps, xdev, M.MOE_BF16, T, k, H, I, E, g.shared, yp,
                            b.y_shared, mode, b.ws_ffn, b.sizes["ffn"])
        torch.cuda.synchronize()
        bits.append(M.moe_device_error())
        ys.append(yp[:T * k * H].clone())
    out[str(mode)] = {"clean": clean, "bits_bad": bits[0], "bits_fixed": bits[1],
                      "same": bool(torch.equal(ys[0], ys[1])), "finite": bool(torch.isfinite(ys[0]).all())}
print(json.dumps(out))
'''


def _run(variant):
    env = dict(os.environ, MOE_LIBRARY=variant)
    r = subprocess.run([sys.executable, "-c", SCRIPT], capture_output=True, text=True, env=env, cwd=ROOT,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("variant", ["debug", "release"])
def test_corrupt_permutation_entry(variant):
    import quantized_expert_ffn_route_b200 as M
    if variant == "debug":
        from quantized_expert_ffn_route_b200.build import build as build_lib
        build_lib(debug=True)
    d = _run(variant)
    assert d["flags"] == (M.MOE_BUILD_DEBUG if variant == "debug" else 0)
    for mode in (str(M.MOE_MODE_GEMV), str(M.MOE_MODE_GEMM)):
        r = d[mode]
        assert r["clean"] == 0 and r["bits_fixed"] == 0
        assert r["bits_bad"] == (M.DEVERR_BAD_ROW if variant == "debug" else 0), r
        assert r["same"] and r["finite"], r
