"""C-ABI checks that need no GPU: the library loads, exports every function
that include/moe.h declares, sizes workspaces, and rejects bad arguments on
the host before touching the device."""
import ctypes as C
import os
import re
import subprocess
import sys
from pathlib import Path

import numpy as np
import pytest

import quantized_expert_ffn_route_b200 as M

ROOT = Path(__file__).resolve().parents[1]


def _declared():
    src = M.HEADER.read_text()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b((?:moe|expcache|devcache|expstore)_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 20
    L = M.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", str(M.LIB_PATH)], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T ((?:moe|expcache|devcache|expstore)_\w+)$", out, flags=re.M))
    assert set(names) <= exported
    assert M.moe_version() == 100


def test_blob_and_workspace_sizes():
    assert M.moe_expert_blob_bytes(4, 2048, 512) == 1_769_472
    assert M.moe_expert_blob_bytes(2, 2048, 512) == 983_040
    assert M.moe_expert_blob_bytes(3, 2048, 512) == 0
    assert M.moe_route_ws_size(8, 512, 10) == 8 * 512 * 4
    assert M.moe_permute_ws_size(1, 10, 512) == 0            # one-block path needs no workspace
    assert M.moe_permute_ws_size(8192, 10, 512) > 0
    assert M.moe_expert_ffn_ws_size(4, 1, 10, 2048, 512, 512, M.MOE_MODE_GEMV) == 11 * 512 * 4
    assert M.moe_expert_ffn_ws_size(4, 0, 10, 2048, 512, 512, 0) == 0


def _rc(fn, *a):
    return getattr(M.lib(), fn)(*a)


def test_route_rejects_bad_arguments_on_host():
    buf = np.zeros(64, np.float32)
    p = buf.ctypes.data
    # k > E, k = 0, E too large, T negative
    assert _rc("moe_route_topk", p, 0, p, 0, None, None, 1, 8, 4, 5, p, p, None, p, 1024, None) == M.MOE_EINVAL
    assert "k must be" in M.moe_last_error()
    assert _rc("moe_route_topk", p, 0, p, 0, None, None, 1, 8, 4, 0, p, p, None, p, 1024, None) == M.MOE_EINVAL
    assert _rc("moe_route_topk", p, 0, p, 0, None, None, 1, 8, 40000, 4, p, p, None, p, 1024, None) == M.MOE_EINVAL
    assert _rc("moe_route_topk", p, 0, p, 0, None, None, -1, 8, 4, 2, p, p, None, p, 1024, None) == M.MOE_EINVAL
    # bad dtype, misaligned pointer, missing workspace, no logits source
    assert _rc("moe_route_topk", p, 7, p, 0, None, None, 1, 8, 4, 2, p, p, None, p, 1024, None) == M.MOE_EINVAL
    assert _rc("moe_route_topk", p + 4, 0, p, 0, None, None, 1, 8, 4, 2, p, p, None, p, 1024, None) == M.MOE_EINVAL
    assert _rc("moe_route_topk", p, 0, p, 0, None, None, 1, 8, 4, 2, p, p, None, p, 8, None) == M.MOE_EINVAL
    assert "workspace" in M.moe_last_error()
    assert _rc("moe_route_topk", None, 0, None, 0, None, None, 1, 8, 4, 2, p, p, None, None, 0, None) == M.MOE_EINVAL
    # T = 0 is a no-op
    assert _rc("moe_route_topk", None, 0, None, 0, None, None, 0, 8, 4, 2, None, None, None, None, 0, None) == 0


def test_permute_and_ffn_reject_bad_arguments_on_host():
    buf = np.zeros(1024, np.int32)
    p = buf.ctypes.data
    assert _rc("moe_permute", p, 1, 0, 16, p, p, p, p, None, 0, None) == M.MOE_EINVAL
    assert _rc("moe_permute", p, 1, 4, 0, p, p, p, p, None, 0, None) == M.MOE_EINVAL
    assert _rc("moe_permute", p, 1, 4, 16, p + 4, p, p, p, None, 0, None) == M.MOE_EINVAL
    assert _rc("moe_permute", p, 8192, 10, 512, p, p, p, p, None, 0, None) == M.MOE_EINVAL   # workspace
    f = M.lib().moe_expert_ffn_q4
    # H not a multiple of 128, I too large, bad mode, NULL pointers, missing workspace
    assert f(p, p, p, p, p, 1, 1, 2, 200, 512, 16, None, p, None, 0, p, 1 << 20, None) == M.MOE_EINVAL
    assert f(p, p, p, p, p, 1, 1, 2, 256, 8192, 16, None, p, None, 0, p, 1 << 20, None) == M.MOE_EINVAL
    assert f(p, p, p, p, p, 1, 1, 2, 256, 128, 16, None, p, None, 9, p, 1 << 20, None) == M.MOE_EINVAL
    assert f(None, p, p, p, p, 1, 1, 2, 256, 128, 16, None, p, None, 0, p, 1 << 20, None) == M.MOE_EINVAL
    assert f(p, p, p, p, p, 1, 1, 2, 256, 128, 16, None, p, None, 0, p, 16, None) == M.MOE_EINVAL
    assert f(p, p, p, p, p, 1, 1, 2, 256, 128, 16, p, p, None, 0, p, 1 << 20, None) == M.MOE_EINVAL  # y_shared
    assert _rc("moe_combine", p, p, p, None, 1, 0, 64, p, None) == M.MOE_EINVAL
    assert _rc("moe_combine", p, p, p, None, 1, 2, 62, p, None) == M.MOE_EINVAL


def test_expcache_rejects_bad_descriptors_on_host():
    pool = np.zeros(4096, np.uint8)
    d = M.ExpCacheDesc(4, 2, 256, 256, pool.ctypes.data, pool.ctypes.data, pool.ctypes.data, None, 8, 0)
    h = C.c_void_p()
    bad = [dict(n_experts=0), dict(capacity=0), dict(blob_bytes=100), dict(slot_stride=128),
           dict(host_pool=None), dict(decay_period=-1), dict(use_staging=1)]
    for b in bad:
        dd = M.ExpCacheDesc.from_buffer_copy(d)
        for k, v in b.items():
            setattr(dd, k, v)
        assert M.lib().expcache_create(C.byref(dd), C.byref(h)) == M.MOE_EINVAL, b
    assert M.lib().expcache_stage(None, None, 0, None, None, None, None) == M.MOE_EINVAL


def test_product_path_has_no_fallback(monkeypatch, tmp_path):
    """Without the shared library the binding raises instead of computing elsewhere."""
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", tmp_path / "missing.so")
    with pytest.raises(RuntimeError, match="libmoe.so not found"):
        M.lib()


def test_fused_decode_shape_checks_on_host():
    """Supported shapes pass host validation (they fail later only for lack of a GPU here)."""
    buf = np.zeros(4096, np.float32)
    p = buf.ctypes.data
    L = M.lib()
    for bits, H, I, E, k in [(4, 2048, 512, 512, 10), (2, 2048, 512, 512, 10), (4, 256, 256, 24, 4)]:
        rc = L.moe_layer_decode(bits, p, M.MOE_BF16, p, M.MOE_BF16, None, None, p, p, H, I, E, k, p, p, None, p,
                                p, M.moe_layer_decode_ws_size(E, k, I), None)
        assert rc != M.MOE_EINVAL, M.moe_last_error()
    # I/32 = 64 chunks per row (more than one per lane), H > 2048, E > 1024, too many groups
    for bits, H, I, E, k in [(4, 2048, 2048, 512, 10), (4, 4096, 512, 512, 10), (4, 2048, 512, 2048, 10),
                             (4, 2048, 1024, 512, 32)]:
        rc = L.moe_layer_decode(bits, p, M.MOE_BF16, p, M.MOE_BF16, None, None, p, p, H, I, E, k, p, p, None, p,
                                p, M.moe_layer_decode_ws_size(E, k, I), None)
        assert rc == M.MOE_EINVAL


def test_ffn_mode_shape_rules_on_host():
    """GEMV takes I/32 (4-bit) or I/64 (2-bit) in {2, 4, 8, 16, 32}; AUTO falls
    back to GEMM for other intermediates; GEMM takes at most 4095 groups."""
    buf = np.zeros(1 << 16, np.int32)
    p = buf.ctypes.data
    L = M.lib()
    gemm_ws = M.moe_expert_ffn_ws_size(4, 4, 2, 256, 384, 16, M.MOE_MODE_GEMM)
    gemv_ws = M.moe_expert_ffn_ws_size(4, 4, 2, 256, 384, 16, M.MOE_MODE_GEMV)
    assert M.moe_expert_ffn_ws_size(4, 4, 2, 256, 384, 16, M.MOE_MODE_AUTO) == gemm_ws != gemv_ws
    assert M.moe_expert_ffn_ws_size(4, 4, 2, 256, 512, 16, M.MOE_MODE_AUTO) == \
        M.moe_expert_ffn_ws_size(4, 4, 2, 256, 512, 16, M.MOE_MODE_GEMV)
    f = L.moe_expert_ffn_q4
    rc = f(p, p, p, p, p, 1, 4, 2, 256, 384, 16, None, p, None, M.MOE_MODE_GEMV, p, 1 << 20, None)
    assert rc == M.MOE_EINVAL and "GEMV mode" in M.moe_last_error()
    # 32768 experts and 4096 * 2 pairs: 4097 groups is one too many for GEMM
    rc = f(p, p, p, p, p, 1, 4096, 2, 256, 256, 32768, None, p, None, M.MOE_MODE_GEMM, p, 1 << 30, None)
    assert rc == M.MOE_EINVAL and "GEMM" in M.moe_last_error()
    # the allocation-free call takes the GEMV shapes only
    rc = L.moe_expert_ffn_noalloc(4, p, p, p, p, p, 1, 1, 2, 256, 2048, 16, None, p, None, None)
    assert rc == M.MOE_EINVAL and "I/32" in M.moe_last_error()


def test_test_hooks_validate_arguments():
    import quantized_expert_ffn_route_b200 as M
    L = M.lib()
    assert L.moe_test_hook(99, 1) == M.MOE_EINVAL
    assert L.moe_test_hook(M.MOE_HOOK_GEMM_SPIN, -1) == M.MOE_EINVAL
    for h in (M.MOE_HOOK_WAIT_LIMIT_NS, M.MOE_HOOK_DECODE_EXTRA_ARRIVALS, M.MOE_HOOK_GEMM_SPIN, M.MOE_HOOK_DECODE_ONE_KERNEL):
        assert L.moe_test_hook(h, 0) == M.MOE_OK


def test_debug_build_exports_every_symbol_and_reports_its_flag():
    """The MOE_DEBUG variant (build --debug) links the same ABI and says so."""
    from quantized_expert_ffn_route_b200.build import build as build_lib
    path = build_lib(debug=True)
    assert path.parent.name == "_build_debug"
    out = subprocess.run(["nm", "-D", "--defined-only", str(path)], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T ((?:moe|expcache|devcache|expstore)_\w+)$", out, flags=re.M))
    assert set(_declared()) <= exported
    code = ("import quantized_expert_ffn_route_b200 as M; "
            "print(M.LIB_PATH.parent.name, M.lib().moe_build_flags(), M.MOE_BUILD_DEBUG)")
    for variant, want in (("debug", "_build_debug 1 1"), ("release", "_build 0 1")):
        env = dict(os.environ, MOE_LIBRARY=variant)
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT)
        assert r.returncode == 0, r.stderr
        assert r.stdout.split() == want.split()


def test_devcache_rejects_bad_descriptors_on_the_host():
    h = C.c_void_p()
    L = M.lib()
    assert L.devcache_create(None, C.byref(h)) == M.MOE_EINVAL
    buf = np.zeros(4096, np.uint8)
    p = buf.ctypes.data
    bad = [
        M.DevCacheDesc(10, 11, 1024, 1024, p, p, p, 0, 0, 0),      # capacity > n_experts
        M.DevCacheDesc(10, 4, 1000, 1024, p, p, p, 0, 0, 0),       # blob_bytes not a multiple of 16
        M.DevCacheDesc(10, 4, 1024, 1000, p, p, p, 0, 0, 0),       # stride not a multiple of 256
        M.DevCacheDesc(10, 4, 1024, 1024, None, p, p, 0, 0, 0),    # no pool
        M.DevCacheDesc(10, 4, 1024, 1024, p, p, p, -1, 0, 0),      # negative decay
    ]
    for d in bad:
        assert L.devcache_create(C.byref(d), C.byref(h)) == M.MOE_EINVAL
        assert h.value is None
    assert L.devcache_stage(None, None, 0, 0, None, None, None) == M.MOE_EINVAL
    assert L.devcache_join(None, None) == M.MOE_EINVAL


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_header_compiles_as_c_and_cpp(lang):
    """include/moe.h is a plain C header (extern "C" in C++)."""
    r = subprocess.run(["gcc" if lang == "c" else "g++", "-fsyntax-only", "-Wall", "-Werror", "-x", lang,
                        str(M.HEADER)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
