"""fp64 CPU oracle for the quantized MoE expert step (ctypes wrapper).

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline leg use this package.  The product library never imports it.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, one
OpenMP loop over independent expert rows).  This wrapper only moves numpy
arrays in and out.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "moe_oracle.c"
_LIB_PATH = _HERE / "_build" / "liboracle.so"
_lib = None

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16}


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc -O2 -fopenmp (no fast-math)."""
    _LIB_PATH.parent.mkdir(parents=True, exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp")
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(str(build()))
        P, I32, U16 = C.c_void_p, C.c_int, C.c_uint16
        _lib.oracle_fp16_to_double.restype = C.c_double
        _lib.oracle_fp16_to_double.argtypes = [U16]
        _lib.oracle_bf16_to_double.restype = C.c_double
        _lib.oracle_bf16_to_double.argtypes = [U16]
        _lib.oracle_dequant_block.argtypes = [I32, P, U16, P]
        _lib.oracle_blob_bytes.restype = C.c_size_t
        _lib.oracle_blob_bytes.argtypes = [I32, I32, I32]
        _lib.oracle_expert_weights.argtypes = [I32, I32, I32, P, P, P, P]
        _lib.oracle_expert_ffn.argtypes = [I32, I32, I32, P, P, P, P]
        _lib.oracle_expert_ffn_rows.argtypes = [I32, I32, I32, I32, P, P, P]
        _lib.oracle_router_logits.argtypes = [I32, I32, I32, P, I32, P, I32, P, P]
        _lib.oracle_topk.restype = I32
        _lib.oracle_topk.argtypes = [I32, I32, I32, P, P, P]
        _lib.oracle_topk_f32.restype = I32
        _lib.oracle_topk_f32.argtypes = [I32, I32, I32, P, P, P]
        _lib.oracle_permute.restype = I32
        _lib.oracle_permute.argtypes = [I32, I32, I32, P, P, P, P, P]
        _lib.oracle_moe_layer.restype = I32
        _lib.oracle_moe_layer.argtypes = [I32, I32, I32, I32, I32, I32, P, I32, P, I32, P, P,
                                          P, P, P, P, P, P, P, P, P, P, P]
        _lib.oracle_combine.argtypes = [I32, I32, I32, P, P, P, P, P]
        _lib.oracle_cache_sim.restype = C.c_long
        _lib.oracle_cache_sim.argtypes = [I32, I32, I32, I32, I32, P, P, P, P, P]
        _lib.oracle_cache_sim_admit.restype = C.c_long
        _lib.oracle_cache_sim_admit.argtypes = [I32, I32, I32, I32, I32, I32, P, P, P, P, P]
        _lib.oracle_cache_sim_prefetch.restype = C.c_long
        _lib.oracle_cache_sim_prefetch.argtypes = [I32, I32, I32, I32, I32, P, I32, P, P, P, P, P, P, P, P]
        _lib.oracle_set_threads.argtypes = [I32]
        _lib.oracle_max_threads.restype = I32
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    """OpenMP thread count for the oracle's later calls."""
    os.environ["OMP_NUM_THREADS"] = str(n)
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    """The thread count the oracle's parallel loops use now."""
    return int(lib().oracle_max_threads())


# ------------------------------------------------------------------ formats
def fp16_to_double(bits: int) -> float:
    return lib().oracle_fp16_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def dequant_block(bits: int, codes: np.ndarray, scale_bits: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    assert codes.size == 4 * bits
    out = np.empty(32, np.float64)
    lib().oracle_dequant_block(bits, _p(codes), int(scale_bits), _p(out))
    return out


def blob_bytes(bits: int, H: int, I: int) -> int:
    return int(lib().oracle_blob_bytes(bits, H, I))


def expert_weights(bits: int, H: int, I: int, blob: np.ndarray):
    blob = _c(blob, np.uint8)
    Wg = np.empty((I, H)); Wu = np.empty((I, H)); Wd = np.empty((H, I))
    lib().oracle_expert_weights(bits, H, I, _p(blob), _p(Wg), _p(Wu), _p(Wd))
    return Wg, Wu, Wd


def expert_ffn(bits: int, H: int, I: int, blob: np.ndarray, x: np.ndarray):
    """One token through one expert: returns (y [H], h [I])."""
    blob = _c(blob, np.uint8)
    x = _c(x, np.float64)
    y = np.empty(H); h = np.empty(I)
    lib().oracle_expert_ffn(bits, H, I, _p(blob), _p(x), _p(y), _p(h))
    return y, h


def expert_ffn_rows(bits: int, H: int, I: int, blobs, xs):
    """Many independent (expert blob, token) pairs: y [n, H], row i = the FFN
    of blobs[i] applied to xs[i] (fp64 rows)."""
    blob_list = [np.ascontiguousarray(b, dtype=np.uint8) for b in blobs]
    xs = _c(xs, np.float64)
    n = len(blob_list)
    assert xs.shape == (n, H)
    ptrs = (C.c_void_p * max(1, n))(*[b.ctypes.data for b in blob_list])
    y = np.empty((n, H))
    lib().oracle_expert_ffn_rows(bits, H, I, n, C.cast(ptrs, C.c_void_p), _p(xs), _p(y))
    return y


# ------------------------------------------------------------------- router
def _xarr(x, dtype):
    return _c(x, np.uint16 if dtype == "bf16" else np.float32)


def router_logits(x, x_dtype, w_router, w_dtype, bias=None):
    x = _xarr(x, x_dtype); wr = _xarr(w_router, w_dtype)
    T, H = x.shape; E = wr.shape[0]
    out = np.empty((T, E))
    b = None if bias is None else _c(bias, np.float32)
    lib().oracle_router_logits(T, H, E, _p(x), _DT[x_dtype], _p(wr), _DT[w_dtype], _p(b), _p(out))
    return out


def topk(logits: np.ndarray, k: int):
    """Returns (ids int32 [T,k], w float64 [T,k], status)."""
    T, E = logits.shape
    ids = np.empty((T, k), np.int32); w = np.empty((T, k))
    if logits.dtype == np.float32:
        st = lib().oracle_topk_f32(T, E, k, _p(_c(logits, np.float32)), _p(ids), _p(w))
    else:
        st = lib().oracle_topk(T, E, k, _p(_c(logits, np.float64)), _p(ids), _p(w))
    return ids, w, st


def permute(ids: np.ndarray, E: int):
    """Returns dict(offsets, perm_src, perm_dst, active) or raises on a bad id."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, np.int32)
    perm_src = np.empty(T * k, np.int32)
    perm_dst = np.empty(T * k, np.int32)
    active = np.empty(E + 1, np.int32)
    st = lib().oracle_permute(T, k, E, _p(ids), _p(offsets), _p(perm_src), _p(perm_dst), _p(active))
    if st != 0:
        raise ValueError("expert id out of range")
    return dict(offsets=offsets, perm_src=perm_src, perm_dst=perm_dst.reshape(T, k),
                active=active[: 1 + active[0]])


# -------------------------------------------------------------------- layer
def moe_layer(bits, x, x_dtype, blobs, *, k, H, I, E, w_router=None, w_dtype="bf16",
              bias=None, logits_in=None, shared_blob=None, want_yperm=False):
    """The whole step in fp64.  blobs: uint8 [E, nbytes] array or a list of E arrays."""
    x = _xarr(x, x_dtype)
    T = x.shape[0]
    if isinstance(blobs, np.ndarray) and blobs.ndim == 2:
        blob_list = [blobs[e] for e in range(E)]
    else:
        blob_list = [np.ascontiguousarray(b, dtype=np.uint8) for b in blobs]
    ptrs = (C.c_void_p * E)(*[b.ctypes.data for b in blob_list])
    wr = None if w_router is None else _xarr(w_router, w_dtype)
    b = None if bias is None else _c(bias, np.float32)
    li = None if logits_in is None else _c(logits_in, np.float32)
    sh = None if shared_blob is None else _c(shared_blob, np.uint8)
    logits = np.empty((T, E)); ids = np.empty((T, k), np.int32); w = np.empty((T, k))
    offsets = np.empty(E + 1, np.int32); ps = np.empty(T * k, np.int32); pd = np.empty(T * k, np.int32)
    yp = np.empty((T * k, H)) if want_yperm else None
    ys = np.empty((T, H)) if sh is not None else None
    y = np.empty((T, H))
    st = lib().oracle_moe_layer(bits, T, H, I, E, k, _p(x), _DT[x_dtype], _p(wr), _DT[w_dtype],
                                _p(b), _p(li), C.cast(ptrs, C.c_void_p), _p(sh), _p(logits),
                                _p(ids), _p(w), _p(offsets), _p(ps), _p(pd), _p(yp), _p(ys), _p(y))
    return dict(status=st, logits=logits, ids=ids, w=w, offsets=offsets, perm_src=ps,
                perm_dst=pd.reshape(T, k), y_perm=yp, y_shared=ys, y=y)


def combine(y_perm, perm_dst, w, y_shared=None):
    T, k = perm_dst.shape
    H = y_perm.shape[1]
    y = np.empty((T, H))
    ys = None if y_shared is None else _c(y_shared, np.float64)
    lib().oracle_combine(T, k, H, _p(_c(y_perm, np.float64)), _p(_c(perm_dst, np.int32)),
                         _p(_c(w, np.float64)), _p(ys), _p(y))
    return y


# -------------------------------------------------------------------- cache
def cache_sim(ids: np.ndarray, n_experts: int, capacity: int, decay_period: int):
    """ids [steps, n] -> dict(slot, hit, victim, misses, counts)."""
    ids = _c(ids, np.int32)
    steps, n = ids.shape
    slot = np.empty((steps, n), np.int32); hit = np.empty((steps, n), np.int8)
    victim = np.empty((steps, n), np.int32); counts = np.empty(n_experts, np.int64)
    m = lib().oracle_cache_sim(n_experts, capacity, decay_period, steps, n, _p(ids), _p(slot),
                               _p(hit), _p(victim), _p(counts))
    if m < 0:
        raise ValueError("invalid cache trace")
    return dict(slot=slot, hit=hit.astype(bool), victim=victim, misses=int(m), counts=counts)


def cache_sim_admit(ids: np.ndarray, n_experts: int, capacity: int, decay_period: int, admit_min: int):
    """cache_sim with the admission threshold: ids [steps, n] -> dict(slot,
    hit (int8: 1 hit, 0 admitted miss, 3 computed in place), victim, misses,
    in_place, counts)."""
    ids = _c(ids, np.int32)
    steps, n = ids.shape
    slot = np.empty((steps, n), np.int32); hit = np.empty((steps, n), np.int8)
    victim = np.empty((steps, n), np.int32); counts = np.empty(n_experts, np.int64)
    m = lib().oracle_cache_sim_admit(n_experts, capacity, decay_period, admit_min, steps, n, _p(ids), _p(slot),
                                     _p(hit), _p(victim), _p(counts))
    if m < 0:
        raise ValueError("invalid cache trace")
    return dict(slot=slot, hit=hit, victim=victim, misses=int(m), in_place=int((hit == 3).sum()), counts=counts)


def cache_sim_prefetch(ids: np.ndarray, pf_ids: np.ndarray, n_experts: int, capacity: int, decay_period: int):
    """ids [steps, n], pf_ids [steps, npf] (-1 = none, prefetched after each
    step's stage) -> dict(slot, hit, victim, pf_slot, pf_victim, misses,
    prefetched, counts)."""
    ids = _c(ids, np.int32)
    pf_ids = _c(pf_ids, np.int32)
    steps, n = ids.shape
    npf = pf_ids.shape[1] if pf_ids.ndim == 2 else 0
    assert pf_ids.shape[0] == steps
    slot = np.empty((steps, n), np.int32); hit = np.empty((steps, n), np.int8)
    victim = np.empty((steps, n), np.int32)
    pf_slot = np.empty((steps, max(1, npf)), np.int32); pf_victim = np.empty((steps, max(1, npf)), np.int32)
    counts = np.empty(n_experts, np.int64)
    adm = C.c_long(0)
    m = lib().oracle_cache_sim_prefetch(n_experts, capacity, decay_period, steps, n, _p(ids), npf, _p(pf_ids),
                                        _p(slot), _p(hit), _p(victim), _p(pf_slot), _p(pf_victim), _p(counts),
                                        C.byref(adm))
    if m < 0:
        raise ValueError("invalid cache trace")
    return dict(slot=slot, hit=hit.astype(bool), victim=victim, pf_slot=pf_slot[:, :npf], pf_victim=pf_victim[:, :npf],
                misses=int(m), prefetched=int(adm.value), counts=counts)
