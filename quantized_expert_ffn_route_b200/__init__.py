"""Python binding of libmoe, the B200 quantized MoE expert step.

Argument marshalling only: every function below forwards to the C ABI
declared in include/moe.h with the same name; all arithmetic runs in the
CUDA kernels of libmoe.so.  There is no CPU fallback: if the shared library
is missing, the first call raises.

Device buffers are passed as torch CUDA tensors (or raw integer pointers);
torch is used only for device memory and streams.
"""
from __future__ import annotations

import ctypes as C
import os
from pathlib import Path

from .layer import MoELayer, alloc_step_buffers  # noqa: F401

_PKG = Path(__file__).resolve().parent
# MOE_LIBRARY=debug loads the MOE_DEBUG build (index checks report to the
# device error word); the default is the release build.
LIB_PATH = _PKG / ("_build_debug" if os.environ.get("MOE_LIBRARY") == "debug" else "_build") / "libmoe.so"
MOE_BUILD_DEBUG = 1
HEADER = _PKG.parent / "include" / "moe.h"

MOE_OK, MOE_EINVAL, MOE_ENOMEM, MOE_ECUDA, MOE_EBUSY, MOE_ETIMEDOUT, MOE_EIO, MOE_EDEVICE = range(8)
MOE_F32, MOE_BF16 = 0, 1
MOE_MODE_AUTO, MOE_MODE_GEMV, MOE_MODE_GEMM = 0, 1, 2
DEVERR_BAD_EXPERT, DEVERR_NULL_BLOB, DEVERR_NONFINITE, DEVERR_BAD_ROW = 1, 2, 4, 8
MOE_DEVERR_TIMEOUT = 16
DEVERR_MISALIGNED = 32
MOE_HOOK_WAIT_LIMIT_NS, MOE_HOOK_DECODE_EXTRA_ARRIVALS, MOE_HOOK_GEMM_SPIN, MOE_HOOK_DECODE_ONE_KERNEL = 1, 2, 3, 4

_STATUS = {1: "MOE_EINVAL", 2: "MOE_ENOMEM", 3: "MOE_ECUDA", 4: "MOE_EBUSY", 5: "MOE_ETIMEDOUT",
           6: "MOE_EIO", 7: "MOE_EDEVICE"}


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class ExpCacheDesc(C.Structure):
    _fields_ = [("n_experts", C.c_int32), ("capacity", C.c_int32), ("blob_bytes", C.c_int64),
                ("slot_stride", C.c_int64), ("host_pool", C.c_void_p), ("hbm_slab", C.c_void_p),
                ("dev_table", C.c_void_p), ("stage_buffer", C.c_void_p), ("decay_period", C.c_int32),
                ("use_staging", C.c_int32)]


class ExpCacheStats(C.Structure):
    _fields_ = [("steps", C.c_int64), ("hits", C.c_int64), ("misses", C.c_int64),
                ("evictions", C.c_int64), ("bytes_staged", C.c_int64), ("resident", C.c_int32),
                ("prefetched", C.c_int64)]


class DevCacheDesc(C.Structure):
    _fields_ = [("n_experts", C.c_int32), ("capacity", C.c_int32), ("blob_bytes", C.c_int64),
                ("slot_stride", C.c_int64), ("host_pool", C.c_void_p), ("hbm_slab", C.c_void_p),
                ("dev_table", C.c_void_p), ("decay_period", C.c_int32), ("admit_min", C.c_int32),
                ("log_steps", C.c_int32)]


class DevCacheStats(C.Structure):
    _fields_ = [("steps", C.c_int64), ("hits", C.c_int64), ("misses", C.c_int64), ("evictions", C.c_int64),
                ("in_place", C.c_int64), ("bytes_copied", C.c_int64), ("bad_steps", C.c_int64)]


class ExpStoreDesc(C.Structure):
    _fields_ = [("path", C.c_char_p), ("n_experts", C.c_int32), ("blob_bytes", C.c_int64),
                ("slot_stride", C.c_int64), ("ram_slots", C.c_int32), ("ram_buffer", C.c_void_p),
                ("io_threads", C.c_int32), ("use_direct", C.c_int32)]


class ExpStoreStats(C.Structure):
    _fields_ = [("fetches", C.c_int64), ("hits", C.c_int64), ("reads", C.c_int64), ("bytes_read", C.c_int64),
                ("evictions", C.c_int64), ("read_seconds", C.c_double)]


MOE_COPY_HIST_BINS = 24
DEVCACHE_ACT_INTS = 66          # two active-expert lists: [0] n_a, [1..32] ids; [33] n_b, [34..65] ids
DEVCACHE_HIT, DEVCACHE_MISS, DEVCACHE_IN_PLACE = 1, 0, 3

_lib = None


def lib():
    """Loads libmoe.so (built in-tree by build()); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"libmoe.so not found at {LIB_PATH}; build it with "
                           "`python -m quantized_expert_ffn_route_b200.build`")
    import torch  # noqa: F401  (loads the CUDA runtime libmoe shares with torch)
    L = C.CDLL(str(LIB_PATH))
    P, I, Z, S = C.c_void_p, C.c_int, C.c_size_t, C.c_void_p
    sig = {
        "moe_last_error": (C.c_char_p, []),
        "moe_version": (I, []),
        "moe_build_flags": (I, []),
        "moe_test_hook": (I, [I, C.c_int64]),
        "moe_kernel_launches": (C.c_uint64, []),
        "moe_device_error": (I, [P, I, S]),
        "moe_expert_blob_bytes": (Z, [I, I, I]),
        "moe_route_ws_size": (Z, [I, I, I]),
        "moe_route_topk": (I, [P, I, P, I, P, P, I, I, I, I, P, P, P, P, Z, S]),
        "moe_permute_ws_size": (Z, [I, I, I]),
        "moe_permute": (I, [P, I, I, I, P, P, P, P, P, Z, S]),
        "moe_expert_ffn_ws_size": (Z, [I, I, I, I, I, I, I]),
        "moe_expert_ffn_q4": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, I, P, Z, S]),
        "moe_expert_ffn_q2": (I, [P, P, P, P, P, I, I, I, I, I, I, P, P, P, I, P, Z, S]),
        "moe_combine": (I, [P, P, P, P, I, I, I, P, S]),
        "moe_layer_decode_ws_size": (Z, [I, I, I]),
        "moe_layer_decode": (I, [I, P, I, P, I, P, P, P, P, I, I, I, I, P, P, P, P, P, Z, S]),
        "moe_expert_ffn_noalloc_max_bytes": (Z, []),
        "moe_expert_ffn_noalloc": (I, [I, P, P, P, P, P, I, I, I, I, I, I, P, P, P, S]),
        "expcache_create": (I, [C.POINTER(ExpCacheDesc), C.POINTER(P)]),
        "expcache_destroy": (None, [P]),
        "expcache_lookup": (I, [P, P, I, P, P]),
        "expcache_stage": (I, [P, P, I, S, P, P, P]),
        "expcache_join": (I, [P, S]),
        "expcache_wait": (I, [P, C.c_int64]),
        "expcache_evict": (I, [P, P, I]),
        "expcache_device_table": (P, [P]),
        "expcache_stats": (I, [P, C.POINTER(ExpCacheStats)]),
        "expcache_snapshot": (I, [P, P, P]),
        "expcache_inject_copy_failures": (I, [P, I]),
        "expcache_copy_times": (I, [P, P, C.POINTER(C.c_float), C.POINTER(C.c_float)]),
        "expcache_prefetch": (I, [P, P, I, S, P, P, C.POINTER(C.c_int)]),
        "expcache_stage_from": (I, [P, P, I, P, S, P, P, P]),
        "expcache_copy_histogram": (I, [P, P, P]),
        "expstore_create": (I, [C.POINTER(ExpStoreDesc), C.POINTER(P)]),
        "expstore_destroy": (None, [P]),
        "expstore_fetch": (I, [P, P, I, P, P]),
        "expstore_stats": (I, [P, C.POINTER(ExpStoreStats)]),
        "expstore_snapshot": (I, [P, P]),
        "moe_decode_session_create": (I, [I, P, I, P, I, P, P, P, I, I, I, I, P, P, P, P, P, P, P, Z, S,
                                          C.POINTER(P)]),
        "moe_decode_session_run": (I, [P]),
        "moe_decode_session_destroy": (None, [P]),
        "devcache_create": (I, [C.POINTER(DevCacheDesc), C.POINTER(P)]),
        "devcache_destroy": (None, [P]),
        "devcache_stage": (I, [P, P, I, C.c_int32, P, S, S]),
        "devcache_join": (I, [P, S]),
        "devcache_events": (I, [P, C.c_int64, I, P, P, P]),
        "devcache_stats": (I, [P, C.POINTER(DevCacheStats)]),
        "devcache_snapshot": (I, [P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _p(t):
    """Pointer of a tensor / numpy array / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):
        return t.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(t)}")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int):
    if rc != MOE_OK:
        raise MoEError(rc, lib().moe_last_error().decode())
    return rc


# ----------------------------------------------------------------- the ABI
def moe_version() -> int:
    return lib().moe_version()


def moe_test_hook(which: int, value: int) -> None:
    """Sets a test hook (MOE_HOOK_*); 0 restores the default."""
    _check(lib().moe_test_hook(which, int(value)))


def moe_kernel_launches() -> int:
    return lib().moe_kernel_launches()


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_device_error(clear: bool = True, stream=None) -> int:
    """Returns the device error bits (0 if none); raises only on CUDA failure."""
    bits = C.c_uint32(0)
    rc = lib().moe_device_error(C.byref(bits), int(clear), _stream(stream))
    if rc not in (MOE_OK, MOE_EDEVICE):
        _check(rc)
    return bits.value


def moe_expert_blob_bytes(bits: int, H: int, I: int) -> int:
    return lib().moe_expert_blob_bytes(bits, H, I)


def moe_route_ws_size(T, E, k):
    return lib().moe_route_ws_size(T, E, k)


def moe_route_topk(x, x_dtype, w_router, w_dtype, logits_in, bias, T, H, E, k, topk_ids, topk_w,
                   logits_out=None, ws=None, ws_bytes=0, stream=None):
    return _check(lib().moe_route_topk(_p(x), x_dtype, _p(w_router), w_dtype, _p(logits_in), _p(bias), T, H, E,
                                       k, _p(topk_ids), _p(topk_w), _p(logits_out), _p(ws), ws_bytes,
                                       _stream(stream)))


def moe_permute_ws_size(T, k, E):
    return lib().moe_permute_ws_size(T, k, E)


def moe_permute(topk_ids, T, k, E, expert_offsets, perm_src, perm_dst, active=None, ws=None, ws_bytes=0,
                stream=None):
    return _check(lib().moe_permute(_p(topk_ids), T, k, E, _p(expert_offsets), _p(perm_src), _p(perm_dst),
                                    _p(active), _p(ws), ws_bytes, _stream(stream)))


def moe_expert_ffn_ws_size(bits, T, k, H, I, E, mode=MOE_MODE_AUTO):
    return lib().moe_expert_ffn_ws_size(bits, T, k, H, I, E, mode)


def _ffn(name, expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob, y_perm,
         y_shared, mode, ws, ws_bytes, stream):
    f = getattr(lib(), name)
    return _check(f(_p(expert_blobs), _p(expert_offsets), _p(active), _p(perm_src), _p(x), x_dtype, T, k, H, I, E,
                    _p(shared_blob), _p(y_perm), _p(y_shared), mode, _p(ws), ws_bytes, _stream(stream)))


def moe_expert_ffn_q4(expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob,
                      y_perm, y_shared, mode=MOE_MODE_AUTO, ws=None, ws_bytes=0, stream=None):
    return _ffn("moe_expert_ffn_q4", expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E,
                shared_blob, y_perm, y_shared, mode, ws, ws_bytes, stream)


def moe_expert_ffn_q2(expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob,
                      y_perm, y_shared, mode=MOE_MODE_AUTO, ws=None, ws_bytes=0, stream=None):
    return _ffn("moe_expert_ffn_q2", expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E,
                shared_blob, y_perm, y_shared, mode, ws, ws_bytes, stream)


def moe_layer_decode_ws_size(E, k, I):
    return lib().moe_layer_decode_ws_size(E, k, I)


def moe_layer_decode(bits, x, x_dtype, w_router, w_dtype, bias, logits_in, expert_blobs, shared_blob, H, I, E, k,
                     topk_ids, topk_w, logits_out, y, ws, ws_bytes, stream=None):
    return _check(lib().moe_layer_decode(bits, _p(x), x_dtype, _p(w_router), w_dtype, _p(bias), _p(logits_in),
                                         _p(expert_blobs), _p(shared_blob), H, I, E, k, _p(topk_ids), _p(topk_w),
                                         _p(logits_out), _p(y), _p(ws), ws_bytes, _stream(stream)))


def moe_expert_ffn_noalloc_max_bytes() -> int:
    return lib().moe_expert_ffn_noalloc_max_bytes()


def moe_expert_ffn_noalloc(bits, expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E,
                           shared_blob, y_perm, y_shared, stream=None):
    return _check(lib().moe_expert_ffn_noalloc(bits, _p(expert_blobs), _p(expert_offsets), _p(active),
                                               _p(perm_src), _p(x), x_dtype, T, k, H, I, E, _p(shared_blob),
                                               _p(y_perm), _p(y_shared), _stream(stream)))


def moe_combine(y_perm, perm_dst, topk_w, y_shared, T, k, H, y, stream=None):
    return _check(lib().moe_combine(_p(y_perm), _p(perm_dst), _p(topk_w), _p(y_shared), T, k, H, _p(y),
                                    _stream(stream)))


class ExpCache:
    """Handle around the expcache_* calls (the caller owns pool, slab and table)."""

    def __init__(self, n_experts, capacity, blob_bytes, slot_stride, host_pool, hbm_slab, dev_table,
                 decay_period=256, stage_buffer=None):
        d = ExpCacheDesc(n_experts, capacity, blob_bytes, slot_stride, _p(host_pool), _p(hbm_slab),
                         _p(dev_table), _p(stage_buffer), decay_period, 1 if stage_buffer is not None else 0)
        h = C.c_void_p()
        _check(lib().expcache_create(C.byref(d), C.byref(h)))
        self.h = h
        self.n_experts = n_experts

    def close(self):
        if self.h:
            lib().expcache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def lookup(self, ids):
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        slots = np.empty(ids.size, np.int32)
        nm = C.c_int(0)
        _check(lib().expcache_lookup(self.h, _p(ids), ids.size, _p(slots), C.byref(nm)))
        return slots, nm.value

    def stage(self, ids, stream=None):
        """One step; returns (hit, slot, victim) numpy arrays."""
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        hit = np.empty(ids.size, np.int32)
        slot = np.empty(ids.size, np.int32)
        victim = np.empty(ids.size, np.int32)
        _check(lib().expcache_stage(self.h, _p(ids), ids.size, _stream(stream), _p(hit), _p(slot), _p(victim)))
        return hit, slot, victim

    def stage_from(self, ids, srcs, stream=None):
        """stage() with the misses copied from the given page-locked host
        addresses (srcs[i] for ids[i]; 0 for hits); returns (hit, slot, victim)."""
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        src = np.ascontiguousarray(srcs, dtype=np.uint64)
        hit = np.empty(ids.size, np.int32)
        slot = np.empty(ids.size, np.int32)
        victim = np.empty(ids.size, np.int32)
        _check(lib().expcache_stage_from(self.h, _p(ids), ids.size, _p(src), _stream(stream), _p(hit), _p(slot),
                                         _p(victim)))
        return hit, slot, victim

    def prefetch(self, ids, stream=None):
        """Loads the given experts (-1 = none) without a use; returns (slot, victim, admitted)."""
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        slot = np.empty(ids.size, np.int32)
        victim = np.empty(ids.size, np.int32)
        adm = C.c_int(0)
        _check(lib().expcache_prefetch(self.h, _p(ids), ids.size, _stream(stream), _p(slot), _p(victim),
                                       C.byref(adm)))
        return slot, victim, adm.value

    def join(self, stream=None):
        _check(lib().expcache_join(self.h, _stream(stream)))

    def wait(self, timeout_us: int):
        return lib().expcache_wait(self.h, int(timeout_us))

    def evict(self, ids):
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        _check(lib().expcache_evict(self.h, _p(ids), ids.size))

    def device_table(self) -> int:
        return lib().expcache_device_table(self.h)

    def stats(self) -> dict:
        s = ExpCacheStats()
        _check(lib().expcache_stats(self.h, C.byref(s)))
        return {f: getattr(s, f) for f, _ in ExpCacheStats._fields_}

    def snapshot(self):
        import numpy as np
        cnt = np.empty(self.n_experts, np.int64)
        slot = np.empty(self.n_experts, np.int32)
        _check(lib().expcache_snapshot(self.h, _p(cnt), _p(slot)))
        return cnt, slot

    def inject_copy_failures(self, n: int):
        _check(lib().expcache_inject_copy_failures(self.h, n))

    def copy_histogram(self):
        """(bins int64 [MOE_COPY_HIST_BINS], steps): bin i counts the steps whose
        copies took [2^i, 2^(i+1)) microseconds."""
        import numpy as np
        bins = np.zeros(MOE_COPY_HIST_BINS, np.int64)
        n = C.c_int64(0)
        _check(lib().expcache_copy_histogram(self.h, _p(bins), C.byref(n)))
        return bins, n.value

    def copy_times(self, ref_event):
        """(start_ms, end_ms) of the last step's copies, measured from `ref_event`
        (a torch.cuda.Event with timing, recorded earlier and completed)."""
        a, b = C.c_float(0.0), C.c_float(0.0)
        _check(lib().expcache_copy_times(self.h, C.c_void_p(ref_event.cuda_event), C.byref(a), C.byref(b)))
        return a.value, b.value


class DevCache:
    """Handle around the devcache_* calls (device-initiated staging; the caller
    owns pool, slab and table).  The pool must be page-locked and mapped
    (torch's pin_memory() is)."""

    def __init__(self, n_experts, capacity, blob_bytes, slot_stride, host_pool, hbm_slab, dev_table,
                 decay_period=256, admit_min=0, log_steps=0):
        d = DevCacheDesc(n_experts, capacity, blob_bytes, slot_stride, _p(host_pool), _p(hbm_slab), _p(dev_table),
                         decay_period, admit_min, log_steps)
        h = C.c_void_p()
        _check(lib().devcache_create(C.byref(d), C.byref(h)))
        self.h = h
        self.n_experts = n_experts

    def close(self):
        if self.h:
            lib().devcache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def stage(self, ids_dev, n, act_dev, id_base=0, stream=None, copy_stream=None):
        """One step from device ids; act_dev: device int32 [66] (DEVCACHE_ACT_INTS)."""
        s = _stream(stream)
        _check(lib().devcache_stage(self.h, _p(ids_dev), int(n), int(id_base), _p(act_dev), s,
                                    s if copy_stream is None else _stream(copy_stream)))

    def join(self, stream=None):
        _check(lib().devcache_join(self.h, _stream(stream)))

    def events(self, first_step, n_steps):
        """(hit, slot, victim) numpy arrays [n_steps, 32] of logged steps."""
        import numpy as np
        hit = np.zeros((n_steps, 32), np.int8)
        slot = np.zeros((n_steps, 32), np.int32)
        victim = np.zeros((n_steps, 32), np.int32)
        _check(lib().devcache_events(self.h, int(first_step), int(n_steps), _p(hit), _p(slot), _p(victim)))
        return hit, slot, victim

    def stats(self) -> dict:
        st = DevCacheStats()
        _check(lib().devcache_stats(self.h, C.byref(st)))
        return {f: getattr(st, f) for f, _ in DevCacheStats._fields_}

    def snapshot(self):
        import numpy as np
        cnt = np.empty(self.n_experts, np.int64)
        slot = np.empty(self.n_experts, np.int32)
        _check(lib().devcache_snapshot(self.h, _p(cnt), _p(slot)))
        return cnt, slot


class ExpStore:
    """Handle around the expstore_* calls: expert blobs in a file, read on
    demand into a RAM tier (the caller owns the page-locked ram_buffer)."""

    def __init__(self, path, n_experts, blob_bytes, slot_stride, ram_slots, ram_buffer, io_threads=8,
                 use_direct=False):
        d = ExpStoreDesc(str(path).encode(), n_experts, blob_bytes, slot_stride, ram_slots, _p(ram_buffer),
                         io_threads, 1 if use_direct else 0)
        h = C.c_void_p()
        _check(lib().expstore_create(C.byref(d), C.byref(h)))
        self.h = h
        self.n_experts = n_experts

    def close(self):
        if self.h:
            lib().expstore_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def fetch(self, ids):
        """Makes the experts resident in RAM; returns (addresses uint64, hit int8)."""
        import numpy as np
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        ptrs = np.zeros(ids.size, np.uint64)
        hit = np.zeros(ids.size, np.int8)
        _check(lib().expstore_fetch(self.h, _p(ids), ids.size, _p(ptrs), _p(hit)))
        return ptrs, hit

    def stats(self) -> dict:
        st = ExpStoreStats()
        _check(lib().expstore_stats(self.h, C.byref(st)))
        return {f: getattr(st, f) for f, _ in ExpStoreStats._fields_}

    def snapshot(self):
        import numpy as np
        slot = np.empty(self.n_experts, np.int32)
        _check(lib().expstore_snapshot(self.h, _p(slot)))
        return slot
