"""The NVMe tier (expstore_*) on the host: blobs read from a file into the RAM
tier land byte for byte, the RAM tier evicts the least recently fetched slot
that the call does not use (checked against a list model of that rule), and
bad calls are rejected before anything changes.  No GPU is needed."""
import ctypes as C
import os

import numpy as np
import pytest

import quantized_expert_ffn_route_b200 as M

N, BLOB, STRIDE, SLOTS = 40, 4000, 4096, 8


def _aligned(nbytes, align=4096):
    raw = np.empty(nbytes + align, np.uint8)
    off = (-raw.ctypes.data) % align
    return raw[off:off + nbytes]


@pytest.fixture
def blob_file(tmp_path):
    rng = np.random.default_rng(11)
    data = rng.integers(0, 256, size=(N, STRIDE), dtype=np.uint8)
    path = tmp_path / "experts.bin"
    data.tofile(path)
    return path, data


def _model_fetch(state, ids):
    """The RAM tier's rule: the call's resident ids are touched first; each
    missing id takes the least recently fetched slot."""
    order, slot_of = state
    hits = []
    for e in ids:
        if e in slot_of:
            order.remove(slot_of[e])
            order.append(slot_of[e])
    for e in ids:
        if e in slot_of:
            hits.append(1)
            continue
        sl = order.pop(0)
        for old, s2 in list(slot_of.items()):
            if s2 == sl:
                del slot_of[old]
        slot_of[e] = sl
        order.append(sl)
        hits.append(0)
    return hits


@pytest.mark.parametrize("threads", [1, 4])
def test_fetch_reads_blobs_and_follows_lru(blob_file, threads):
    path, data = blob_file
    ram = _aligned(SLOTS * STRIDE)
    st = M.ExpStore(path, N, BLOB, STRIDE, SLOTS, ram, io_threads=threads)
    state = (list(range(SLOTS)), {})
    rng = np.random.default_rng(5 + threads)
    misses = 0
    try:
        for _ in range(200):
            n = int(rng.integers(1, 7))
            ids = rng.choice(N, n, replace=False).astype(np.int32)
            ptrs, hit = st.fetch(ids)
            want = _model_fetch(state, ids.tolist())
            assert hit.tolist() == want
            misses += n - sum(want)
            for e, p in zip(ids.tolist(), ptrs.tolist()):
                got = np.frombuffer(C.string_at(int(p), BLOB), np.uint8)
                assert np.array_equal(got, data[e, :BLOB]), e
            snap = st.snapshot()
            assert {e: int(s) for e, s in enumerate(snap) if s >= 0} == state[1]
        s = st.stats()
        assert s["fetches"] == 200 and s["reads"] == misses and s["bytes_read"] == misses * BLOB
        assert s["evictions"] == misses - SLOTS
    finally:
        st.close()


def test_bad_calls_are_rejected(blob_file, tmp_path):
    path, data = blob_file
    ram = _aligned(SLOTS * STRIDE)
    st = M.ExpStore(path, N, BLOB, STRIDE, SLOTS, ram)
    try:
        for ids, status in (([1, 2, 1], M.MOE_EINVAL), ([N], M.MOE_EINVAL), ([-1], M.MOE_EINVAL),
                            (list(range(SLOTS + 1)), M.MOE_EBUSY)):
            with pytest.raises(M.MoEError) as ei:
                st.fetch(ids)
            assert ei.value.status == status
        assert (st.snapshot() == -1).all() and st.stats()["fetches"] == 0
    finally:
        st.close()
    with pytest.raises(M.MoEError) as ei:                       # the file is shorter than N + 1 experts
        M.ExpStore(path, N + 1, BLOB, STRIDE, SLOTS, ram)
    assert ei.value.status == M.MOE_EINVAL
    with pytest.raises(M.MoEError) as ei:
        M.ExpStore(tmp_path / "missing.bin", N, BLOB, STRIDE, SLOTS, ram)
    assert ei.value.status == M.MOE_EIO


def test_direct_io_reads_the_same_bytes(blob_file):
    """O_DIRECT where the file system offers it (tmpfs does not: the store
    then refuses to open with MOE_EIO and says so)."""
    path, data = blob_file
    ram = _aligned(SLOTS * STRIDE)
    try:
        st = M.ExpStore(path, N, BLOB, STRIDE, SLOTS, ram, io_threads=4, use_direct=True)
    except M.MoEError as e:
        assert e.status == M.MOE_EIO and "O_DIRECT" in M.moe_last_error()
        pytest.skip("no O_DIRECT on this file system")
    try:
        ids = np.array([3, 17, 39, 0], np.int32)
        ptrs, hit = st.fetch(ids)
        assert hit.tolist() == [0, 0, 0, 0]
        for e, p in zip(ids.tolist(), ptrs.tolist()):
            assert np.array_equal(np.frombuffer(C.string_at(int(p), BLOB), np.uint8), data[e, :BLOB])
        assert st.stats()["bytes_read"] == 4 * STRIDE             # whole 4096-byte blocks
    finally:
        st.close()
