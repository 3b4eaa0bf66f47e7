"""Expert cache on the GPU: the event sequence (hits, slots, victims) equals
the oracle's simulator bit for bit; outputs computed from cache slots equal
the all-resident outputs bit for bit; failures are injected on the host
(a failing copy, a wait that runs out) and never fault the GPU."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import dev_x

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402


def _pool(layer, stride, pinned=True):
    E, nb = layer.blobs.shape
    host = torch.zeros(E * stride, dtype=torch.uint8, pin_memory=pinned)
    host.view(E, stride)[:, :nb].copy_(torch.from_numpy(layer.blobs))
    return host


def _make_cache(layer, capacity, decay, pinned=True):
    E, nb = layer.blobs.shape
    stride = (nb + 255) // 256 * 256
    host = _pool(layer, stride, pinned)
    slab = torch.zeros(capacity * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    stage = torch.zeros(2 * stride, dtype=torch.uint8, pin_memory=True) if not pinned else None
    c = M.ExpCache(E, capacity, nb, stride, host, slab, table, decay, stage_buffer=stage)
    return c, (host, slab, table, stage)


def _trace(seed, E, k, steps):
    gen = W.paging_trace(seed, E, k, steps, drift_every=25, hot=max(k, E // 4))
    return np.stack([np.argsort(-l, kind="stable")[:k] for l in gen]).astype(np.int32), \
        np.stack(list(W.paging_trace(seed, E, k, steps, drift_every=25, hot=max(k, E // 4))))


@pytest.mark.parametrize("pinned", [True, False])
def test_cache_events_and_outputs(pinned):
    E, k, cap, decay, steps = 96, 6, 16, 8, 120
    layer = W.make_layer(91, 2, 256, 128, E, k, shared=False, w_dtype="bf16")
    ids_trace, logits_trace = _trace(92, E, k, steps)
    ref = oracle.cache_sim(ids_trace, E, cap, decay)
    cache, keep = _make_cache(layer, cap, decay, pinned)
    resident = M.MoELayer(2, 256, 128, E, k, layer.blobs, None, None, "bf16")
    paged = M.MoELayer(2, 256, 128, E, k, layer.blobs, None, None, "bf16")
    table = keep[2]
    x = W.make_tokens(93, steps, 256, "bf16")
    xdev = dev_x(x, "bf16")
    s = torch.cuda.current_stream()
    for st in range(steps):
        li = torch.from_numpy(logits_trace[st][None]).cuda()
        # route + permute on the device; the ids come back to the host for the cache
        b = paged.buffers(1, M.MOE_MODE_GEMV)
        M.moe_route_topk(None, 0, None, 0, li, None, 1, 256, E, k, b.ids, b.w)
        ids = b.ids[:k].cpu().numpy()
        assert np.array_equal(ids, ids_trace[st])
        hit, slot, victim = cache.stage(ids)
        assert np.array_equal(hit.astype(bool), ref["hit"][st])
        assert np.array_equal(slot, ref["slot"][st])
        assert np.array_equal(victim, ref["victim"][st])
        cache.join()
        paged.table = table          # FFN reads blob pointers from the cache's device table
        out = paged.forward(xdev[st:st + 1], M.MOE_BF16, T=1, mode=M.MOE_MODE_GEMV, logits_in=li)
        y_paged = out.y[:256].clone()
        out2 = resident.forward(xdev[st:st + 1], M.MOE_BF16, T=1, mode=M.MOE_MODE_GEMV, logits_in=li)
        assert torch.equal(y_paged, out2.y[:256])
    assert M.moe_device_error() == 0
    stt = cache.stats()
    assert stt["misses"] == ref["misses"]
    assert stt["hits"] == steps * k - ref["misses"]
    cnt, _ = cache.snapshot()
    assert np.array_equal(cnt, ref["counts"])
    s.synchronize()
    cache.close()


def test_cache_injected_copy_failure_changes_nothing():
    E, k, cap = 32, 4, 8
    layer = W.make_layer(95, 2, 256, 128, E, k, shared=False, w_dtype="bf16")
    cache, keep = _make_cache(layer, cap, 0)
    cache.stage(np.array([0, 1, 2, 3]))
    before = cache.snapshot()
    cache.inject_copy_failures(1)
    with pytest.raises(M.MoEError) as ei:
        cache.stage(np.array([4, 5, 0, 1]))
    assert ei.value.status == M.MOE_EIO
    after = cache.snapshot()
    assert np.array_equal(before[0], after[0]) and np.array_equal(before[1], after[1])
    hit, slot, victim = cache.stage(np.array([4, 5, 0, 1]))     # next attempt succeeds
    assert hit.tolist() == [0, 0, 1, 1]
    assert cache.wait(10_000_000) == M.MOE_OK
    cache.close()


def test_cache_wait_times_out_then_completes():
    """The copy stream waits behind a bounded busy kernel on the compute stream."""
    E, k, cap = 16, 2, 4
    layer = W.make_layer(96, 2, 256, 128, E, k, shared=False, w_dtype="bf16")
    cache, keep = _make_cache(layer, cap, 0)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1.5e9))          # ~0.75 s at 2 GHz; ends by itself
    cache.stage(np.array([3, 7]))
    assert cache.wait(1000) == M.MOE_ETIMEDOUT
    assert cache.wait(30_000_000) == M.MOE_OK
    torch.cuda.synchronize()
    cache.close()


def test_cache_rejects_oversubscription_and_bad_ids():
    layer = W.make_layer(97, 2, 256, 128, 8, 2, shared=False, w_dtype="bf16")
    cache, keep = _make_cache(layer, 2, 0)
    with pytest.raises(M.MoEError) as ei:
        cache.stage(np.array([0, 1, 2]))
    assert ei.value.status == M.MOE_EBUSY
    with pytest.raises(M.MoEError) as ei:
        cache.stage(np.array([1, 1]))
    assert ei.value.status == M.MOE_EINVAL
    with pytest.raises(M.MoEError):
        cache.stage(np.array([9]))
    cache.stage(np.array([0, 1]))
    cache.evict(np.array([0]))
    slots, nm = cache.lookup(np.array([0, 1]))
    assert slots[0] == -1 and slots[1] >= 0 and nm == 1
    cache.close()


def test_cache_events_full_paging_trace():
    """The paging workload's whole trace (24,576 experts, 2048 HBM slots,
    5000 steps of 10 Gumbel-top-k ids over a Zipf popularity that drifts every
    200 steps, halving every 256 steps) through expcache_stage: every hit,
    slot and victim equals the oracle simulator's.  Blobs are 16 bytes here:
    the policy, not the copy size, is under test."""
    c = W.PAGING
    E, k, cap, steps, decay = c["E"], c["k"], c["capacity"], c["steps"], 256
    # the k largest logits of each step (any k distinct ids serve: the cache
    # and the simulator see the same ones)
    ids = np.stack([np.argpartition(-l, k - 1)[:k] for l in
                    W.paging_trace(W.SEED["paging"], E, k, steps, s=c["zipf_s"], drift_every=c["drift_every"],
                                   drift_prob=c["drift_prob"], hot=c["hot"])]).astype(np.int32)
    ref = oracle.cache_sim(ids, E, cap, decay)
    stride = 256
    host = torch.zeros(E * stride, dtype=torch.uint8, pin_memory=True)
    slab = torch.zeros(cap * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    cache = M.ExpCache(E, cap, 16, stride, host, slab, table, decay)
    try:
        for st in range(steps):
            hit, slot, victim = cache.stage(ids[st])
            assert np.array_equal(hit.astype(bool), ref["hit"][st]), st
            assert np.array_equal(slot, ref["slot"][st]), st
            assert np.array_equal(victim, ref["victim"][st]), st
        assert cache.wait(10_000_000) == M.MOE_OK
        st = cache.stats()
        assert st["misses"] == ref["misses"] and st["hits"] == steps * k - ref["misses"]
        cnt, _ = cache.snapshot()
        assert np.array_equal(cnt, ref["counts"])
    finally:
        cache.close()


def test_cache_copy_time_histogram():
    """Every step that staged copies is counted once in the copy-time
    histogram after the copies complete -- more steps than the event ring
    holds included -- and steps without misses are not counted."""
    E, k, cap = 12, 2, 8                             # hits are common: some steps stage nothing
    layer = W.make_layer(97, 2, 256, 128, E, k, shared=False, w_dtype="bf16")
    cache, keep = _make_cache(layer, cap, 0)
    rng = np.random.default_rng(3)
    with_copies = 0
    try:
        for step in range(80):                       # more than the 32-entry ring
            ids = rng.choice(E, k, replace=False)
            hit, _, _ = cache.stage(ids)
            with_copies += int((hit == 0).any())
            if step % 10 == 9:
                cache.join()
        assert cache.wait(30_000_000) == M.MOE_OK
        bins, n = cache.copy_histogram()
        assert n == with_copies == int(bins.sum()) and 0 < n < 80
        nz = np.nonzero(bins)[0]
        assert nz.min() >= 1 and nz.max() <= 16       # between 2 us and 130 ms per step's copies
        cache.stage(np.zeros(0, np.int32))           # an empty step: nothing to count
        resident = np.nonzero(cache.snapshot()[1] >= 0)[0][:k].astype(np.int32)
        hit, _, _ = cache.stage(resident)            # an all-hit step: nothing to count
        assert (hit == 1).all()
        assert cache.wait(30_000_000) == M.MOE_OK and cache.copy_histogram()[1] == n
    finally:
        torch.cuda.synchronize()
        cache.close()
