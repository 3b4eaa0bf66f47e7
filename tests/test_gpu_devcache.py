"""Device-initiated staging (devcache_*) on the GPU: the policy runs in a
kernel on the ids the router left in device memory, the admitted misses are
copied by a kernel from the mapped page-locked pool, and with an admission
threshold cold experts are computed in place from host memory.  Every layer's
output equals the all-resident output bit for bit; the logged events equal
the oracle simulator's; slots hold the pool's bytes exactly; whole steps
replay from a CUDA graph."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import dev_x

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402
from quantized_expert_ffn_route_b200.paged import DevicePagedExpertStack  # noqa: E402

L, El, K, H, I, CAP, DECAY = 4, 32, 4, 256, 128, 24, 8


def _stack(admit_min, log_steps, seed=600):
    layers = [W.make_layer(seed + l, 2, H, I, El, K, shared=False, w_dtype="bf16") for l in range(L)]
    nb = layers[0].blobs.shape[1]
    stride = (nb + 255) // 256 * 256
    pool = torch.zeros(L * El * stride, dtype=torch.uint8, pin_memory=True)
    pv = pool.view(L * El, stride)
    for l in range(L):
        pv[l * El:(l + 1) * El, :nb].copy_(torch.from_numpy(layers[l].blobs))
    slab = torch.zeros(CAP * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(L * El, dtype=torch.int64, device="cuda")
    stack = DevicePagedExpertStack(L, El, 2, H, I, K, pool, slab, table, CAP, nb, stride, decay_period=DECAY,
                                   admit_min=admit_min, log_steps=log_steps)
    resident = [M.MoELayer(2, H, I, El, K, layers[l].blobs, None, None, "bf16") for l in range(L)]
    return stack, resident, pool, slab, table, nb, stride


def _resident_outputs(resident, xd, li, tokens):
    out = np.empty((tokens, L, H), np.float32)
    for t in range(tokens):
        for l in range(L):
            ref = resident[l].forward(xd[t:t + 1], M.MOE_BF16, mode=M.MOE_MODE_GEMV, logits_in=li[t, l][None])
            torch.cuda.synchronize()
            out[t, l] = ref.y[:H].cpu().numpy()
    return out


@pytest.mark.parametrize("admit_min", [0, 2])
def test_device_staged_layers_equal_resident_and_oracle_events(admit_min):
    tokens = 40
    stack, resident, pool, slab, table, nb, stride = _stack(admit_min, log_steps=tokens * L)
    trace = np.stack(list(W.paging48_trace(610, L, El, tokens, drift_every=4, hot=6)))
    x = W.make_tokens(611, tokens, H, "bf16")
    xd = dev_x(x, "bf16")
    li = torch.from_numpy(trace).cuda()
    outs = torch.empty(tokens, L, H, dtype=torch.float32, device="cuda")
    stack.ids_log = torch.empty(tokens * L, K, dtype=torch.int32, device="cuda")
    try:
        # every layer of every token enqueued back to back: no host synchronisation
        for t in range(tokens):
            for l in range(L):
                y = stack.layer_step(l, xd[t:t + 1], M.MOE_BF16, li[t, l])
                outs[t, l].copy_(y[:H])
        torch.cuda.synchronize()
        assert M.moe_device_error() == 0
        ref = _resident_outputs(resident, xd, li, tokens)
        assert np.array_equal(outs.cpu().numpy(), ref)
        # events against the oracle (global ids: layer base added)
        ids = stack.ids_log.cpu().numpy() + (np.arange(tokens * L) % L * El)[:, None]
        want = oracle.cache_sim_admit(ids, L * El, CAP, DECAY, admit_min)
        hit, slot, victim = stack.cache.events(0, tokens * L)
        assert np.array_equal(hit[:, :K], want["hit"])
        assert np.array_equal(slot[:, :K], want["slot"])
        assert np.array_equal(victim[:, :K], want["victim"])
        st = stack.cache.stats()
        assert st["steps"] == tokens * L and st["misses"] == want["misses"] and st["bad_steps"] == 0
        assert st["in_place"] == want["in_place"] and (want["in_place"] > 0) == (admit_min > 1)
        assert st["hits"] == int((want["hit"] == 1).sum())
        assert st["evictions"] == int((want["victim"] >= 0).sum()) > 0
        cnt, slot_of = stack.cache.snapshot()
        assert np.array_equal(cnt, want["counts"])
        # slots hold the pool's bytes; the table points at them; the last
        # step's in-place experts point into the pool, all others are NULL
        pv = pool.view(L * El, stride)
        tab = table.cpu().numpy()
        base_slab, base_pool = slab.data_ptr(), pool.data_ptr()
        last_in_place = set(ids[-1][want["hit"][-1] == 3].tolist())
        for e in range(L * El):
            if slot_of[e] >= 0:
                got = slab[slot_of[e] * stride:slot_of[e] * stride + nb].cpu()
                assert torch.equal(got, pv[e, :nb]), e
                assert int(tab[e]) == base_slab + int(slot_of[e]) * stride
            elif e in last_in_place:
                assert int(tab[e]) == base_pool + e * stride
            else:
                assert tab[e] == 0
    finally:
        stack.close()


def test_device_staging_rejects_repeated_ids_without_state_change():
    stack, resident, pool, slab, table, nb, stride = _stack(0, log_steps=4)
    try:
        ids = torch.tensor([3, 5, 3, 7], dtype=torch.int32, device="cuda")
        act = torch.full((M.DEVCACHE_ACT_INTS,), 99, dtype=torch.int32, device="cuda")
        stack.cache.stage(ids, 4, act)
        torch.cuda.synchronize()
        assert M.moe_device_error() == M.DEVERR_BAD_EXPERT
        a = act.cpu().numpy()
        assert a[0] == 0 and a[33] == 0
        st = stack.cache.stats()
        assert st["bad_steps"] == 1 and st["steps"] == 0 and st["misses"] == 0
        cnt, slot_of = stack.cache.snapshot()
        assert (cnt == 0).all() and (slot_of == -1).all() and (table.cpu().numpy() == 0).all()
        ok = torch.tensor([3, 5, 6, 7], dtype=torch.int32, device="cuda")
        stack.cache.stage(ok, 4, act)                        # the next good step runs normally
        torch.cuda.synchronize()
        assert M.moe_device_error() == 0
        a = act.cpu().numpy()
        assert a[0] == 0 and a[33] == 4 and sorted(a[34:38].tolist()) == [3, 5, 6, 7]
        with pytest.raises(M.MoEError):
            stack.cache.stage(ok, 33, act)                   # more ids than a step may hold
    finally:
        stack.close()


def test_device_staged_steps_replay_from_a_cuda_graph():
    """Two tokens x L layers of device-staged steps in one CUDA graph: every
    replay (the cache state moving on each time) gives the all-resident
    outputs bit for bit."""
    tokens = 2
    stack, resident, pool, slab, table, nb, stride = _stack(2, log_steps=0, seed=640)
    trace = np.stack(list(W.paging48_trace(650, L, El, tokens, drift_every=4, hot=6)))
    x = W.make_tokens(651, tokens, H, "bf16")
    xd = dev_x(x, "bf16")
    li = torch.from_numpy(trace).cuda()
    outs = torch.empty(tokens, L, H, dtype=torch.float32, device="cuda")
    try:
        for t in range(tokens):                              # warm-up: first launches outside the capture
            for l in range(L):
                stack.layer_step(l, xd[t:t + 1], M.MOE_BF16, li[t, l])
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(graph, stream=s):
                for t in range(tokens):
                    for l in range(L):
                        y = stack.layer_step(l, xd[t:t + 1], M.MOE_BF16, li[t, l], stream=s)
                        outs[t, l].copy_(y[:H])
        torch.cuda.current_stream().wait_stream(s)
        ref = _resident_outputs(resident, xd, li, tokens)
        steps0 = stack.cache.stats()["steps"]
        for r in range(3):
            outs.zero_()
            graph.replay()
            torch.cuda.synchronize()
            assert M.moe_device_error() == 0
            assert np.array_equal(outs.cpu().numpy(), ref), r
        assert stack.cache.stats()["steps"] == steps0 + 3 * tokens * L
        del graph
    finally:
        stack.close()
