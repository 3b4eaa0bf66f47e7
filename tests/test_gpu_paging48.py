"""Model-scale paging on the GPU: several layers of experts drawn from one
pool, one expert cache, the next layer's likely experts prefetched while the
current layer computes.  Every layer's output equals the all-resident output
bit for bit, and the cache's event sequence (stage and prefetch) equals the
oracle simulator's."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import dev_x

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402
from quantized_expert_ffn_route_b200.paged import PagedExpertStack  # noqa: E402


@pytest.mark.parametrize("prefetch", [0, 4])
def test_paged_layers_equal_resident_and_oracle_events(prefetch):
    L, El, k, H, I, cap, tokens, decay = 4, 32, 4, 256, 128, 24, 12, 8
    layers = [W.make_layer(500 + l, 2, H, I, El, k, shared=False, w_dtype="bf16") for l in range(L)]
    nb = layers[0].blobs.shape[1]
    stride = (nb + 255) // 256 * 256
    pool = torch.zeros(L * El * stride, dtype=torch.uint8, pin_memory=True)
    pv = pool.view(L * El, stride)
    for l in range(L):
        pv[l * El:(l + 1) * El, :nb].copy_(torch.from_numpy(layers[l].blobs))
    slab = torch.zeros(cap * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(L * El, dtype=torch.int64, device="cuda")
    stack = PagedExpertStack(L, El, 2, H, I, k, pool, slab, table, cap, nb, stride, decay_period=decay,
                             prefetch=prefetch)
    stack.record = True
    resident = [M.MoELayer(2, H, I, El, k, layers[l].blobs, None, None, "bf16") for l in range(L)]
    trace = np.stack(list(W.paging48_trace(510, L, El, tokens, drift_every=4, hot=6)))
    x = W.make_tokens(511, tokens, H, "bf16")
    xd = dev_x(x, "bf16")
    li = torch.from_numpy(trace).cuda()
    outs = torch.empty(tokens, L, H, dtype=torch.float32, device="cuda")
    try:
        # the paged steps run back to back (no synchronisation between layers,
        # so prefetched copies overlap the next layers' work), each layer's
        # output kept; then the all-resident reference, layer by layer
        for t in range(tokens):
            for l in range(L):
                y = stack.layer_step(l, xd[t:t + 1], M.MOE_BF16, li[t, l])
                outs[t, l].copy_(y[:H])
        torch.cuda.synchronize()
        assert M.moe_device_error() == 0
        for t in range(tokens):
            for l in range(L):
                ref = resident[l].forward(xd[t:t + 1], M.MOE_BF16, mode=M.MOE_MODE_GEMV, logits_in=li[t, l][None])
                torch.cuda.synchronize()
                assert np.array_equal(outs[t, l].cpu().numpy(), ref.y[:H].cpu().numpy()), (t, l)
        ids = np.stack([e[0] for e in stack.events])
        pf = np.stack([e[4] for e in stack.events])
        want = oracle.cache_sim_prefetch(ids, pf, L * El, cap, decay)
        hits = np.stack([e[1] for e in stack.events])
        assert np.array_equal(hits.astype(bool), want["hit"])
        if prefetch:
            assert (hits == 2).any()                      # prefetched experts were used before a join
        assert np.array_equal(np.stack([e[2] for e in stack.events]), want["slot"])
        assert np.array_equal(np.stack([e[3] for e in stack.events]), want["victim"])
        assert np.array_equal(np.stack([e[5] for e in stack.events]), want["pf_slot"])
        assert np.array_equal(np.stack([e[6] for e in stack.events]), want["pf_victim"])
        st = stack.cache.stats()
        assert st["misses"] == want["misses"] and st["prefetched"] == want["prefetched"]
        if prefetch:
            assert want["prefetched"] > 0
    finally:
        stack.close()
