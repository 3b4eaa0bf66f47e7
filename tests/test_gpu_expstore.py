"""Three tiers on the GPU: expert blobs in a file (the NVMe tier), read on
demand into a page-locked RAM tier (expstore_fetch), copied from there into
HBM slots (expcache_stage_from).  Every layer's output equals the
all-resident output bit for bit and the HBM tier's events equal the oracle
simulator's; the RAM tier reads each expert only when it is not held."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import dev_x

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import quantized_expert_ffn_route_b200 as M  # noqa: E402
from quantized_expert_ffn_route_b200.paged import PagedExpertStack  # noqa: E402


@pytest.mark.parametrize("direct", [False, True])
def test_drive_ram_hbm_tiers_equal_resident_and_oracle_events(tmp_path, direct):
    L, El, k, H, I, cap, ram_slots, tokens, decay = 2, 32, 4, 256, 128, 8, 12, 16, 8
    layers = [W.make_layer(700 + l, 2, H, I, El, k, shared=False, w_dtype="bf16") for l in range(L)]
    nb = layers[0].blobs.shape[1]
    stride = (nb + 4095) // 4096 * 4096                    # whole 4096-byte blocks, as O_DIRECT reads them
    data = np.zeros((L * El, stride), np.uint8)
    for l in range(L):
        data[l * El:(l + 1) * El, :nb] = layers[l].blobs
    path = tmp_path / "experts.bin"
    data.tofile(path)
    ram_raw = torch.zeros(ram_slots * stride + 4096, dtype=torch.uint8, pin_memory=True)
    off = (-ram_raw.data_ptr()) % 4096                     # O_DIRECT reads need 4096-byte-aligned targets
    ram = ram_raw[off:off + ram_slots * stride]
    try:
        store = M.ExpStore(path, L * El, nb, stride, ram_slots, ram, io_threads=4, use_direct=direct)
    except M.MoEError as e:
        if direct and e.status == M.MOE_EIO:
            pytest.skip("no O_DIRECT on this file system: " + M.moe_last_error())
        raise
    slab = torch.zeros(cap * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(L * El, dtype=torch.int64, device="cuda")
    # the cache's nominal pool is the RAM tier: every miss names its source
    stack = PagedExpertStack(L, El, 2, H, I, k, ram, slab, table, cap, nb, stride, decay_period=decay, prefetch=0,
                             store=store)
    stack.record = True
    resident = [M.MoELayer(2, H, I, El, k, layers[l].blobs, None, None, "bf16") for l in range(L)]
    trace = np.stack(list(W.paging48_trace(710, L, El, tokens, drift_every=4, hot=6)))
    x = W.make_tokens(711, tokens, H, "bf16")
    xd = dev_x(x, "bf16")
    li = torch.from_numpy(trace).cuda()
    try:
        for t in range(tokens):
            for l in range(L):
                y = stack.layer_step(l, xd[t:t + 1], M.MOE_BF16, li[t, l])
                got = y[:H].cpu().numpy().copy()
                ref = resident[l].forward(xd[t:t + 1], M.MOE_BF16, mode=M.MOE_MODE_GEMV, logits_in=li[t, l][None])
                torch.cuda.synchronize()
                assert np.array_equal(got, ref.y[:H].cpu().numpy()), (t, l)
        assert M.moe_device_error() == 0
        ids = np.stack([e[0] for e in stack.events])
        want = oracle.cache_sim(ids, L * El, cap, decay)
        assert np.array_equal(np.stack([e[1] for e in stack.events]).astype(bool), want["hit"])
        assert np.array_equal(np.stack([e[2] for e in stack.events]), want["slot"])
        assert np.array_equal(np.stack([e[3] for e in stack.events]), want["victim"])
        st = store.stats()
        assert st["reads"] > 0 and st["hits"] > 0                      # both RAM misses and RAM hits happened
        assert st["reads"] + st["hits"] == want["misses"]              # every HBM miss went through the RAM tier
        assert st["bytes_read"] == st["reads"] * (stride if direct else nb)
    finally:
        stack.close()
        store.close()
