"""Model-scale expert paging: L layers of E_l experts each, all drawn from one
pool of L * E_l expert blobs in page-locked host memory, served through one
expert cache (HBM slots).  Expert e of layer l is pool entry l * E_l + e.

Per layer of a token (Strata article, section 2 item 2: resident experts are
computed at once, only the others must first be moved in):
  route over the layer's E_l experts -> the selected ids cross to the host ->
  expcache_stage -> the FFN of the resident (hit) experts, overlapping the
  miss copies -> expcache_join -> expcache_prefetch of the next layer's most
  frequently used experts (their copies overlap this layer's remaining work
  and the next layer's routing) -> the FFN of the missed experts -> combine.

Everything here is host-side orchestration and argument marshalling; every
arithmetic step runs in libmoe's kernels.
"""
from __future__ import annotations

import numpy as np


class PagedExpertStack:
    """L layers x E_l experts of one blob format behind one expert cache.

    pool: page-locked host tensor [L * E_l * stride] uint8; slab: device
    [capacity * stride]; table: device int64 [L * E_l] (the cache's table);
    the compute of layer l reads table[l * E_l : (l + 1) * E_l].
    prefetch: experts of the next layer to prefetch per layer (0 = none),
    chosen by the number of times each expert was selected so far (ties: the
    lower id).
    store: an ExpStore (the NVMe tier) to read missed experts from, into its
    RAM tier, before the cache copies them to HBM; pool is then only the
    cache's nominal pool and prefetch must be 0.
    """

    def __init__(self, layers, experts_per_layer, bits, H, I, k, pool, slab, table, capacity, blob_bytes, stride,
                 decay_period=256, prefetch=10, device="cuda", store=None):
        import torch
        from . import MOE_MODE_GEMV, ExpCache, alloc_step_buffers
        self.L, self.El, self.bits, self.H, self.I, self.k = layers, experts_per_layer, bits, H, I, k
        if store is not None and prefetch:
            raise ValueError("prefetch copies from the pool; with an expert store it must be 0")
        self.prefetch_n = prefetch
        self.store = store
        self.pool, self.slab, self.table = pool, slab, table
        self.cache = ExpCache(layers * experts_per_layer, capacity, blob_bytes, stride, pool, slab, table,
                              decay_period)
        self.dev = torch.device(device)
        self.b = alloc_step_buffers(1, H, I, experts_per_layer, k, bits, MOE_MODE_GEMV, self.dev, False)
        self.ids_h = torch.empty(k, dtype=torch.int32).pin_memory()
        self.act_h = torch.zeros(64, dtype=torch.int32).pin_memory()
        self.act_d = torch.zeros(64, dtype=torch.int32, device=self.dev)
        self.freq = np.zeros(layers * experts_per_layer, np.int64)
        self.events = []          # per layer step: (global ids, hit, slot, victim, pf ids, pf slot, pf victim)
        self.record = False

    def close(self):
        self.cache.close()

    def predict(self, layer):
        """The next layer's prefetch list: its most often selected experts."""
        if self.prefetch_n <= 0:
            return np.full(max(1, self.prefetch_n), -1, np.int32)
        f = self.freq[layer * self.El:(layer + 1) * self.El]
        order = np.lexsort((np.arange(self.El), -f))[:self.prefetch_n]
        return (order + layer * self.El).astype(np.int32)

    def layer_step(self, layer, x, x_dtype, logits, y_out=None, stream=None):
        """One token through one layer: logits [E_l] fp32 device, x [H] device;
        returns the output buffer (fp32 [H])."""
        import torch
        from . import moe_combine, moe_expert_ffn_q2, moe_expert_ffn_q4, moe_permute, moe_route_topk
        b, k, El, H, I = self.b, self.k, self.El, self.H, self.I
        s = torch.cuda.current_stream() if stream is None else stream
        moe_route_topk(None, 0, None, 0, logits, None, 1, H, El, k, b.ids, b.w, None, b.ws_route, b.sizes["route"],
                       stream=s)
        moe_permute(b.ids, 1, k, El, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"],
                    stream=s)
        self.ids_h.copy_(b.ids[:k], non_blocking=True)
        s.synchronize()                                   # the ids cross to the host
        local = self.ids_h.numpy().copy()
        gids = (local + layer * El).astype(np.int32)
        if self.store is not None:                        # missed experts: drive -> RAM tier -> HBM
            from . import MOE_OK
            slots, _ = self.cache.lookup(gids)
            srcs = np.zeros(gids.size, np.uint64)
            if (slots < 0).any():
                if self.cache.wait(10_000_000) != MOE_OK:   # copies out of RAM slots the fetch may reuse
                    raise RuntimeError("expert copies did not finish within 10 s")
                ptrs, _ = self.store.fetch(gids[slots < 0])
                srcs[slots < 0] = ptrs
            hit, slot, victim = self.cache.stage_from(gids, srcs, stream=s)
        else:
            hit, slot, victim = self.cache.stage(gids, stream=s)
        np.add.at(self.freq, gids, 1)
        # hit 1: resident and settled, computed at once; hit 2 (admitted by a
        # prefetch whose copy may still be in flight) and misses after the join
        hits, miss = np.sort(local[hit == 1]), np.sort(local[hit != 1])
        a = self.act_h.numpy()
        a[0], a[1:1 + hits.size] = hits.size, hits
        a[32], a[33:33 + miss.size] = miss.size, miss
        self.act_d.copy_(self.act_h, non_blocking=True)
        ffn = moe_expert_ffn_q4 if self.bits == 4 else moe_expert_ffn_q2
        tview = self.table[layer * El:(layer + 1) * El]
        if hits.size:                                     # resident experts: at once, overlapping the copies
            ffn(tview, b.offsets, self.act_d[0:], b.perm_src, x, x_dtype, 1, k, H, I, El, None, b.y_perm, None,
                1, b.ws_ffn, b.sizes["ffn"], stream=s)
        self.cache.join(stream=s)                         # the misses' and the prefetched experts' copies
        pf = self.predict((layer + 1) % self.L)            # the next layer (of this or the next token)
        if self.prefetch_n > 0:
            pf_slot, pf_victim, _ = self.cache.prefetch(pf, stream=s)
        else:
            pf_slot = pf_victim = np.full(pf.size, -1, np.int32)
        if miss.size:
            ffn(tview, b.offsets, self.act_d[32:], b.perm_src, x, x_dtype, 1, k, H, I, El, None, b.y_perm, None,
                1, b.ws_ffn, b.sizes["ffn"], stream=s)
        y = b.y if y_out is None else y_out
        moe_combine(b.y_perm, b.perm_dst, b.w, None, 1, k, H, y, stream=s)
        if self.record:
            self.events.append((gids, hit, slot, victim, pf, pf_slot, pf_victim))
        return y


class DevicePagedExpertStack:
    """The same L x E_l stack with device-initiated staging (devcache_*): a
    layer step enqueues route -> the policy kernel (reading the selected ids
    where the router left them; its copy kernel starts at once) -> permute ->
    the FFN of the hits and of
    experts computed in place from the host pool -> devcache_join (the copy
    kernel of the admitted misses) -> the FFN of the admitted misses ->
    combine, with no host synchronisation, so whole tokens can be enqueued
    back to back or captured in a CUDA graph.

    pool: page-locked (mapped) host tensor [L * E_l * stride] uint8; slab:
    device [capacity * stride]; table: device int64 [L * E_l].  admit_min > 1
    computes a missed expert used fewer than admit_min times in place instead
    of admitting it.  log_steps > 0 keeps that many steps of events on the
    device (DevCache.events).
    """

    def __init__(self, layers, experts_per_layer, bits, H, I, k, pool, slab, table, capacity, blob_bytes, stride,
                 decay_period=256, admit_min=0, log_steps=0, device="cuda"):
        import torch
        from . import DEVCACHE_ACT_INTS, MOE_MODE_GEMV, DevCache, alloc_step_buffers
        self.L, self.El, self.bits, self.H, self.I, self.k = layers, experts_per_layer, bits, H, I, k
        self.pool, self.slab, self.table = pool, slab, table
        self.cache = DevCache(layers * experts_per_layer, capacity, blob_bytes, stride, pool, slab, table,
                              decay_period, admit_min, log_steps)
        self.dev = torch.device(device)
        self.b = alloc_step_buffers(1, H, I, experts_per_layer, k, bits, MOE_MODE_GEMV, self.dev, False)
        self.act = torch.zeros(DEVCACHE_ACT_INTS, dtype=torch.int32, device=self.dev)
        self.copy_stream = torch.cuda.Stream(device=self.dev)
        self.ids_log = None                 # optional device int32 [steps, k]: each step's ids (local)
        self.steps = 0

    def close(self):
        self.cache.close()

    def layer_step(self, layer, x, x_dtype, logits, y_out=None, stream=None):
        """One token through one layer: logits [E_l] fp32 device, x [H] device;
        returns the output buffer (fp32 [H])."""
        import torch
        from . import MOE_MODE_GEMV, moe_combine, moe_expert_ffn_q2, moe_expert_ffn_q4, moe_permute, moe_route_topk
        b, k, El, H, I = self.b, self.k, self.El, self.H, self.I
        s = torch.cuda.current_stream() if stream is None else stream
        moe_route_topk(None, 0, None, 0, logits, None, 1, H, El, k, b.ids, b.w, None, b.ws_route, b.sizes["route"],
                       stream=s)
        if self.ids_log is not None:
            with torch.cuda.stream(s):
                self.ids_log[self.steps].copy_(b.ids[:k])
        # the policy needs only the ids: its copies start before the permute, which only the FFN needs
        self.cache.stage(b.ids, k, self.act, id_base=layer * El, stream=s, copy_stream=self.copy_stream)
        self.steps += 1
        moe_permute(b.ids, 1, k, El, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"],
                    stream=s)
        ffn = moe_expert_ffn_q4 if self.bits == 4 else moe_expert_ffn_q2
        tview = self.table[layer * El:(layer + 1) * El]
        ffn(tview, b.offsets, self.act[0:], b.perm_src, x, x_dtype, 1, k, H, I, El, None, b.y_perm, None,
            MOE_MODE_GEMV, b.ws_ffn, b.sizes["ffn"], stream=s)   # hits and in-place experts, overlapping the copies
        self.cache.join(stream=s)
        ffn(tview, b.offsets, self.act[33:], b.perm_src, x, x_dtype, 1, k, H, I, El, None, b.y_perm, None,
            MOE_MODE_GEMV, b.ws_ffn, b.sizes["ffn"], stream=s)   # the admitted misses
        y = b.y if y_out is None else y_out
        moe_combine(b.y_perm, b.perm_dst, b.w, None, 1, k, H, y, stream=s)
        return y
