"""Expert parallelism: the experts of a layer spread over the ranks of a
torch.distributed group, tokens exchanged by all-to-all.

Rank r holds the experts e with e % world == r (their blobs in its memory;
local index e // world).  Every rank routes its own tokens over all E experts
(the router is replicated), then
  1. dispatch: each (token, slot) row goes to the rank owning its expert --
     the per-destination counts first (all-to-all of one integer per rank),
     then the rows' activations and local expert indices (all-to-all with
     those split sizes), in ascending (token, slot) order per destination;
  2. the received rows run through the owner's expert FFN as tokens with one
     expert each;
  3. return: the outputs go back by the inverse all-to-all, so each rank gets
     the rows it sent, in the order it sent them;
  4. combine: y[t] = sum_j w[t, j] * out[t, j] (slot order) + the shared
     expert, which every rank computes for its own tokens.
Each (token, expert) output is computed exactly as on one GPU (one row of the
same FFN), so the result equals the single-rank layer's.

Strata article, section 2 item 2: only the selected experts run; spreading
them over GPUs is the scale-out of the same step.  The arithmetic runs in a
backend: `GpuBackend` (this library's kernels; the default) or any object
with the same four methods.  The exchange itself is this module's job.
"""
from __future__ import annotations

import numpy as np


def owner_of(ids: np.ndarray, world: int):
    """(rank, local index) of each expert id."""
    return ids % world, ids // world


def dispatch_plan(ids: np.ndarray, world: int):
    """The exchange of one rank's (token, slot) pairs.  ids [T, k] ->
    order: pair indices p = t * k + j sorted by destination rank (stable, so
    ascending p within a destination); counts [world]; local [n] the local
    expert index of each pair in send order; pos [T * k] each pair's place in
    send order (where its output comes back)."""
    flat = np.ascontiguousarray(ids, dtype=np.int64).reshape(-1)
    dest, local = owner_of(flat, world)
    order = np.argsort(dest, kind="stable")
    counts = np.bincount(dest, minlength=world).astype(np.int64)
    pos = np.empty(flat.size, np.int64)
    pos[order] = np.arange(flat.size)
    return order, counts, local[order].astype(np.int32), pos.astype(np.int32)


class ExpertParallelLayer:
    """One MoE layer with its routed experts spread over `group`.

    backend: route(x) -> (ids [T, k] int numpy, w [T, k] device/host tensor);
    local_ffn(rows [n, H], local_ids [n] int32 numpy) -> out [n, H] fp32;
    shared_ffn(x) -> [T, H] fp32 or None; combine(out [T*k, H], pos [T*k]
    int32, w, shared) -> y [T, H] fp32.  Tensors live on the backend's device;
    the all-to-alls run on the group's backend (NCCL for CUDA tensors, gloo
    for CPU tensors).
    """

    def __init__(self, group, E, k, H, backend):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.k, self.H = E, k, H
        self.backend = backend
        self.last = {}

    def local_experts(self):
        return np.arange(self.rank, self.E, self.world)

    def forward(self, x):
        import torch
        import torch.distributed as dist
        be, world = self.backend, self.world
        ids, w = be.route(x)
        T = ids.shape[0]
        order, counts, local, pos = dispatch_plan(ids, world)
        dev = x.device
        # 1. counts, then rows and their local expert indices
        send_counts = torch.from_numpy(counts).to(dev)
        recv_counts = torch.empty_like(send_counts)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        sc, rc = counts.tolist(), recv_counts.cpu().numpy().astype(np.int64).tolist()
        tok = torch.from_numpy((order // self.k).astype(np.int64)).to(dev)
        send_rows = x.index_select(0, tok).contiguous()
        recv_rows = torch.empty((sum(rc), self.H), dtype=x.dtype, device=dev)
        dist.all_to_all_single(recv_rows, send_rows, output_split_sizes=rc, input_split_sizes=sc, group=self.group)
        send_local = torch.from_numpy(local.astype(np.int32)).to(dev)
        recv_local = torch.empty(sum(rc), dtype=torch.int32, device=dev)
        dist.all_to_all_single(recv_local, send_local, output_split_sizes=rc, input_split_sizes=sc, group=self.group)
        # 2. this rank's experts on the rows it received
        out_local = be.local_ffn(recv_rows, recv_local.cpu().numpy())
        # 3. the outputs back to their senders, in the order they were sent
        back = torch.empty((T * self.k, self.H), dtype=out_local.dtype, device=dev)
        dist.all_to_all_single(back, out_local.contiguous(), output_split_sizes=sc, input_split_sizes=rc,
                               group=self.group)
        # 4. slot-order combine with the shared expert
        y = be.combine(back, pos, w, be.shared_ffn(x))
        self.last = dict(sent=sc, received=rc)
        return y


class GpuBackend:
    """The arithmetic of an expert-parallel layer in this library's kernels:
    route (moe_route_topk), the local experts' FFN on received rows (each row
    a token with one expert: moe_permute + moe_expert_ffn, the outputs put
    back in received order by moe_combine with unit gates), the shared
    expert, and the slot-order combine.

    local_blobs: uint8 [E_local, blob_bytes], this rank's experts in local
    order (expert rank + i * world); shared_blob or None; w_router [E, H]
    (bf16 bit patterns or fp32) and bias [E] or None, replicated.
    """

    def __init__(self, bits, H, I, E, k, local_blobs, shared_blob, w_router, w_dtype="bf16", bias=None, mode=0,
                 device="cuda"):
        import torch
        from . import MOE_BF16, MOE_F32, MoELayer, moe_expert_blob_bytes
        self.bits, self.H, self.I, self.E, self.k, self.mode = bits, H, I, E, k, mode
        self.dev = torch.device(device)
        nb = moe_expert_blob_bytes(bits, H, I)
        self.El = int(local_blobs.shape[0])
        self.experts = MoELayer(bits, H, I, self.El, 1, local_blobs, None, None, w_dtype) if self.El else None
        self.shared = None
        if shared_blob is not None:
            self.shared = torch.zeros((nb + 255) // 256 * 256, dtype=torch.uint8, device=self.dev)
            self.shared[:nb].copy_(torch.as_tensor(np.asarray(shared_blob)).to(self.dev))
        self.no_table = torch.zeros(max(1, E), dtype=torch.int64, device=self.dev)   # the shared-only call reads none
        wr = np.asarray(w_router)
        self.w_dtype = MOE_BF16 if w_dtype == "bf16" else MOE_F32
        self.w_router = (torch.from_numpy(wr.view(np.int16).copy()).view(torch.bfloat16) if w_dtype == "bf16"
                         else torch.from_numpy(wr.astype(np.float32))).to(self.dev)
        self.bias = None if bias is None else torch.as_tensor(np.asarray(bias, np.float32)).to(self.dev)
        self._bufs = {}

    def _buffers(self, T):
        from .layer import alloc_step_buffers
        if T not in self._bufs:
            self._bufs[T] = alloc_step_buffers(T, self.H, self.I, self.E, self.k, self.bits, self.mode, self.dev,
                                               self.shared is not None)
        return self._bufs[T]

    def route(self, x):
        from . import moe_route_topk
        T = x.shape[0]
        b = self._buffers(T)
        moe_route_topk(x, _dtype_code(x), self.w_router, self.w_dtype, None, self.bias, T, self.H, self.E, self.k,
                       b.ids, b.w, b.logits, b.ws_route, b.sizes["route"])
        ids = b.ids[:T * self.k].view(T, self.k).cpu().numpy()
        return ids, b.w[:T * self.k].clone()

    def local_ffn(self, rows, local_ids):
        import torch
        from . import moe_combine, moe_expert_ffn_q2, moe_expert_ffn_q4, moe_permute
        n = rows.shape[0]
        if n == 0:
            return torch.empty((0, self.H), dtype=torch.float32, device=self.dev)
        L = self.experts
        b = L.buffers(n, self.mode)
        b.ids[:n].copy_(torch.from_numpy(np.ascontiguousarray(local_ids, np.int32)).to(self.dev))
        moe_permute(b.ids, n, 1, L.E, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"])
        ffn = moe_expert_ffn_q4 if self.bits == 4 else moe_expert_ffn_q2
        ffn(L.table, b.offsets, b.active, b.perm_src, rows, _dtype_code(rows), n, 1, self.H, self.I, L.E, None,
            b.y_perm, None, self.mode, b.ws_ffn, b.sizes["ffn"])
        ones = torch.ones(n, dtype=torch.float32, device=self.dev)
        out = torch.empty((n, self.H), dtype=torch.float32, device=self.dev)
        moe_combine(b.y_perm, b.perm_dst, ones, None, n, 1, self.H, out)   # back to received order, exactly
        return out

    def shared_ffn(self, x):
        from . import moe_expert_ffn_q2, moe_expert_ffn_q4
        if self.shared is None:
            return None
        T = x.shape[0]
        b = self._buffers(T)
        b.active[:1].zero_()                              # no routed expert: the shared expert alone
        ffn = moe_expert_ffn_q4 if self.bits == 4 else moe_expert_ffn_q2
        ffn(self.no_table, b.offsets, b.active, b.perm_src, x, _dtype_code(x), T, self.k, self.H, self.I, self.E,
            self.shared, b.y_perm, b.y_shared, self.mode, b.ws_ffn, b.sizes["ffn"])
        return b.y_shared[:T * self.H].view(T, self.H).clone()

    def combine(self, out, pos, w, shared):
        import torch
        from . import moe_combine
        T = w.numel() // self.k
        y = torch.empty((T, self.H), dtype=torch.float32, device=self.dev)
        p = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).to(self.dev)
        moe_combine(out, p, w, shared, T, self.k, self.H, y)
        return y


def _dtype_code(x):
    import torch
    from . import MOE_BF16, MOE_F32
    return MOE_BF16 if x.dtype == torch.bfloat16 else MOE_F32
