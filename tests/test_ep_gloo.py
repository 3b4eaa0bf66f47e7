"""Expert parallelism's exchange on CPU ranks (gloo): experts spread over 2 and
3 ranks, each rank's tokens routed over all experts, dispatched to the owners
by all-to-all, computed there, returned and combined -- equal to the whole
layer computed in one process.  The arithmetic of each step is the oracle's
(a test backend), so this checks the dispatch plan and the exchange, which are
the product's; on a GPU the same exchange runs with the library's kernels."""
import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
BITS, H, I, E, K = 4, 256, 128, 12, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBackend:
    """The four arithmetic steps of an expert-parallel layer in the fp64
    oracle, on CPU tensors."""

    def __init__(self, layer, rank, world):
        import oracle
        self.o, self.layer, self.rank, self.world = oracle, layer, rank, world

    def route(self, x):
        xb = x.numpy().astype(np.float32)
        logits = self.o.router_logits(xb, "f32", self.layer.w_router, self.layer.w_dtype)
        ids, w, st = self.o.topk(logits, K)
        assert st == 0
        return ids, torch.from_numpy(w)

    def local_ffn(self, rows, local_ids):
        if rows.shape[0] == 0:
            return torch.empty((0, H), dtype=torch.float64)
        blobs = [self.layer.blobs[self.rank + self.world * int(l)] for l in local_ids]
        return torch.from_numpy(self.o.expert_ffn_rows(BITS, H, I, blobs, rows.numpy().astype(np.float64)))

    def shared_ffn(self, x):
        T = x.shape[0]
        return torch.from_numpy(self.o.expert_ffn_rows(BITS, H, I, [self.layer.shared] * T,
                                                       x.numpy().astype(np.float64)))

    def combine(self, out, pos, w, shared):
        T = w.shape[0]
        return torch.from_numpy(self.o.combine(out.numpy(), np.asarray(pos, np.int32).reshape(T, K), w.numpy(),
                                               shared.numpy()))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, str(ROOT))
    import oracle
    import workloads as W
    from quantized_expert_ffn_route_b200.ep import ExpertParallelLayer
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layer = W.make_layer(321, BITS, H, I, E, K, shared=True, w_dtype="f32")
        T = 4 + rank                                    # ranks hold different numbers of tokens
        x = W.make_tokens(400 + rank, T, H, "f32")
        ep = ExpertParallelLayer(dist.group.WORLD, E, K, H, OracleBackend(layer, rank, world))
        y = ep.forward(torch.from_numpy(np.asarray(x, np.float64)))
        ref = oracle.moe_layer(BITS, x, "f32", layer.blobs, k=K, H=H, I=I, E=E, w_router=layer.w_router,
                               w_dtype="f32", shared_blob=layer.shared)
        err = float(np.max(np.abs(y.numpy() - ref["y"])) / np.sqrt(np.mean(ref["y"] ** 2)))
        q.put((rank, err, ep.last["sent"], ep.last["received"], ref["ids"].tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_exchange_equals_the_whole_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    sent = np.array([r[2] for r in res])                # sent[r][d]: rows rank r sent to rank d
    recv = np.array([r[3] for r in res])
    assert np.array_equal(sent.T, recv)                 # what r sent to d is what d received from r
    for rank, err, s, rc, ids in res:
        assert err <= 1e-12, (rank, err)
        flat = np.array(ids).reshape(-1)
        assert s == np.bincount(flat % world, minlength=world).tolist()   # each row went to its expert's owner
        assert sum(s) == (4 + rank) * K


def test_dispatch_plan_orders_pairs_by_owner_stably():
    from quantized_expert_ffn_route_b200.ep import dispatch_plan
    ids = np.array([[5, 2, 7], [1, 4, 0]])              # world 3: owners 2 2 1 / 1 1 0
    order, counts, local, pos = dispatch_plan(ids, 3)
    assert counts.tolist() == [1, 3, 2]
    assert order.tolist() == [5, 2, 3, 4, 0, 1]         # by owner, ascending pair index within one
    assert local.tolist() == [0, 2, 0, 1, 1, 0]         # e // 3 in send order
    assert np.array_equal(order[pos], np.arange(6))     # pos is where each pair's output comes back
