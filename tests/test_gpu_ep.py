"""Expert parallelism on the GPU with this library's kernels (GpuBackend) and
NCCL: with one rank -- the only GPU count this test can use -- the whole
dispatch / expert FFN / return / combine path must give the resident layer's
output bit for bit (each (token, expert) row is computed by the same kernel
either way).  The exchange between several ranks is covered on CPU ranks
(test_ep_gloo.py)."""
import os
import socket
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _main(port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
    sys.path.insert(0, str(ROOT))
    import numpy as np
    import torch
    import torch.distributed as dist
    import quantized_expert_ffn_route_b200 as M
    import workloads as W
    from quantized_expert_ffn_route_b200.ep import ExpertParallelLayer, GpuBackend
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1)
    res = []
    try:
        for bits, T, mode in ((4, 6, M.MOE_MODE_GEMV), (2, 5, M.MOE_MODE_GEMV), (4, 96, M.MOE_MODE_GEMM)):
            H, I, E, k = 256, 128, 16, 4
            layer = W.make_layer(900 + T, bits, H, I, E, k, shared=True, w_dtype="bf16")
            x = W.make_tokens(901 + T, T, H, "bf16")
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            be = GpuBackend(bits, H, I, E, k, layer.blobs, layer.shared, layer.w_router, "bf16", mode=mode)
            ep = ExpertParallelLayer(dist.group.WORLD, E, k, H, be)
            y = ep.forward(xd)
            ref = M.MoELayer(bits, H, I, E, k, layer.blobs, layer.shared, layer.w_router, "bf16").forward(
                xd, M.MOE_BF16, mode=mode)
            torch.cuda.synchronize()
            res.append((bits, T, mode, bool(torch.equal(y.reshape(-1), ref.y[:T * H])), M.moe_device_error(),
                        ep.last["sent"]))
    finally:
        dist.destroy_process_group()
    q.put(res)


def test_single_rank_expert_parallel_equals_resident_layer():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    p = ctx.Process(target=_main, args=(_free_port(), q))
    p.start()
    p.join(timeout=300)
    assert p.exitcode == 0
    for bits, T, mode, same, err, sent in q.get():
        assert err == 0 and same, (bits, T, mode)
        assert sent == [T * 4]
