"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
step through the C ABI, and compare against the oracle with the acceptance
rules (ids and permutation bit-exact; max |y - y_oracle| <= 2e-3 * RMS)."""
from __future__ import annotations

import numpy as np

TOL = 2e-3          # output tolerance, in units of RMS(y_oracle)
U32 = 2.0 ** -24    # fp32 unit roundoff


def dev_x(x, x_dtype):
    import torch
    if x_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def xd(x, x_dtype):
    import workloads as W
    return (W.bf16_bits_to_f32(x) if x_dtype == "bf16" else np.asarray(x, np.float32)).astype(np.float64)


def wd(layer):
    import workloads as W
    return (W.bf16_bits_to_f32(layer.w_router) if layer.w_dtype == "bf16" else layer.w_router).astype(np.float64)


def logit_bound(layer, x, x_dtype):
    """Rigorous bound on |fp32-accumulated logit - exact logit| (products of
    bf16/fp32 inputs are formed exactly or rounded once, then H additions)."""
    X, Wr = np.abs(xd(x, x_dtype)), np.abs(wd(layer))
    H = X.shape[1]
    gamma = (H + 2) * U32 / (1 - (H + 2) * U32)
    s = X @ Wr.T
    if layer.bias is not None:
        s = s + np.abs(layer.bias.astype(np.float64))
    return gamma * s + 2 * U32 * s


def decisive_tokens(logits64, eps, k):
    """Tokens whose gap between ranks k-1 and k exceeds twice the error bound."""
    T, E = logits64.shape
    out = np.ones(T, bool)
    if k >= E:
        return out
    for t in range(T):
        srt = np.sort(logits64[t])[::-1]
        out[t] = (srt[k - 1] - srt[k]) > 2 * eps[t].max()
    return out


def run_gpu(layer_gpu, x, x_dtype, mode=0, logits_in=None):
    import torch
    import quantized_expert_ffn_route_b200 as M
    T = x.shape[0]
    xdev = dev_x(x, x_dtype)
    li = None if logits_in is None else torch.from_numpy(np.ascontiguousarray(logits_in, np.float32)).cuda()
    b = layer_gpu.forward(xdev, M.MOE_BF16 if x_dtype == "bf16" else M.MOE_F32, T=T, mode=mode, logits_in=li)
    torch.cuda.synchronize()
    err = M.moe_device_error(clear=True)
    k, E, H = layer_gpu.k, layer_gpu.E, layer_gpu.H
    n_act = int(b.active[0].item())
    return dict(
        err=err,
        ids=b.ids[:T * k].cpu().numpy().reshape(T, k),
        w=b.w[:T * k].cpu().numpy().reshape(T, k),
        logits=b.logits[:T * E].cpu().numpy().reshape(T, E),
        offsets=b.offsets[:E + 1].cpu().numpy(),
        perm_src=b.perm_src[:T * k].cpu().numpy(),
        perm_dst=b.perm_dst[:T * k].cpu().numpy().reshape(T, k),
        active=b.active[:1 + n_act].cpu().numpy(),
        y_perm=b.y_perm[:T * k * H].cpu().numpy().reshape(T * k, H),
        y_shared=None if b.y_shared is None else b.y_shared[:T * H].cpu().numpy().reshape(T, H),
        y=b.y[:T * H].cpu().numpy().reshape(T, H),
    )


def rel_err(a, ref):
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(a - ref))) / rms if rms > 0 else float(np.max(np.abs(a - ref)))
