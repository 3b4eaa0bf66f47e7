"""One MoE layer held in HBM, run through the C ABI.

The blobs of all experts live in one device arena (one slot per expert);
the device table holds each expert's blob pointer.  ``MoELayer.forward`` is
the whole step: route -> permute -> expert FFN (routed + shared) -> combine,
four library calls on one stream.  Buffers are torch tensors (device memory
only); nothing here computes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def _round_up(n: int, a: int) -> int:
    return (n + a - 1) // a * a


@dataclass
class StepBuffers:
    T: int
    ids: object
    w: object
    logits: object
    offsets: object
    perm_src: object
    perm_dst: object
    active: object
    ws_route: object
    ws_perm: object
    ws_ffn: object
    y_perm: object
    y_shared: object
    y: object
    sizes: dict


def alloc_step_buffers(T: int, H: int, I: int, E: int, k: int, bits: int, mode: int, device, shared: bool):
    import torch
    from . import moe_expert_ffn_ws_size, moe_permute_ws_size, moe_route_ws_size
    i32 = dict(dtype=torch.int32, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    u8 = dict(dtype=torch.uint8, device=device)
    Tk = max(1, T * k)
    sizes = dict(route=moe_route_ws_size(T, E, k), perm=moe_permute_ws_size(T, k, E),
                 ffn=moe_expert_ffn_ws_size(bits, T, k, H, I, E, mode))
    return StepBuffers(
        T=T,
        ids=torch.empty(_round_up(Tk, 4), **i32), w=torch.empty(_round_up(Tk, 4), **f32),
        logits=torch.empty(max(1, T) * E, **f32),
        offsets=torch.empty(_round_up(E + 1, 4), **i32),
        perm_src=torch.empty(_round_up(Tk, 4), **i32), perm_dst=torch.empty(_round_up(Tk, 4), **i32),
        active=torch.empty(_round_up(1 + min(E, Tk), 4), **i32),
        ws_route=torch.empty(max(16, sizes["route"]), **u8),
        ws_perm=torch.empty(max(16, sizes["perm"]), **u8),
        ws_ffn=torch.empty(max(16, sizes["ffn"]), **u8),
        y_perm=torch.empty(Tk * H, **f32),
        y_shared=torch.empty(max(1, T) * H, **f32) if shared else None,
        y=torch.empty(max(1, T) * H, **f32),
        sizes=sizes)


class MoELayer:
    """Resident quantized MoE layer (all experts in HBM).

    blobs: uint8 [E, blob_bytes] (numpy or torch); shared: uint8 [blob_bytes] or None;
    w_router: [E, H] float32 or bf16 bit patterns (uint16) with w_dtype "f32" | "bf16";
    bias: [E] float32 or None.
    """

    def __init__(self, bits, H, I, E, k, blobs, shared=None, w_router=None, w_dtype="bf16", bias=None,
                 device="cuda", slot_align=256):
        import torch
        from . import MOE_BF16, MOE_F32, moe_expert_blob_bytes
        self.bits, self.H, self.I, self.E, self.k = bits, H, I, E, k
        self.device = torch.device(device)
        nb = moe_expert_blob_bytes(bits, H, I)
        if nb <= 0 or tuple(blobs.shape) != (E, nb):
            raise ValueError(f"blobs must be uint8 [E={E}, {nb}] for bits={bits}, H={H}, I={I}; got {tuple(blobs.shape)}")
        if shared is not None and int(np.asarray(shared).size) != nb:
            raise ValueError(f"shared blob must hold {nb} bytes")
        self.blob_bytes = nb
        self.stride = _round_up(nb, slot_align)
        self.arena = torch.empty(E * self.stride, dtype=torch.uint8, device=self.device)
        view = self.arena.view(E, self.stride)[:, :nb]
        src = torch.as_tensor(np.asarray(blobs)) if not isinstance(blobs, torch.Tensor) else blobs
        view.copy_(src.to(self.device, non_blocking=False))
        base = self.arena.data_ptr()
        self.table = torch.tensor([base + e * self.stride for e in range(E)], dtype=torch.int64,
                                  device=self.device)
        self.shared = None
        if shared is not None:
            self.shared = torch.empty(self.stride, dtype=torch.uint8, device=self.device)
            self.shared[:nb].copy_(torch.as_tensor(np.asarray(shared)).to(self.device))
        self.w_dtype = MOE_BF16 if w_dtype == "bf16" else MOE_F32
        self.w_router = None
        if w_router is not None:
            wr = np.asarray(w_router)
            if w_dtype == "bf16":
                self.w_router = torch.from_numpy(wr.view(np.int16).copy()).view(torch.bfloat16).to(self.device)
            else:
                self.w_router = torch.from_numpy(wr.astype(np.float32)).to(self.device)
        self.bias = None if bias is None else torch.as_tensor(np.asarray(bias, np.float32)).to(self.device)
        self._bufs = {}

    def clone(self):
        """A copy of the layer at new device addresses (same bytes)."""
        import copy
        import torch
        c = copy.copy(self)
        c.arena = self.arena.clone()
        base = c.arena.data_ptr()
        c.table = torch.tensor([base + e * self.stride for e in range(self.E)], dtype=torch.int64,
                               device=self.device)
        c.shared = None if self.shared is None else self.shared.clone()
        c.w_router = None if self.w_router is None else self.w_router.clone()
        c.bias = None if self.bias is None else self.bias.clone()
        c._bufs = {}
        return c

    def buffers(self, T, mode):
        key = (T, mode)
        if key not in self._bufs:
            self._bufs[key] = alloc_step_buffers(T, self.H, self.I, self.E, self.k, self.bits, mode, self.device,
                                                 self.shared is not None)
        return self._bufs[key]

    def decode_buffers(self):
        """Buffers of the fused one-token step."""
        import torch
        from . import moe_layer_decode_ws_size
        if "decode" not in self._bufs:
            n = moe_layer_decode_ws_size(self.E, self.k, self.I)
            d = self.device
            self._bufs["decode"] = dict(
                ws=torch.zeros(n, dtype=torch.uint8, device=d), ws_bytes=n,
                ids=torch.empty(_round_up(self.k, 4), dtype=torch.int32, device=d),
                w=torch.empty(_round_up(self.k, 4), dtype=torch.float32, device=d),
                logits=torch.empty(self.E, dtype=torch.float32, device=d),
                y=torch.empty(self.H, dtype=torch.float32, device=d))
        return self._bufs["decode"]

    def forward_decode(self, x, x_dtype, logits_in=None, stream=None, bufs=None):
        """One token [1, H] through the fused decode step; returns the buffer dict (y in ["y"])."""
        from . import moe_layer_decode
        b = bufs or self.decode_buffers()
        moe_layer_decode(self.bits, x, x_dtype, None if logits_in is not None else self.w_router, self.w_dtype,
                         self.bias, logits_in, self.table, self.shared, self.H, self.I, self.E, self.k, b["ids"],
                         b["w"], b["logits"], b["y"], b["ws"], b["ws_bytes"], stream)
        return b

    def decode_session(self, x_host, x_dtype, y_host, stream, ids_host=None, bufs=None):
        """A DecodeSession over page-locked host buffers x_host [H] (x_dtype)
        and y_host [H] fp32 (ids_host [k] int32 optional): each run() copies x
        in, runs the step and copies y back, replaying one CUDA graph recorded
        on `stream` (a torch.cuda.Stream, not the default stream).  Creation
        runs the step once on x_host's current contents, so it should hold a
        valid token (or the device error word may report it)."""
        import torch
        b = bufs or self.decode_buffers()
        x_dev = torch.empty(self.H, dtype=torch.bfloat16 if x_host.dtype == torch.bfloat16 else torch.float32,
                            device=self.device)
        return DecodeSession(self, x_host, x_dtype, y_host, ids_host, x_dev, b, stream)

    def prepare_decode(self, x, x_dtype, stream=None, bufs=None):
        """A prepared one-token step on fixed buffers: every argument of
        moe_layer_decode is marshalled once, so each call of the returned
        function is one C call (the step reads x from the same device buffer
        and runs on the stream given, or current, at preparation)."""
        from . import _check, _p, _stream, lib
        b = bufs or self.decode_buffers()
        fn = lib().moe_layer_decode
        args = (self.bits, _p(x), x_dtype, _p(self.w_router), self.w_dtype, _p(self.bias), None, _p(self.table),
                _p(self.shared), self.H, self.I, self.E, self.k, _p(b["ids"]), _p(b["w"]), _p(b["logits"]),
                _p(b["y"]), _p(b["ws"]), b["ws_bytes"], _stream(stream))

        def step():
            rc = fn(*args)
            if rc:
                _check(rc)
            return b
        return step

    def forward(self, x, x_dtype, T=None, mode=0, logits_in=None, stream=None, bufs=None):
        """x: device tensor [T, H] (float32 or bfloat16); returns the StepBuffers (y in bufs.y)."""
        from . import moe_combine, moe_expert_ffn_q2, moe_expert_ffn_q4, moe_permute, moe_route_topk
        T = x.shape[0] if T is None else T
        b = bufs or self.buffers(T, mode)
        E, k, H, I = self.E, self.k, self.H, self.I
        moe_route_topk(x, x_dtype, None if logits_in is not None else self.w_router, self.w_dtype, logits_in,
                       self.bias, T, H, E, k, b.ids, b.w, b.logits, b.ws_route, b.sizes["route"], stream)
        moe_permute(b.ids, T, k, E, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"],
                    stream)
        ffn = moe_expert_ffn_q4 if self.bits == 4 else moe_expert_ffn_q2
        ffn(self.table, b.offsets, b.active, b.perm_src, x, x_dtype, T, k, H, I, E, self.shared, b.y_perm,
            b.y_shared, mode, b.ws_ffn, b.sizes["ffn"], stream)
        moe_combine(b.y_perm, b.perm_dst, b.w, b.y_shared, T, k, H, b.y, stream)
        return b


class DecodeSession:
    """Handle around moe_decode_session_* (keeps the buffers it records alive)."""

    def __init__(self, layer, x_host, x_dtype, y_host, ids_host, x_dev, bufs, stream):
        import ctypes as C
        from . import _check, _p, lib
        self._keep = (layer, x_host, y_host, ids_host, x_dev, bufs, stream)
        h = C.c_void_p()
        _check(lib().moe_decode_session_create(
            layer.bits, _p(x_host), x_dtype, _p(layer.w_router), layer.w_dtype, _p(layer.bias), _p(layer.table),
            _p(layer.shared), layer.H, layer.I, layer.E, layer.k, _p(y_host), _p(ids_host), _p(x_dev), _p(bufs["ids"]),
            _p(bufs["w"]), _p(bufs["y"]), _p(bufs["ws"]), bufs["ws_bytes"], stream.cuda_stream, C.byref(h)))
        self.h = h

    def run(self):
        from . import _check, lib
        _check(lib().moe_decode_session_run(self.h))

    def close(self):
        from . import lib
        if self.h:
            lib().moe_decode_session_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
