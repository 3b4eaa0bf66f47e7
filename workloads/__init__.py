"""Seeded synthetic inputs for the quantized MoE expert step.

This module only draws random numbers and lays bytes out.  It holds none of
the step's arithmetic (no routing, no dequantisation, no FFN): the oracle and
the CUDA library each read the bytes made here with their own code.

Sources for the shapes and distributions (the pages print no weights):

* Strata article, section 2 item 1 and the 30-second summary table: 10 of
  24,576 experts active per token.
* Strata code review, section 4: 512 experts per layer.
* 27B dense report (trawling.dev), model-file paragraph: a Q4_0 value costs
  0.5625 B, i.e. 32 four-bit codes plus one fp16 scale per block.
* Strata article, summary table: the Q2_0 size (two-bit codes, same block).
* Strata article, section 2 item 3: verify windows of a few drafted tokens and
  prompt chunks of up to 8,192 tokens.

Expert blob layout (one contiguous blob per expert, so a cache miss is one
copy).  With b bits per code and block length 32:

    codes W_g  [I rows][H/32 blocks][4*b bytes]
    codes W_u  [I rows][H/32 blocks][4*b bytes]
    codes W_d  [H rows][I/32 blocks][4*b bytes]
    scales W_g [I][H/32] fp16, scales W_u [I][H/32] fp16, scales W_d [H][I/32] fp16

4-bit block (16 B): element i sits in byte i % 16, low nibble for i < 16 and
high nibble for i >= 16.  2-bit block (8 B): element i sits in byte i % 8 at
bit 2*(i // 8).  A weight is d * (q - 2**(b-1)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BLOCK = 32


# --------------------------------------------------------------------------
# number formats (bit patterns only)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_significant(d: np.ndarray, sig_bits: int) -> np.ndarray:
    """Round float64 values to `sig_bits` significant bits (ties to even)."""
    m, e = np.frexp(d)
    return np.ldexp(np.round(m * (1 << sig_bits)) / (1 << sig_bits), e)


# --------------------------------------------------------------------------
# block packer (input preparation: turns Gaussian weights into blobs)
# --------------------------------------------------------------------------
def pack_matrix(w: np.ndarray, bits: int, scale_sig_bits: int = 8):
    """Pack a [rows, cols] float matrix into b-bit blocks of 32 along cols.

    Per block: m = the element of largest magnitude (sign kept),
    d = fp16(m / -2**(b-1)) rounded to `scale_sig_bits` significant bits,
    q = clamp(rint(w / d), -2**(b-1), 2**(b-1) - 1) + 2**(b-1).
    An all-zero block gets d = 0 and q = 2**(b-1).  With scale_sig_bits <= 8
    every product d * (q - 2**(b-1)) is exact in fp16; 11 keeps plain fp16.

    Returns (codes uint8 [rows, cols/32 * 4*bits], scales uint16 [rows, cols/32]).
    """
    assert bits in (2, 4)
    rows, cols = w.shape
    assert cols % BLOCK == 0
    nb = cols // BLOCK
    half = 1 << (bits - 1)
    wb = w.reshape(rows, nb, BLOCK).astype(np.float32)
    idx = np.argmax(np.abs(wb), axis=2)
    m = np.take_along_axis(wb, idx[..., None], axis=2)[..., 0].astype(np.float64)
    d = m / -half
    if scale_sig_bits < 11:
        d = round_significant(d, scale_sig_bits)
    d16 = d.astype(np.float16)
    d32 = d16.astype(np.float32)
    safe = np.where(d32 == 0, np.float32(1), d32)
    q = np.rint(wb / safe[..., None])
    q = np.clip(q, -half, half - 1)
    q = np.where((d32 == 0)[..., None], 0, q) + half
    q = q.astype(np.uint8)
    if bits == 4:
        lo = q[..., :16]
        hi = q[..., 16:]
        codes = (lo | (hi << 4)).astype(np.uint8)           # [rows, nb, 16]
    else:
        c = q.reshape(rows, nb, 4, 8)                         # [.., crumb, byte]
        codes = (c[:, :, 0] | (c[:, :, 1] << 2) | (c[:, :, 2] << 4) | (c[:, :, 3] << 6)).astype(np.uint8)
    return codes.reshape(rows, nb * 4 * bits), d16.view(np.uint16)


def blob_bytes(bits: int, H: int, I: int) -> int:
    codes = 3 * I * H * bits // 8
    scales = 3 * I * H // BLOCK * 2
    return codes + scales


def assemble_blob(bits: int, H: int, I: int, Wg, Wu, Wd, scale_sig_bits: int = 8) -> np.ndarray:
    """Wg, Wu: [I, H]; Wd: [H, I] (rows are output features, cols the reduction)."""
    cg, sg = pack_matrix(Wg, bits, scale_sig_bits)
    cu, su = pack_matrix(Wu, bits, scale_sig_bits)
    cd, sd = pack_matrix(Wd, bits, scale_sig_bits)
    parts = [cg.ravel(), cu.ravel(), cd.ravel(),
             sg.ravel().view(np.uint8), su.ravel().view(np.uint8), sd.ravel().view(np.uint8)]
    blob = np.concatenate(parts)
    assert blob.size == blob_bytes(bits, H, I)
    return blob


def random_expert_blob(rng: np.random.Generator, bits: int, H: int, I: int,
                       sigma: float, scale_sig_bits: int = 8) -> np.ndarray:
    Wg = rng.standard_normal((I, H), dtype=np.float32) * np.float32(sigma)
    Wu = rng.standard_normal((I, H), dtype=np.float32) * np.float32(sigma)
    Wd = rng.standard_normal((H, I), dtype=np.float32) * np.float32(sigma)
    return assemble_blob(bits, H, I, Wg, Wu, Wd, scale_sig_bits)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclass
class Layer:
    bits: int
    H: int
    I: int
    E: int
    k: int
    blobs: np.ndarray                  # uint8 [E, blob_bytes]
    shared: np.ndarray | None          # uint8 [blob_bytes] or None
    w_router: np.ndarray | None        # [E, H] float32 or uint16 (bf16 bits)
    w_dtype: str                       # "f32" | "bf16"
    bias: np.ndarray | None = None     # [E] float32
    meta: dict = field(default_factory=dict)


def make_layer(seed: int, bits: int, H: int, I: int, E: int, k: int, *, shared: bool,
               sigma_w: float = 0.02, sigma_r: float = 0.1, w_dtype: str = "bf16",
               scale_sig_bits: int = 8, bias: np.ndarray | None = None,
               distinct_experts: int | None = None) -> Layer:
    """One MoE layer of E packed experts (+ optional shared expert) and a router.

    distinct_experts: draw only that many experts and repeat them cyclically
    (used for the 24,576-expert paging pool, where only bytes moved matter).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    nb = blob_bytes(bits, H, I)
    n_draw = E if distinct_experts is None else min(E, distinct_experts)
    base = np.empty((n_draw, nb), dtype=np.uint8)
    for e in range(n_draw):
        base[e] = random_expert_blob(rng, bits, H, I, sigma_w, scale_sig_bits)
    if n_draw == E:
        blobs = base
    else:
        blobs = np.empty((E, nb), dtype=np.uint8)
        for e in range(E):
            blobs[e] = base[e % n_draw]
    sh = random_expert_blob(rng, bits, H, I, sigma_w, scale_sig_bits) if shared else None
    wr = rng.standard_normal((E, H), dtype=np.float32) * np.float32(sigma_r)
    if w_dtype == "bf16":
        wr = f32_to_bf16_bits(wr)
    return Layer(bits, H, I, E, k, blobs, sh, wr, w_dtype, bias,
                 meta=dict(seed=seed, sigma_w=sigma_w, sigma_r=sigma_r,
                           scale_sig_bits=scale_sig_bits))


def make_tokens(seed: int, T: int, H: int, dtype: str = "bf16") -> np.ndarray:
    """x ~ N(0, 1), [T, H]; float32 or bf16 bits (uint16)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((T, H), dtype=np.float32)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


def zipf_log_popularity(seed: int, E: int, s: float = 1.1) -> np.ndarray:
    """ln p_e with p_e proportional to rank**-s over a seeded rank permutation."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rank = rng.permutation(E) + 1
    p = rank.astype(np.float64) ** (-s)
    p /= p.sum()
    return np.log(p)


# The five workloads (sizes from the pages, see module docstring).
TINY = dict(bits=4, H=256, I=128, E=16, k=2, T=8, shared=False, x_dtype="f32",
            w_dtype="f32", sigma_w=0.02, sigma_r=0.1)
DECODE = dict(bits=4, H=2048, I=512, E=512, k=10, T=1, steps=1000, shared=True,
              x_dtype="bf16", w_dtype="bf16", sigma_w=0.02, sigma_r=0.1)
VERIFY = dict(bits=2, H=2048, I=512, E=512, k=10, windows=(2, 3, 5, 9, 16),
              windows_each=200, shared=True, x_dtype="bf16", w_dtype="bf16",
              sigma_w=0.02, sigma_r=1.0 / math.sqrt(2048), zipf_s=1.1)
PREFILL = dict(bits=4, H=2048, I=512, E=512, k=10, chunks=(512, 2048, 8192),
               shared=True, x_dtype="bf16", w_dtype="bf16", sigma_w=0.02, sigma_r=0.1)
PAGING = dict(bits=2, H=2048, I=512, E=24576, k=10, capacity=2048, steps=5000,
              drift_every=200, drift_prob=0.1, hot=2048, zipf_s=1.1, shared=False,
              x_dtype="bf16", sigma_w=0.02)

# Model-scale paging: 48 layers x 512 experts = the 24,576-expert pool, 10
# experts per layer per token (480 accesses per token), one HBM cache.
PAGING48 = dict(bits=2, H=2048, I=512, layers=48, experts_per_layer=512, k=10, capacity=2048, tokens=100,
                drift_every=50, drift_prob=0.1, hot_per_layer=42, zipf_s=1.1, prefetch=10)

# Three tiers: every expert in a file on the drive, the most used in a
# page-locked RAM tier, the hottest in HBM (the pages' SSD -> RAM -> VRAM
# picture at a size whose file a test box can write in seconds).
PAGING_SSD = dict(bits=2, H=2048, I=512, E=4096, k=10, hbm_slots=512, ram_slots=1536, steps=2000,
                  drift_every=200, drift_prob=0.1, hot=512, zipf_s=1.1, io_threads=8)

SEED = {"tiny": 1001, "decode": 1002, "verify": 1003, "prefill": 1004, "paging": 1005, "paging48": 1006,
        "paging_ssd": 1007}


def tiny_case(seed: int = SEED["tiny"], **over):
    c = dict(TINY, **over)
    layer = make_layer(seed, c["bits"], c["H"], c["I"], c["E"], c["k"], shared=c["shared"],
                       sigma_w=c["sigma_w"], sigma_r=c["sigma_r"], w_dtype=c["w_dtype"])
    x = make_tokens(seed + 7, c["T"], c["H"], c["x_dtype"])
    return layer, x


def verify_layer(seed: int = SEED["verify"], **over) -> Layer:
    c = dict(VERIFY, **over)
    lnp = zipf_log_popularity(seed + 11, c["E"], c["zipf_s"]).astype(np.float32)
    return make_layer(seed, c["bits"], c["H"], c["I"], c["E"], c["k"], shared=c["shared"],
                      sigma_w=c["sigma_w"], sigma_r=c["sigma_r"], w_dtype=c["w_dtype"],
                      bias=lnp)


def paging_trace(seed: int, E: int, k: int, steps: int, *, s: float = 1.1,
                 drift_every: int = 200, drift_prob: float = 0.1, hot: int = 2048):
    """Per-step router logits ln p_e + G_e (G standard Gumbel) with drifting popularity.

    Every `drift_every` steps each of the `hot` most popular ranks swaps its
    expert with a uniformly drawn cold expert with probability `drift_prob`.
    Yields float32 logits [E] per step (the top-k of these is a Gumbel-top-k
    draw of k distinct experts in proportion to p).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    order = rng.permutation(E)                     # order[r] = expert at rank r
    p = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    lnp_rank = np.log(p / p.sum())
    lnp = np.empty(E)
    for st in range(steps):
        if st % drift_every == 0 and st > 0:
            for r in range(hot):
                if rng.random() < drift_prob:
                    c = int(rng.integers(hot, E))
                    order[r], order[c] = order[c], order[r]
        lnp[order] = lnp_rank
        g = rng.gumbel(size=E)
        yield (lnp + g).astype(np.float32)


def paging48_trace(seed: int, layers: int, experts: int, tokens: int, *, s: float = 1.1, drift_every: int = 50,
                   drift_prob: float = 0.1, hot: int = 42):
    """Per-token router logits of every layer, [layers, experts] float32 per
    token: ln p + G with G standard Gumbel, p a Zipf(s) popularity over a
    seeded rank order of each layer's experts.  Every `drift_every` tokens
    each of a layer's `hot` most popular ranks swaps its expert with a
    uniformly drawn colder one with probability `drift_prob`."""
    rng = np.random.Generator(np.random.PCG64(seed))
    order = np.stack([rng.permutation(experts) for _ in range(layers)])
    p = (np.arange(1, experts + 1, dtype=np.float64)) ** (-s)
    lnp_rank = np.log(p / p.sum())
    lnp = np.empty((layers, experts))
    for t in range(tokens):
        if t % drift_every == 0 and t > 0:
            for l in range(layers):
                for r in range(hot):
                    if rng.random() < drift_prob:
                        c = int(rng.integers(hot, experts))
                        order[l, r], order[l, c] = order[l, c], order[l, r]
        for l in range(layers):
            lnp[l, order[l]] = lnp_rank
        g = rng.gumbel(size=(layers, experts))
        yield (lnp + g).astype(np.float32)
