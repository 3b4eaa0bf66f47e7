"""Pins for the oracle's number formats, block dequantisation and blob parsing.

Everything here is checked against something other than the oracle: numpy's
and torch's own float16/bfloat16 conversions, values worked out by hand
(tests/golden/dequant_blocks.txt), the byte sizes the pages print, and exact
round trips through weights that are representable by construction.
"""
from pathlib import Path

import numpy as np
import pytest
import torch

import workloads as W

GOLDEN = Path(__file__).parent / "golden"


def test_fp16_decode_all_patterns(oracle_lib):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle_lib.fp16_to_double(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decode_against_torch(oracle_lib):
    rng = np.random.default_rng(5)
    pats = np.concatenate([rng.integers(0, 65536, 4000), [0, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x7F7F]])
    pats = pats.astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle_lib.bf16_to_double(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _golden_blocks():
    rows = []
    for line in (GOLDEN / "dequant_blocks.txt").read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        left, right = line.split("|")
        bits, scale, codes = left.split()
        vals = []
        for tok in right.split(","):
            tok = tok.strip()
            if "x" in tok:
                v, n = tok.rsplit("x", 1)
                vals += [float(v)] * int(n)
            else:
                vals.append(float(tok))
        rows.append((int(bits), int(scale, 16), bytes.fromhex(codes), vals))
    return rows


@pytest.mark.parametrize("row", _golden_blocks(), ids=lambda r: f"q{r[0]}-{r[1]:04x}-{r[2].hex()[:8]}")
def test_dequant_hand_built_blocks(oracle_lib, row):
    bits, scale, codes, vals = row
    assert len(codes) == 4 * bits
    assert len(vals) == 32
    got = oracle_lib.dequant_block(bits, np.frombuffer(codes, np.uint8), scale)
    assert np.array_equal(got, np.array(vals))


def test_blob_bytes_match_pages(oracle_lib):
    # 27B dense report: Q4_0 costs 0.5625 B per value.  Q2_0 by the same block
    # rule: 8 B of codes + 2 B of scale per 32 values = 0.3125 B per value.
    H, I = 2048, 512
    n = 3 * H * I
    assert oracle_lib.blob_bytes(4, H, I) == 1_769_472
    assert oracle_lib.blob_bytes(4, H, I) / n == 0.5625
    assert oracle_lib.blob_bytes(2, H, I) == 983_040
    assert oracle_lib.blob_bytes(2, H, I) / n == 0.3125
    assert oracle_lib.blob_bytes(4, H, I) == W.blob_bytes(4, H, I)


def _representable(rng, bits, rows, cols):
    """Weights d*(q - 2^(b-1)) whose packing is exact: every block holds code 0."""
    half = 1 << (bits - 1)
    nb = cols // 32
    q = rng.integers(0, 1 << bits, size=(rows, nb, 32))
    q[:, :, 0] = 0                                     # the block minimum -half*d
    perm = rng.permuted(np.tile(np.arange(32), (rows, nb, 1)), axis=2)
    q = np.take_along_axis(q, perm, axis=2)
    d = W.round_significant(rng.uniform(0.001, 0.05, size=(rows, nb)), 8)
    d = d.astype(np.float16).astype(np.float64)
    return (d[..., None] * (q - half)).reshape(rows, cols)


@pytest.mark.parametrize("bits", [4, 2])
def test_blob_parse_orientation_exact(oracle_lib, bits):
    """Hand-chosen representable matrices survive pack -> oracle parse exactly,
    which pins the byte offsets and orientation of Wg, Wu and Wd."""
    rng = np.random.default_rng(11 + bits)
    H, I = 128, 64
    Wg = _representable(rng, bits, I, H)
    Wu = _representable(rng, bits, I, H)
    Wd = _representable(rng, bits, H, I)
    blob = W.assemble_blob(bits, H, I, Wg, Wu, Wd, scale_sig_bits=8)
    g, u, d = oracle_lib.expert_weights(bits, H, I, blob)
    assert np.array_equal(g, Wg)
    assert np.array_equal(u, Wu)
    assert np.array_equal(d, Wd)


@pytest.mark.parametrize("bits", [4, 2])
def test_packer_error_bound(oracle_lib, bits):
    """Gaussian weights: |w - dequant| <= |d|/2 except where the code clamps."""
    rng = np.random.default_rng(3)
    H, I = 256, 128
    Wg = rng.standard_normal((I, H)) * 0.02
    Wu = rng.standard_normal((I, H)) * 0.02
    Wd = rng.standard_normal((H, I)) * 0.02
    blob = W.assemble_blob(bits, H, I, Wg, Wu, Wd, scale_sig_bits=11)
    g, _, _ = oracle_lib.expert_weights(bits, H, I, blob)
    half = 1 << (bits - 1)
    wb = Wg.reshape(I, H // 32, 32)
    amax = np.abs(wb).max(axis=2, keepdims=True)
    d = amax / half
    err = np.abs(g.reshape(wb.shape) - wb)
    # elements on the side opposite the block maximum can clamp at (half-1)*d
    inside = np.abs(wb) <= (half - 1) * d
    assert np.all(err[inside] <= d.repeat(32, 2)[inside] * 0.5 * (1 + 2 ** -9) + 1e-12)
