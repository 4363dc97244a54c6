"""Pins for the oracle's block quantization, double quantization and dequant.

Pinned against closed forms the pages fix (64-value blocks, 8-bit constants,
the ~0.37 bit saving, the 4x size against 16-bit), brute force on tiny
inputs, and invariants of the construction.
"""
import math
import os

import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _figs():
    out = {}
    with open(os.path.join(GOLDEN, "page_figures.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = [s.strip() for s in line.split("=")]
                out[k] = float(v)
    return out


def _bits(a_f32):
    return torch.from_numpy(np.asarray(a_f32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _unpack(packed):
    hi = (packed >> 4) & 0xF
    lo = packed & 0xF
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = hi
    out[..., 1::2] = lo
    return out


def test_overhead_closed_form(oracle_mod):
    figs = _figs()
    bs = int(figs["nf4_block_size"])
    for (N, K) in [(4096, 4096), (11008, 4096), (4096, 11008), (8192, 8192), (28672, 8192), (8192, 28672)]:
        nblocks = N * K // bs
        G = math.ceil(nblocks / 256)
        assert nblocks % 256 == 0  # all workload shapes fill whole groups
        before = figs["dq_constant_bits_before"] * nblocks / (N * K)
        after = (figs["dq_constant_bits_after"] * nblocks + 64 * G) / (N * K)
        assert before == 0.5
        assert after == 0.12890625
        assert round(before - after, 2) == figs["dq_saving_bits_per_param"]
        assert 4 + after == 4.12890625
    # 7B parameters: 16-bit 14 GB -> 4-bit 3.5 GB ("4x")
    p7 = 7e9
    assert p7 * 16 / 8 / 1e9 == figs["fp16_bytes_7b_gb"]
    assert p7 * 4 / 8 / 1e9 == figs["nf4_bytes_7b_gb"]
    assert figs["fp16_bytes_7b_gb"] / figs["nf4_bytes_7b_gb"] == figs["compression_vs_16bit"]


def test_storage_sizes_from_oracle_output(oracle_mod):
    W = inputs.weight(9, 0, 64, 512, 0.02)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    N, K = 64, 512
    assert q["packed"].nbytes * 8 == 4 * N * K
    bits = (q["codes"].nbytes + q["scale"].nbytes + q["mean"].nbytes) * 8
    assert bits / (N * K) == 0.12890625


def test_zero_block_and_packing_order(oracle_mod):
    _, L = oracle_mod.codebook()
    w = np.zeros((2, 64), np.float32)
    w[1, 0] = 1.0       # -> level 15 in the high nibble of byte 0
    w[1, 1] = -1.0      # -> level 0 in the low nibble of byte 0
    w[1, 2] = 0.0       # -> level 7
    w[1, 3] = float(L[9])
    q = oracle_mod.quantize_dq(_bits(w))
    assert np.all(q["packed"][0] == 0x77)
    assert q["packed"][1, 0] == 0xF0
    assert q["packed"][1, 1] == 0x79
    assert q["absmax"][0] == 0.0 and q["absmax"][1] == 1.0


def test_brute_force_tiny(oracle_mod):
    _, L = oracle_mod.codebook()
    m = oracle_mod.midpoints(L).astype(np.float64)
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, (3, 192)).astype(np.float32)
    w[0, :64] = 0.0
    wb = _bits(w)
    wf = oracle_mod.bf16_to_f32(wb).reshape(-1, 64)
    q = oracle_mod.quantize_dq(wb)
    nib = _unpack(q["packed"]).reshape(-1, 64)
    c = np.abs(wf).max(axis=1)
    assert np.array_equal(c, q["absmax"])
    for b in range(wf.shape[0]):
        for j in range(64):
            if c[b] == 0:
                assert nib[b, j] == 7
                continue
            x = np.float32(wf[b, j]) / np.float32(c[b])      # IEEE fp32 division
            best = int(np.argmin(np.abs(float(x) - L.astype(np.float64))))
            if np.min(np.abs(m - float(x))) > 1e-6:
                assert nib[b, j] == best


def test_codebook_valued_blocks_round_trip_exactly(oracle_mod):
    _, L = oracle_mod.codebook()
    # every block holds the 16 levels times the same power of two, so every
    # group has one constant: mean = c, scale = 0, code = 0, c' = c.
    c = 0.03125
    base = np.tile(np.concatenate([L, L[::-1], L, L[::-1]]), 512)  # 64 per block
    w = (base * c).astype(np.float32).reshape(16, 2048)
    wb = _bits(w)
    q = oracle_mod.quantize_dq(wb)
    assert np.all(q["scale"] == 0) and np.all(q["codes"] == 0) and np.all(q["mean"] == np.float32(c))
    nib = _unpack(q["packed"]).reshape(-1)
    want = np.tile(np.concatenate([np.arange(16), np.arange(16)[::-1]] * 2), 512)
    assert np.array_equal(nib, want)
    back = oracle_mod.dequant(q)
    assert np.array_equal(back, wb)


def test_double_quant_invariants(oracle_mod):
    W = inputs.weight(9, 1, 96, 4096, 0.02, t4_mix=0.1)   # 6144 blocks = 24 groups
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    c = q["absmax"].astype(np.float64)
    codes = q["codes"].astype(np.int64)
    assert codes.min() >= -127 and codes.max() <= 127
    for g in range(q["scale"].size):
        sl = slice(256 * g, 256 * (g + 1))
        cg = c[sl]
        sc, mu = float(q["scale"][g]), float(q["mean"][g])
        # mean: within one fp32 ulp of the exact average
        exact = math.fsum(cg) / cg.size
        assert abs(mu - exact) <= np.spacing(np.float32(exact))
        assert sc > 0
        assert np.max(np.abs(codes[sl])) == 127
        cprime = np.array([oracle_mod.block_constant(int(k), sc, mu) for k in codes[sl]])
        err = np.abs(cprime - cg)
        assert np.all(err <= sc / 2 + 2 * np.spacing(np.float32(cg.max()))), err.max()


def test_short_last_group(oracle_mod):
    # 5 blocks: one group of 5 constants
    W = inputs.weight(9, 2, 5, 64, 0.02)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    assert q["scale"].size == 1 and q["codes"].size == 5
    exact = math.fsum(q["absmax"].astype(np.float64)) / 5
    assert abs(float(q["mean"][0]) - exact) <= np.spacing(np.float32(exact))


def test_dequant_error_bound_and_idempotence(oracle_mod):
    _, L = oracle_mod.codebook()
    half_gap = np.diff(L.astype(np.float64)).max() / 2
    W = inputs.weight(9, 3, 64, 1024, 0.02, outlier_frac=0.001)
    wb = inputs.bf16_bits(W)
    q = oracle_mod.quantize_dq(wb)
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q)).astype(np.float64).reshape(-1, 64)
    wf = oracle_mod.bf16_to_f32(wb).astype(np.float64).reshape(-1, 64)
    c = q["absmax"].astype(np.float64)[:, None]
    g = np.arange(c.shape[0]) // 256
    cprime = np.array([oracle_mod.block_constant(int(k), float(q["scale"][gg]), float(q["mean"][gg]))
                       for k, gg in zip(q["codes"], g)])[:, None]
    bound = half_gap * c + np.abs(cprime - c) + 2.0 ** -8 * np.abs(cprime)
    assert np.all(np.abs(Wd - wf) <= bound + 1e-12)
    # re-quantizing the dequantized weight reproduces the nibbles
    q2 = oracle_mod.quantize_dq(oracle_mod.dequant(q))
    assert np.array_equal(q2["packed"], q["packed"])


def test_dequant_rows_matches_full(oracle_mod):
    W = inputs.weight(9, 4, 40, 320, 0.02)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    full = oracle_mod.dequant(q)
    rows = [0, 7, 39, 13]
    assert np.array_equal(oracle_mod.dequant_rows(q, rows), full[rows])


def test_rejects_bad_shapes(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.quantize_dq(np.zeros((2, 96), np.uint16))
