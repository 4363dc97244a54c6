"""Pins for the oracle's NF4 codebook and scalar encoder.

The pages say the 16 NF4 levels sit at quantiles of N(0,1), are normalised
to [-1, 1] by the block absmax, and are denser near zero than uniform INT4
("QLoRA Guide", NF4 vs uniform INT4; "Qlora Expert", Core Concept).  They
print no level values, so the values are pinned against an independent
library inverse-normal (scipy), not against the oracle itself.
"""
import math
import os

import numpy as np
import pytest
from scipy import special, stats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _page_figures():
    out = {}
    with open(os.path.join(GOLDEN, "page_figures.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = [s.strip() for s in line.split("=")]
                out[k] = float(v)
    return out


def test_ppnd16_matches_library_inverse_normal(oracle_mod):
    # AS 241 against scipy's ndtri over the whole range used and beyond.
    ps = np.concatenate([np.linspace(1e-12, 1e-6, 50), np.linspace(1e-6, 1 - 1e-6, 2001),
                         1 - np.linspace(1e-12, 1e-6, 50)])
    for p in ps:
        a = oracle_mod.ppnd16(p)
        b = special.ndtri(p)
        assert abs(a - b) <= 1e-14 * max(1.0, abs(b)), (p, a, b)
    # closed forms
    assert oracle_mod.ppnd16(0.5) == 0.0
    assert abs(oracle_mod.ppnd16(0.975) - 1.959963984540054) < 1e-14
    assert abs(oracle_mod.ppnd16(0.8413447460685429) - 1.0) < 1e-14


def test_codebook_against_scipy_construction(oracle_mod):
    v64, v32 = oracle_mod.codebook()
    delta = 0.5 * ((1 - 1 / 32) + (1 - 1 / 30))
    pos = stats.norm.ppf(np.linspace(delta, 0.5, 9)[:-1])
    neg = -stats.norm.ppf(np.linspace(delta, 0.5, 8)[:-1])
    ref = np.sort(np.concatenate([pos, [0.0], neg]))
    ref = ref / ref.max()
    assert np.allclose(v64, ref, rtol=0, atol=1e-14)
    assert np.array_equal(v32, ref.astype(np.float32))


def test_codebook_invariants(oracle_mod):
    figs = _page_figures()
    v64, L = oracle_mod.codebook()
    assert L.size == int(figs["nf4_levels"]) == 16
    assert np.all(np.diff(L) > 0), "levels must be strictly increasing"
    assert L[0] == -1.0 and L[15] == 1.0 and L[7] == 0.0
    assert np.count_nonzero(L > 0) == 8 and np.count_nonzero(L < 0) == 7
    gaps = np.diff(L.astype(np.float64))
    # denser near zero than in the tails on each side (normal quantiles)
    assert np.all(np.diff(gaps[7:]) > 0) and np.all(np.diff(gaps[:7]) < 0)
    # and denser near zero than uniform INT4's step of 2/15
    assert gaps[7] < 2 / 15 and gaps[6] < 2 / 15
    assert abs(gaps.min() - 0.0796) < 1e-4 and abs(gaps.max() - 0.3038) < 1e-4


def test_codebook_regression_fixture(oracle_mod):
    _, L = oracle_mod.codebook()
    with open(os.path.join(GOLDEN, "nf4_codebook_reading.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 16
    for i, (idx, _, hx) in enumerate(rows):
        assert int(idx) == i
        assert np.float32(L[i]).view(np.uint32) == int(hx, 16)


def test_every_level_round_trips(oracle_mod):
    _, L = oracle_mod.codebook()
    m = oracle_mod.midpoints(L)
    for i in range(16):
        assert oracle_mod.encode_value(float(L[i]), m) == i


def test_encoder_is_nearest_level_brute_force(oracle_mod):
    _, L = oracle_mod.codebook()
    m = oracle_mod.midpoints(L)
    rng = np.random.default_rng(1234)
    xs = np.concatenate([rng.uniform(-1, 1, 4000), rng.normal(0, 0.3, 2000).clip(-1, 1)]).astype(np.float32)
    L64 = L.astype(np.float64)
    for x in xs:
        d = np.abs(float(x) - L64)
        best = int(np.argmin(d))
        q = oracle_mod.encode_value(float(x), m)
        # only a value within one fp32 ulp of a decision threshold may differ
        near = np.min(np.abs(m.astype(np.float64) - float(x))) <= np.spacing(np.float32(abs(x) + 1e-30))
        if not near:
            assert q == best, (x, q, best)
        else:
            assert abs(q - best) <= 1


def test_ties_go_to_lower_index(oracle_mod):
    _, L = oracle_mod.codebook()
    m = oracle_mod.midpoints(L)
    for i in range(15):
        mi = np.float32(m[i])
        assert oracle_mod.encode_value(float(mi), m) == i
        assert oracle_mod.encode_value(float(np.nextafter(mi, np.float32(np.inf))), m) == i + 1
        assert oracle_mod.encode_value(float(np.nextafter(mi, np.float32(-np.inf))), m) == i
        # the threshold lies strictly between its two levels
        assert L[i] < mi < L[i + 1]


def test_encode_error_bound(oracle_mod):
    _, L = oracle_mod.codebook()
    m = oracle_mod.midpoints(L)
    half_gap = np.diff(L.astype(np.float64)).max() / 2
    for x in np.linspace(-1, 1, 3001, dtype=np.float32):
        q = oracle_mod.encode_value(float(x), m)
        assert abs(float(x) - float(L[q])) <= half_gap + 1e-7


def test_bf16_rounding_is_round_to_nearest_even(oracle_mod):
    # the bf16 rounding used by dequantization, against torch's conversion
    import torch
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 2000), [0.0, -0.0, 1.0, -1.0,
                           1.00390625, 1.01171875, 3.0e38, 1e-39]]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.f32_to_bf16_scalar(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)
    # exact ties: 1 + 2^-8 sits halfway between bf16 1.0 and 1.0078125 -> even (1.0)
    assert oracle_mod.f32_to_bf16_scalar(1.00390625) == 0x3F80
    assert oracle_mod.f32_to_bf16_scalar(1.01171875) == 0x3F82


def test_lora_scaling_page_example(oracle_mod):
    figs = _page_figures()
    s = oracle_mod.lora_scaling(int(figs["lora_r_example"]), figs["lora_alpha_example"])
    assert s == figs["lora_scaling_example"] == 0.25
    assert oracle_mod.lora_scaling(16, 32) == 2.0
    assert math.isclose(oracle_mod.lora_scaling(16, 32), 32 / 16)


@pytest.mark.parametrize("p", [0.5, 0.6, 0.9, 0.9677083333333334])
def test_ppnd16_inverts_erfc(oracle_mod, p):
    x = oracle_mod.ppnd16(p)
    assert abs(0.5 * math.erfc(-x / math.sqrt(2)) - p) < 1e-15
