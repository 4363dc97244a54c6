"""Pins for the oracle's FP4 codebook variant and its dequantize-and-merge.

FP4 ("Qlora Expert", Hyperparameter Guidance: quant type "nf4" or "fp4"):
the table is pinned against the E2M1 bit-field definition (sign, 2 exponent
bits with bias 1, 1 mantissa bit, subnormals at exponent 0), rebuilt here
from that definition; the encoder against a brute-force nearest level.

Merge ("Qlora Expert", Common Pitfalls: merging requires dequantization;
"QLoRA Implementation Details (2025 Edition)", Step 7: merge for inference):
B = 0 gives the plain dequantized weight, a rank-1 adapter has a closed form,
the LoRA sum is taken one fma per term in order (a case where order changes
the result), and the merged weight used as a dense layer reproduces the
forward of the quantized layer with its adapter.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _e2m1(code):
    """Value of a 4-bit E2M1 bit pattern from its fields."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * 0.5 * m                   # subnormal: 2^(1 - bias) * (m / 2), bias 1
    return s * 2.0 ** (e - 1) * (1.0 + 0.5 * m)


# --------------------------------------------------------------------------
# FP4 codebook
# --------------------------------------------------------------------------
def test_fp4_table_is_e2m1_over_its_max(oracle_mod):
    v64, v32 = oracle_mod.fp4_codebook()
    ref = np.array([_e2m1(c) for c in range(16)]) / max(_e2m1(c) for c in range(16))
    assert np.array_equal(v64, ref)
    assert np.array_equal(v32, ref.astype(np.float32))
    assert np.array_equal(oracle_mod.codebook_qt(1), v32)
    assert v32[7] == 1.0 and v32[15] == -1.0 and v32[0] == 0.0 and v32[8] == 0.0
    assert np.array_equal(v32[8:], -v32[:8])                      # sign bit is bit 3
    assert np.all(np.diff(v32[:8]) > 0)                            # magnitudes ascend with the code
    assert len(set(v32.tolist())) == 15                            # +0 and -0 coincide


def test_fp4_encoder_is_nearest_level(oracle_mod):
    L = oracle_mod.codebook_qt(1).astype(np.float64)
    levels = np.array(sorted(set(L.tolist())))
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.uniform(-1, 1, 4000), levels, [-1.0, 0.0, 1.0]]).astype(np.float32)
    mids = ((levels[:-1].astype(np.float32) + levels[1:].astype(np.float32)) * np.float32(0.5)).astype(np.float32)
    near = []
    for m in mids:                       # each threshold and its fp32 neighbours
        near += [np.nextafter(m, np.float32(-2)), m, np.nextafter(m, np.float32(2))]
    xs = np.concatenate([xs, np.array(near, np.float32)])
    for x in xs:
        q = oracle_mod.encode_value_qt(1, float(x))
        v = L[q]
        d = np.abs(levels - float(x))
        best = levels[np.argmin(d)]            # argmin takes the lower level on a tie
        if float(x) in mids:
            assert v == levels[np.searchsorted(levels, float(x)) - 1], x   # on a threshold: lower level
        else:
            assert v == best, (x, q, v, best)
        if v == 0.0:
            assert q == 0                      # zero is always +0
    # every level encodes to a code of that value
    for c in range(16):
        assert L[oracle_mod.encode_value_qt(1, float(L[c]))] == L[c]


def test_generic_quantizer_reproduces_nf4(oracle_mod):
    W = inputs.weight(7, 1, 48, 640, 0.02, outlier_frac=0.01)
    b = inputs.bf16_bits(W)
    q0 = oracle_mod.quantize_dq(b)
    q1 = oracle_mod.quantize_dq_qt(b, 0)
    for k in ("packed", "codes", "scale", "mean"):
        assert np.array_equal(q0[k], q1[k]), k
    assert np.array_equal(oracle_mod.dequant(q0), oracle_mod.dequant_qt(q1))
    rows = [0, 5, 47]
    assert np.array_equal(oracle_mod.dequant_rows(q0, rows), oracle_mod.dequant_qt(q1, rows))


def test_fp4_quantize_brute_force_tiny(oracle_mod):
    W = inputs.weight(8, 0, 4, 128, 0.02)
    b = inputs.bf16_bits(W)
    q = oracle_mod.quantize_dq_qt(b, 1)
    L = oracle_mod.codebook_qt(1).astype(np.float64)
    levels = np.array(sorted(set(L.tolist())))
    w = _f32(b).reshape(-1, 64)
    nib = np.empty(w.shape, np.int64)
    packed = q["packed"].reshape(-1)
    nib[:, :] = np.stack([(packed >> 4) & 15, packed & 15], -1).reshape(w.shape)
    for i in range(w.shape[0]):
        c = np.abs(w[i]).max()
        assert q["absmax"][i] == c
        x = (w[i] / np.float32(c)).astype(np.float32)
        for j in range(64):
            best = levels[np.argmin(np.abs(levels - float(x[j])))]
            assert L[nib[i, j]] == best
    # decoded values are the levels times the recovered block constants, rounded to bf16
    Wd = _f32(oracle_mod.dequant_qt(q)).reshape(-1, 64)
    cp = (q["codes"].astype(np.float64) * q["scale"][0] + q["mean"][0]).astype(np.float32)
    for i in range(w.shape[0]):
        assert np.array_equal(Wd[i], _f32(_bf16_bits((L[nib[i]].astype(np.float32) * cp[i]).astype(np.float32))))


def test_fp4_codebook_valued_blocks_round_trip(oracle_mod):
    """Blocks whose weights are bf16(L[q] c) with the block max exactly c encode back to the
    same codes (-0 comes back as +0): bf16 rounding (2^-9 relative) is far below half the
    smallest gap between levels (1/24)."""
    L = oracle_mod.codebook_qt(1)
    rng = np.random.default_rng(5)
    rows, want = [], []
    for c in (1.0, 0.25, 2.0 ** -10, 3.0):
        codes = rng.integers(0, 16, 64)
        codes[0] = 7                              # the block max: exactly c
        rows.append(L[codes] * np.float32(c))
        want.append(np.where(codes == 8, 0, codes))
    b = _bf16_bits(np.array(rows, np.float32))
    q = oracle_mod.quantize_dq_qt(b, 1)
    packed = q["packed"].reshape(-1)
    got = np.stack([(packed >> 4) & 15, packed & 15], -1).reshape(len(rows), 64)
    assert np.array_equal(got, np.array(want))


def test_fp4_zero_block(oracle_mod):
    b = np.zeros((2, 128), np.uint16)
    q = oracle_mod.quantize_dq_qt(b, 1)
    assert not q["packed"].any() and not q["codes"].any()
    assert np.all(_f32(oracle_mod.dequant_qt(q)) == 0.0)


# --------------------------------------------------------------------------
# dequantize-and-merge
# --------------------------------------------------------------------------
@pytest.mark.parametrize("qt", [0, 1])
def test_merge_with_zero_B_is_the_dequantized_weight(oracle_mod, qt):
    W = inputs.weight(9, 0, 24, 192, 0.02)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), qt)
    A = inputs.bf16_bits(inputs.uniform(10, (8, 192), 0.1))
    B = np.zeros((24, 8), np.uint16)
    m = _f32(oracle_mod.dequant_merge(q, A, B, 2.0))
    assert np.array_equal(m, _f32(oracle_mod.dequant_qt(q)))       # as values (a -0 may become +0)


@pytest.mark.parametrize("qt", [0, 1])
def test_merge_rank1_closed_form(oracle_mod, qt):
    N, K = 16, 128
    W = inputs.weight(11, 0, N, K, 0.02)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), qt)
    a = inputs.bf16_bits(inputs.uniform(12, (1, K), 1.0))
    b = inputs.bf16_bits(inputs.normal(13, (N, 1), 0.5))
    s = 2.0
    got = oracle_mod.dequant_merge(q, a, b, s)
    wd = _f32(oracle_mod.dequant_qt(q)).astype(np.float64)
    exact = s * _f32(b).astype(np.float64) * _f32(a).astype(np.float64) + wd   # exact in fp64 here
    want = _bf16_bits(exact.astype(np.float32))                                 # one fp32 rounding, then bf16
    assert np.array_equal(got, want)


def test_merge_sums_the_terms_in_order_in_fp32(oracle_mod):
    """A = [1, 2^-30, -1] down every column, B = 1: the fp32 chain gives
    ((1 + 2^-30) - 1) = 0 because 1 + 2^-30 rounds to 1; an fp64 or reordered
    sum would give 2^-30.  On an all-zero weight the merged value shows it."""
    N, K, r = 8, 64, 3
    q = oracle_mod.quantize_dq_qt(np.zeros((N, K), np.uint16), 0)
    A = _bf16_bits(np.repeat(np.array([[1.0], [2.0 ** -30], [-1.0]], np.float32), K, 1))
    B = _bf16_bits(np.ones((N, r), np.float32))
    assert not _f32(oracle_mod.dequant_merge(q, A, B, 1.0)).any()
    # the same terms in the order [1, -1, 2^-30] keep 2^-30
    A2 = A[[0, 2, 1]]
    assert np.all(_f32(oracle_mod.dequant_merge(q, A2, B, 1.0)) == np.float32(2.0 ** -30))


def test_merge_rows_subset(oracle_mod):
    W = inputs.weight(14, 0, 40, 256, 0.02)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), 0)
    A = inputs.bf16_bits(inputs.uniform(15, (5, 256), 0.1))
    B = inputs.bf16_bits(inputs.normal(16, (40, 5), 0.1))
    full = oracle_mod.dequant_merge(q, A, B, 0.5)
    rows = [39, 0, 17]
    assert np.array_equal(oracle_mod.dequant_merge(q, A, B, 0.5, rows=rows), full[rows])


@pytest.mark.parametrize("qt", [0, 1])
def test_merged_weight_reproduces_the_adapted_layer(oracle_mod, qt):
    M, N, K, r, s = 6, 64, 256, 8, 2.0
    W = inputs.weight(17, 0, N, K, 0.02)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), qt)
    X = inputs.to_f64(inputs.normal(18, (M, K), 1.0))
    A = inputs.uniform(19, (r, K), 1.0 / 16)
    B = inputs.normal(20, (N, r), 0.05)
    Wm = _f32(oracle_mod.dequant_merge(q, inputs.bf16_bits(A), inputs.bf16_bits(B), s)).astype(np.float64)
    Wd = _f32(oracle_mod.dequant_qt(q)).astype(np.float64)
    Y, _ = oracle_mod.linear_fwd(X, Wd, inputs.to_f64(A), inputs.to_f64(B), s)
    # the merged weight differs from W' + s B A only by its bf16 rounding (2^-9 relative per entry)
    assert np.all(np.abs(X @ Wm.T - Y) <= 1e-2 * np.maximum(1.0, np.abs(Y)))
