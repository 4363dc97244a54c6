"""Pins for the oracle's LoRA dropout ("Qlora Expert", Implementation Pattern:
lora_dropout=0.05; "QLoRA Implementation Details (2025 Edition)", Step 4).

* Philox4x64-10 against numpy's Philox bit generator (the same published
  generator; numpy advances its counter before each block, so its block k is
  this generator's counter k + 1).
* The mask: the dropped fraction within 5 sigma of p, p = 0 keeps everything,
  (seed, offset) decides it, and neighbouring offsets give different masks.
* Forward and backward: p = 0 reduces to the plain layer; the backward is the
  gradient of <Y, dY> under a fixed mask (central differences in fp64).
"""
import numpy as np
import pytest

from bit_nf4_quantized_quant_b200 import inputs


@pytest.mark.parametrize("key", [0, 123, 2 ** 63 + 5])
def test_philox_matches_numpy(oracle_mod, key):
    bg = np.random.Philox(key=np.array([key, 0], np.uint64), counter=np.array([7, 9, 0, 0], np.uint64))
    raw = bg.random_raw(12)
    for blk in range(3):
        got = oracle_mod.philox4x64([8 + blk, 9, 0, 0], [key, 0])
        assert np.array_equal(got, raw[4 * blk: 4 * blk + 4])


@pytest.mark.parametrize("p", [0.05, 0.1, 0.5])
def test_mask_rate(oracle_mod, p):
    keep = oracle_mod.dropout_mask(1234, 0, 64, 4096, p)
    n = keep.size
    dropped = n - keep.sum()
    assert abs(dropped - p * n) <= 5 * np.sqrt(n * p * (1 - p))


def test_mask_determinism_and_offsets(oracle_mod):
    a = oracle_mod.dropout_mask(7, 3, 16, 256, 0.1)
    assert np.array_equal(a, oracle_mod.dropout_mask(7, 3, 16, 256, 0.1))
    assert not np.array_equal(a, oracle_mod.dropout_mask(7, 4, 16, 256, 0.1))
    assert not np.array_equal(a, oracle_mod.dropout_mask(8, 3, 16, 256, 0.1))
    assert oracle_mod.dropout_mask(7, 3, 16, 256, 0.0).all()
    # element e uses field e % 16 of block e // 16: a row-major [M, K] mask is one flat stream
    flat = oracle_mod.dropout_mask(7, 3, 1, 16 * 256, 0.1).reshape(16, 256)
    assert np.array_equal(a, flat)


def test_p0_is_the_plain_layer(oracle_mod):
    rng = np.random.default_rng(0)
    M, N, K, r, s = 5, 12, 64, 3, 2.0
    X, dY = rng.standard_normal((M, K)), rng.standard_normal((M, N))
    W, A, B = rng.standard_normal((N, K)), rng.standard_normal((r, K)), rng.standard_normal((N, r))
    keep = np.ones((M, K), bool)
    Y0, T0 = oracle_mod.linear_fwd(X, W, A, B, s)
    Y1, T1 = oracle_mod.linear_fwd_dropout(X, W, A, B, s, keep, 1.0)
    assert np.array_equal(Y0, Y1) and np.array_equal(T0, T1)
    for a, b in zip(oracle_mod.linear_bwd(X, dY, W, A, B, s), oracle_mod.linear_bwd_dropout(X, dY, W, A, B, s, keep, 1.0)):
        assert np.array_equal(a, b)


def test_backward_is_the_gradient_under_a_fixed_mask(oracle_mod):
    rng = np.random.default_rng(1)
    M, N, K, r, s = 3, 5, 64, 2, 1.5
    X, dY = rng.standard_normal((M, K)), rng.standard_normal((M, N))
    W, A, B = rng.standard_normal((N, K)), rng.standard_normal((r, K)), rng.standard_normal((N, r))
    keep = oracle_mod.dropout_mask(5, 1, M, K, 0.3)
    c = oracle_mod.dropout_scale(0.3)
    f = lambda X_, A_, B_: float(np.sum(oracle_mod.linear_fwd_dropout(X_, W, A_, B_, s, keep, c)[0] * dY))
    dX, dA, dB = oracle_mod.linear_bwd_dropout(X, dY, W, A, B, s, keep, c)
    h = 1e-6
    for arr, grad, which in ((X, dX, 0), (A, dA, 1), (B, dB, 2)):
        for idx in [(0, 0), (1, arr.shape[1] // 2), (arr.shape[0] - 1, arr.shape[1] - 1)]:
            e = np.zeros_like(arr)
            e[idx] = h
            args_p = [X, A, B]
            args_m = [X, A, B]
            args_p[which] = arr + e
            args_m[which] = arr - e
            fd = (f(*args_p) - f(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd))
    # dropped inputs get no gradient through the branch, kept ones get c times it
    U = dY @ B
    assert np.allclose(dX - dY @ W, s * (U @ A) * keep * c)
