"""Pins for the oracle's QLoRA linear forward and backward (fp64).

The pages fix the structure ("QLoRA Guide", Forward pass, "Dequant + LoRA
path": base path through the dequantized W plus the A-then-B adapter path,
summed; only A and B get gradients) and the scaling alpha/r ("QLoRA
Implementation Details (2025 Edition)", Step 4).  The backward is pinned to
the forward by central finite differences; the forward by special cases that
reduce to a library matrix product and by a unit-vector closed form.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs


def _case(oracle_mod, M=3, N=5, K=64, r=2, seed=0):
    rng = np.random.default_rng(seed)
    W = inputs.weight(90 + seed, 0, N, K, 0.05)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q)).astype(np.float64)
    X = rng.normal(size=(M, K))
    A = rng.uniform(-0.2, 0.2, (r, K))
    B = rng.normal(0, 0.3, (N, r))
    dY = rng.normal(size=(M, N))
    return X, Wd, A, B, dY


def _loss(oracle_mod, X, Wd, A, B, s, dY):
    Y, _ = oracle_mod.linear_fwd(X, Wd, A, B, s)
    return float(np.sum(Y * dY))


@pytest.mark.parametrize("s", [2.0, 0.25])
def test_backward_matches_finite_differences(oracle_mod, s):
    X, Wd, A, B, dY = _case(oracle_mod)
    dX, dA, dB = oracle_mod.linear_bwd(X, dY, Wd, A, B, s)
    rng = np.random.default_rng(11)
    eps = 1e-4
    for name, arr, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for _ in range(4):
            E = rng.normal(size=arr.shape)
            args = dict(X=X, A=A, B=B)
            args[name] = arr + eps * E
            lp = _loss(oracle_mod, args["X"], Wd, args["A"], args["B"], s, dY)
            args[name] = arr - eps * E
            lm = _loss(oracle_mod, args["X"], Wd, args["A"], args["B"], s, dY)
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(grad * E))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_no_gradient_for_the_frozen_weight(oracle_mod):
    X, Wd, A, B, dY = _case(oracle_mod)
    out = oracle_mod.linear_bwd(X, dY, Wd, A, B, 2.0)
    assert len(out) == 3          # dX, dA, dB only


def test_adjoint_identity(oracle_mod):
    X, Wd, A, B, dY = _case(oracle_mod, M=7, N=9, K=128, r=4, seed=3)
    Y, _ = oracle_mod.linear_fwd(X, Wd, A, B, 2.0)
    dX, _, _ = oracle_mod.linear_bwd(X, dY, Wd, A, B, 2.0)
    lhs, rhs = np.sum(Y * dY), np.sum(X * dX)
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_zero_B_reduces_to_library_matmul(oracle_mod):
    X, Wd, A, B, dY = _case(oracle_mod, M=4, N=6, K=192, r=3, seed=4)
    Y, T = oracle_mod.linear_fwd(X, Wd, A, np.zeros_like(B), 2.0)
    ref = torch.matmul(torch.from_numpy(X), torch.from_numpy(Wd).T).numpy()
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
    _, dA, dB = oracle_mod.linear_bwd(X, dY, Wd, A, np.zeros_like(B), 2.0)
    assert np.all(dA == 0)


def test_zero_A_gives_zero_T_and_dB(oracle_mod):
    X, Wd, A, B, dY = _case(oracle_mod, seed=5)
    Y, T = oracle_mod.linear_fwd(X, Wd, np.zeros_like(A), B, 2.0)
    assert np.all(T == 0)
    _, _, dB = oracle_mod.linear_bwd(X, dY, Wd, np.zeros_like(A), B, 2.0)
    assert np.all(dB == 0)


def test_unit_vector_closed_form(oracle_mod):
    # a one-hot input row picks column k of W' plus s * B @ A[:, k]
    X, Wd, A, B, _ = _case(oracle_mod, M=1, N=5, K=64, r=2, seed=6)
    s = 0.25
    for k in (0, 17, 63):
        e = np.zeros((1, 64))
        e[0, k] = 1.0
        Y, T = oracle_mod.linear_fwd(e, Wd, A, B, s)
        for n in range(5):
            want = Wd[n, k] + s * (B[n, 0] * A[0, k] + B[n, 1] * A[1, k])
            assert abs(Y[0, n] - want) <= 1e-15
        assert abs(T[0, 0] - A[0, k]) == 0 and abs(T[0, 1] - A[1, k]) == 0


def test_linearity_and_scaling(oracle_mod):
    X, Wd, A, B, _ = _case(oracle_mod, M=3, N=5, K=128, r=2, seed=8)
    X2 = np.random.default_rng(9).normal(size=X.shape)
    Y1, _ = oracle_mod.linear_fwd(X, Wd, A, B, 2.0)
    Y2, _ = oracle_mod.linear_fwd(X2, Wd, A, B, 2.0)
    Y12, _ = oracle_mod.linear_fwd(X + X2, Wd, A, B, 2.0)
    assert np.allclose(Y12, Y1 + Y2, atol=1e-12)
    Y0, _ = oracle_mod.linear_fwd(X, Wd, A, B, 0.0)
    Y4, _ = oracle_mod.linear_fwd(X, Wd, A, B, 4.0)
    assert np.allclose(Y4 - Y0, 2 * (Y1 - Y0), atol=1e-12)


def test_adapter_only_backward_matches_full(oracle_mod):
    X, Wd, A, B, dY = _case(oracle_mod, M=6, N=9, K=128, r=3, seed=12)
    _, dA, dB = oracle_mod.linear_bwd(X, dY, Wd, A, B, 0.5)
    dA2, dB2 = oracle_mod.linear_bwd_adapters(X, dY, A, B, 0.5)
    assert np.array_equal(dA, dA2) and np.array_equal(dB, dB2)
