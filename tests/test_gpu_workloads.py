"""GPU parity of the forward and backward at the full sizes of the training
and 70B-shape workloads, against the fp64 oracle.

Rows of Y and dX are independent, so the oracle computes a seeded sample of
them (plus the first and last row) from the whole dequantized weight; dA and
dB sum over every token and are computed in full.  Tolerance
|err| <= 1e-2 * max(1, |ref|) per element.  The GPU's quantized weight is
first checked to be the oracle's, byte for byte.

Workloads:
  * the 7 projections of a 7B decoder block at M = 2048 (r = 16, s = 2, 0.1 %
    of the weights x10): gate (4096 -> 11008) and down (11008 -> 4096), which
    run the SM-pair kernel over 8 x 43 = 344 and 8 x 16 = 128 pair tiles;
  * 70B shapes 8192^2, 8192 -> 28672 and 28672 -> 8192 at M = 1, 512, 4096
    (r = 64, s = 0.25): the decode kernels over 28672-long reductions, and
    the SM-pair kernel with up to 16 x 112 tiles.
"""
import functools

import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import _ops as ops
from bit_nf4_quantized_quant_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    lim = TOL * np.maximum(1.0, np.abs(ref))
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst err "
                           f"{err.max():.4g} at {np.unravel_index(np.argmax(err - lim), err.shape)}")


@functools.lru_cache(maxsize=1)
def _oracle_weight(oracle_mod, wl_index, proj):
    """The oracle's quantization of one projection's weight and its fp64 W' (cached across M)."""
    wl = inputs.WORKLOADS[wl_index]
    W = inputs.layer_weight(wl, proj, device="cuda")
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q)).astype(np.float64)
    return W, q, Wd


def _parity(oracle_mod, wl_index, proj, M, rows_n=16):
    wl = inputs.WORKLOADS[wl_index]
    s = wl.scaling
    W, q, Wd = _oracle_weight(oracle_mod, wl_index, proj)
    X, A, B, dY = inputs.layer_inputs(wl, proj, M, device="cuda")
    w = ops.nf4_quantize_dq(W)
    X64, A64, B64, dY64 = (inputs.to_f64(t) for t in (X, A, B, dY))
    # the backward with T given takes T as an input: feed it the oracle's T rounded to bf16
    T_in = torch.from_numpy(X64 @ A64.T).to(torch.bfloat16).cuda()
    T = torch.empty((M, wl.r), dtype=torch.bfloat16, device="cuda")
    Y = ops.qlora_linear_fwd(X, w, A, B, s, T_out=T)
    path = ops.qlora_last_path()
    dX, dA, dB = ops.qlora_linear_bwd(X, dY, w, A, B, s)              # T recomputed
    dX2, dA2, dB2 = ops.qlora_linear_bwd(X, dY, w, A, B, s, T=T_in)   # T given
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    assert path == (1 if M <= 32 else 2 if M <= 128 else 3)
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])
    assert np.array_equal(w.codes.cpu().numpy(), q["codes"])

    rng = np.random.default_rng(1000 * wl.index + 10 * proj + M)
    rows = np.unique(np.concatenate([rng.choice(M, size=min(rows_n, M), replace=False), [0, M - 1]]))
    Yr, Tr = oracle_mod.linear_fwd(X64[rows], Wd, A64, B64, s)
    _close(inputs.to_f64(Y)[rows], Yr, "Y rows")
    _close(inputs.to_f64(T)[rows], Tr, "T rows")
    dXr, _, _ = oracle_mod.linear_bwd(X64[rows], dY64[rows], Wd, A64, B64, s)
    _close(inputs.to_f64(dX)[rows], dXr, "dX rows")
    _close(inputs.to_f64(dX2)[rows], dXr, "dX rows (T given)")
    dAr, dBr = oracle_mod.linear_bwd_adapters(X64, dY64, A64, B64, s)
    _close(inputs.to_f64(dA), dAr, "dA")
    _close(inputs.to_f64(dB), dBr, "dB")
    _close(inputs.to_f64(dA2), dAr, "dA (T given)")
    _close(inputs.to_f64(dB2), s * (dY64.T @ inputs.to_f64(T_in)), "dB (T given)")


@pytest.mark.parametrize("proj", [4, 6])
def test_workload3_block_M2048(oracle_mod, proj):
    _parity(oracle_mod, 3, proj, 2048)


# ordered by projection so that the cached oracle weight is reused across M
@pytest.mark.parametrize("proj,M", [(p, m) for p in (0, 1, 2) for m in (1, 512, 4096)])
def test_workload4_70b_shapes(oracle_mod, proj, M):
    _parity(oracle_mod, 4, proj, M)
