"""GPU parity of the FP4 quant type and of dequantize-and-merge against the oracle.

* FP4 ("Qlora Expert", Hyperparameter Guidance: quant type "fp4"): packed
  nibbles, int8 codes, scale, mean and the dequantized weight bit-exact;
  forward and backward of every kernel family within 1e-2 * max(1, |ref|)
  (the same kernels as NF4 with the FP4 table).
* Merge ("QLoRA Implementation Details (2025 Edition)", Step 7: merge for
  inference): bit-exact against the oracle's fixed-order fp32 definition, on
  both quant types, at small ragged shapes, the single 4096^2 linear and the
  7B gate projection in full, and sampled rows of the 70B up projection.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import _ops as ops
from bit_nf4_quantized_quant_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = 1e-2
NF4, FP4 = 0, 1


def _close(got, ref, what):
    err = np.abs(np.asarray(got, np.float64) - ref)
    lim = TOL * np.maximum(1.0, np.abs(ref))
    assert not (err > lim).any(), f"{what}: {(err > lim).sum()} outside tolerance, worst {err.max():.4g}"


def test_fp4_codebook_matches_oracle(oracle_mod):
    assert np.array_equal(np.array(ops.quant4_codebook(FP4), np.float32), oracle_mod.codebook_qt(FP4))
    assert np.array_equal(np.array(ops.quant4_codebook(NF4), np.float32), oracle_mod.codebook_qt(NF4))


@pytest.mark.parametrize("N,K,kind", [(8, 64, "normal"), (96, 4032, "normal"), (1000, 1088, "outliers"),
                                      (64, 256, "zeros"), (4096, 4096, "normal"), (333, 640, "t4")])
def test_fp4_quantize_dequant_bit_exact(oracle_mod, N, K, kind):
    if kind == "zeros":
        W = torch.zeros((N, K), dtype=torch.bfloat16)
        W[::3, 64:128] = inputs.normal(5, (len(range(0, N, 3)), 64), 0.02)
    else:
        W = inputs.weight(30, N % 7, N, K, 0.02, outlier_frac=0.01 if kind == "outliers" else 0.0,
                          t4_mix=0.1 if kind == "t4" else 0.0)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), FP4)
    w = ops.quant4_quantize_dq(W.cuda(), FP4)
    Wd = ops.nf4_dequant(w)
    torch.cuda.synchronize()
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])
    assert np.array_equal(w.codes.cpu().numpy(), q["codes"])
    assert np.array_equal(w.scale.cpu().numpy().view(np.uint32), q["scale"].view(np.uint32))
    assert np.array_equal(w.mean.cpu().numpy().view(np.uint32), q["mean"].view(np.uint32))
    assert np.array_equal(inputs.bf16_bits(Wd), oracle_mod.dequant_qt(q))


def test_fp4_encoder_near_thresholds(oracle_mod):
    """Weights within 1.5 % of every FP4 decision threshold times the block max, for several
    block maxima: the encoder's fast path must hand these to its exact fallback."""
    L = oracle_mod.codebook_qt(FP4).astype(np.float64)
    levels = np.array(sorted(set(L.tolist())))
    mids = (levels[:-1] + levels[1:]) / 2
    rng = np.random.default_rng(11)
    rows = []
    for c in (1.0, 0.0371, 3.5, 2.0 ** -20, 0.02):
        for _ in range(8):
            x = rng.choice(mids, 63) * (1 + rng.uniform(-0.015, 0.015, 63))
            rows.append(np.concatenate([[c], x * c]).astype(np.float32))
    W = torch.from_numpy(np.array(rows, np.float32)).to(torch.bfloat16)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), FP4)
    w = ops.quant4_quantize_dq(W.cuda(), FP4)
    torch.cuda.synchronize()
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])


@pytest.mark.parametrize("M,N,K,r", [(1, 256, 512, 16), (16, 512, 1024, 16), (24, 136, 192, 8),
                                     (64, 256, 512, 16), (200, 520, 448, 24), (300, 768, 1216, 64)])
def test_fp4_linear_fwd_bwd(oracle_mod, M, N, K, r):
    s = 32.0 / r
    W = inputs.weight(31, 0, N, K, 0.02)
    X = inputs.normal(32, (M, K), 1.0)
    A = inputs.uniform(33, (r, K), 1.0 / np.sqrt(K))
    B = inputs.normal(34, (N, r), 0.05)
    dY = inputs.normal(35, (M, N), 1.0)
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), FP4)
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant_qt(q)).astype(np.float64)
    w = ops.quant4_quantize_dq(W.cuda(), FP4)
    Y = ops.qlora_linear_fwd(X.cuda(), w, A.cuda(), B.cuda(), s)
    path = ops.qlora_last_path()
    dX, dA, dB = ops.qlora_linear_bwd(X.cuda(), dY.cuda(), w, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    assert path == (1 if M <= 32 else 2 if M <= 128 else 3)
    X64, A64, B64, dY64 = (inputs.to_f64(t) for t in (X, A, B, dY))
    Yr, _ = oracle_mod.linear_fwd(X64, Wd, A64, B64, s)
    dXr, dAr, dBr = oracle_mod.linear_bwd(X64, dY64, Wd, A64, B64, s)
    _close(inputs.to_f64(Y), Yr, "Y")
    _close(inputs.to_f64(dX), dXr, "dX")
    _close(inputs.to_f64(dA), dAr, "dA")
    _close(inputs.to_f64(dB), dBr, "dB")


def test_unknown_quant_type_is_rejected():
    W = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    w = ops.nf4_quantize_dq(W)
    w.quant_type = 2
    with pytest.raises(ops.QLoRAError) as e:
        ops.nf4_dequant(w)
    assert e.value.code == -9


# --------------------------------------------------------------------------
# dequantize-and-merge
# --------------------------------------------------------------------------
def _merge_case(oracle_mod, N, K, r, s, qt, seed, rows=None, w_std=0.02, b_std=0.05):
    W = inputs.weight(40 + seed, 0, N, K, w_std, device="cuda")
    A = inputs.uniform(41 + seed, (r, K), 1.0 / np.sqrt(K), "cuda")
    B = inputs.normal(42 + seed, (N, r), b_std, "cuda")
    w = ops.quant4_quantize_dq(W, qt)
    Wm = ops.nf4_dequant_merge(w, A, B, s)
    torch.cuda.synchronize()
    q = oracle_mod.quantize_dq_qt(inputs.bf16_bits(W), qt)
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])
    ref = oracle_mod.dequant_merge(q, inputs.bf16_bits(A), inputs.bf16_bits(B), s, rows=rows)
    got = inputs.bf16_bits(Wm)
    if rows is not None:
        got = got[rows]
    assert np.array_equal(got, ref), f"{(got != ref).sum()} of {ref.size} merged weights differ"
    return w, A, B, Wm


@pytest.mark.parametrize("qt", [NF4, FP4])
@pytest.mark.parametrize("N,K,r", [(1, 64, 1), (8, 64, 3), (100, 320, 16), (33, 192, 5), (264, 1088, 64),
                                   (70, 576, 100), (16, 256, 256)])
def test_merge_bit_exact_small(oracle_mod, qt, N, K, r):
    _merge_case(oracle_mod, N, K, r, 32.0 / r, qt, seed=N + K + r)


@pytest.mark.parametrize("qt", [NF4, FP4])
def test_merge_workload_shapes_full(oracle_mod, qt):
    # the single 4096^2 linear (r = 16, s = 2) and the 7B gate projection 4096 -> 11008
    _merge_case(oracle_mod, 4096, 4096, 16, 2.0, qt, seed=1)
    _merge_case(oracle_mod, 11008, 4096, 16, 2.0, qt, seed=3)


def test_merge_70b_up_projection_sampled_rows(oracle_mod):
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(28672, 48, replace=False))
    _merge_case(oracle_mod, 28672, 8192, 64, 0.25, NF4, seed=4, rows=rows, w_std=0.015)


def test_merge_with_zero_B_is_dequant():
    W = inputs.weight(50, 0, 512, 1024, 0.02, device="cuda")
    w = ops.nf4_quantize_dq(W)
    A = inputs.uniform(51, (16, 1024), 0.03, "cuda")
    Wm = ops.nf4_dequant_merge(w, A, torch.zeros((512, 16), dtype=torch.bfloat16, device="cuda"), 2.0)
    Wd = ops.nf4_dequant(w)
    torch.cuda.synchronize()
    assert torch.equal(Wm.float(), Wd.float())        # equal values (-0 may come back as +0)
