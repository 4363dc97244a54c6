"""GPU parity of the LoRA-dropout forward and backward against the fp64 oracle
("Qlora Expert", Implementation Pattern: lora_dropout=0.05; "QLoRA
Implementation Details (2025 Edition)", Step 4: lora_dropout=0.1).

The oracle draws the same Philox4x64-10 keep mask (written from the
generator's definition and pinned against numpy's Philox), and computes
Y, T, dX, dA, dB in fp64 with Xd = X * keep * c exactly; the GPU rounds Xd
to bf16 once, so the tolerance is the usual 1e-2 * max(1, |ref|).  Every
kernel family is covered (small-M GEMV / backward, single-SM and SM-pair
tcgen05 kernels), with T recomputed and with the forward's T given.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import _ops as ops
from bit_nf4_quantized_quant_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _close(got, ref, what):
    err = np.abs(np.asarray(got, np.float64) - ref)
    lim = TOL * np.maximum(1.0, np.abs(ref))
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, worst {err.max():.4g}"


@pytest.mark.parametrize("M,N,K,r,p", [(1, 256, 512, 16, 0.1), (8, 512, 1024, 16, 0.05), (24, 136, 192, 8, 0.5),
                                       (64, 256, 512, 16, 0.1), (100, 264, 640, 24, 0.1), (200, 520, 448, 64, 0.05),
                                       (300, 768, 1216, 16, 0.1), (16, 4096, 4096, 16, 0.05)])
def test_dropout_fwd_bwd_parity(oracle_mod, M, N, K, r, p):
    s = 32.0 / r
    seed, offset = 1234 + M, 7
    W = inputs.weight(70, 0, N, K, 0.02)
    X = inputs.normal(71, (M, K), 1.0)
    A = inputs.uniform(72, (r, K), 1.0 / np.sqrt(K))
    B = inputs.normal(73, (N, r), 0.05)
    dY = inputs.normal(74, (M, N), 1.0)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q)).astype(np.float64)
    w = ops.nf4_quantize_dq(W.cuda())
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = ops.qlora_linear_fwd_dropout(Xc, w, Ac, Bc, s, p, seed, offset, T_out=T)
    path = ops.qlora_last_path()
    dX, dA, dB = ops.qlora_linear_bwd_dropout(Xc, dYc, w, Ac, Bc, s, p, seed, offset)
    dX2, dA2, dB2 = ops.qlora_linear_bwd_dropout(Xc, dYc, w, Ac, Bc, s, p, seed, offset, T=T)
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    assert path == (1 if M <= 32 else 2 if M <= 128 else 3)
    keep = oracle_mod.dropout_mask(seed, offset, M, K, p)
    c = oracle_mod.dropout_scale(p)
    X64, A64, B64, dY64 = (inputs.to_f64(t) for t in (X, A, B, dY))
    Yr, Tr = oracle_mod.linear_fwd_dropout(X64, Wd, A64, B64, s, keep, c)
    dXr, dAr, dBr = oracle_mod.linear_bwd_dropout(X64, dY64, Wd, A64, B64, s, keep, c)
    _close(inputs.to_f64(Y), Yr, "Y")
    _close(inputs.to_f64(T), Tr, "T")
    for tag, (gx, ga, gb) in (("recomputed T", (dX, dA, dB)), ("T given", (dX2, dA2, dB2))):
        _close(inputs.to_f64(gx), dXr, f"dX ({tag})")
        _close(inputs.to_f64(ga), dAr, f"dA ({tag})")
    _close(inputs.to_f64(dB), dBr, "dB")
    _close(inputs.to_f64(dB2), s * (dY64.T @ inputs.to_f64(T)), "dB (T given)")


@pytest.mark.parametrize("M", [4, 160])
def test_dropout_zero_rate_is_the_plain_layer(M):
    N, K, r, s = 512, 1024, 16, 2.0
    W = inputs.weight(75, 0, N, K, 0.02, device="cuda")
    X = inputs.normal(76, (M, K), 1.0, "cuda")
    A = inputs.uniform(77, (r, K), 1.0 / 32, "cuda")
    B = inputs.normal(78, (N, r), 0.05, "cuda")
    dY = inputs.normal(79, (M, N), 1.0, "cuda")
    w = ops.nf4_quantize_dq(W)
    Y0 = ops.qlora_linear_fwd(X, w, A, B, s)
    Y1 = ops.qlora_linear_fwd_dropout(X, w, A, B, s, 0.0, 5, 6)
    g0 = ops.qlora_linear_bwd(X, dY, w, A, B, s)
    g1 = ops.qlora_linear_bwd_dropout(X, dY, w, A, B, s, 0.0, 5, 6)
    torch.cuda.synchronize()
    assert torch.equal(Y0, Y1)
    for a, b in zip(g0[1:], g1[1:]):            # dA, dB: the same products on the same operands
        assert torch.equal(a, b)
    # dX: the small-M path applies the same single rounding; the tcgen05 path adds the LoRA
    # term after a bf16 rounding of dY W' (a second rounding), so compare within tolerance
    ref = g0[0].double()
    assert torch.all((g1[0].double() - ref).abs() <= TOL * ref.abs().clamp(min=1.0))


def test_dropout_rejects_a_rate_of_one():
    W = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    w = ops.nf4_quantize_dq(W)
    X = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((8, 4), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.QLoRAError) as e:
        ops.qlora_linear_fwd_dropout(X, w, A, B, 1.0, 1.0, 0, 0)
    assert e.value.code == -9
