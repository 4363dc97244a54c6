"""GPU parity of nf4_quantize_dq and nf4_dequant against the CPU oracle.

Bit-exact on every packed byte, int8 code, fp32 scale and mean, and every
dequantized bf16 weight, on shapes that span several CTAs and a ragged last
double-quant group, on the degenerate blocks of the method, and at the full
workload sizes (sampled where the oracle would take too long).
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs
from bit_nf4_quantized_quant_b200 import _ops as ops

pytestmark = pytest.mark.gpu


def _gpu_quant(W):
    w = ops.nf4_quantize_dq(W.cuda())
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    return w


def _assert_same_quant(w, q):
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])
    assert np.array_equal(w.codes.cpu().numpy(), q["codes"])
    assert np.array_equal(w.scale.cpu().numpy().view(np.uint32), q["scale"].view(np.uint32))
    assert np.array_equal(w.mean.cpu().numpy().view(np.uint32), q["mean"].view(np.uint32))


@pytest.mark.parametrize("N,K,kind", [
    (8, 64, "normal"),          # 8 blocks: one short group
    (5, 64, "normal"),          # odd N
    (64, 4096, "normal"),       # exactly 16 groups
    (96, 4032, "outliers"),     # 6048 blocks: ragged last group
    (1000, 1088, "t4"),         # many CTAs, ragged group
    (256, 512, "zeros"),
    (128, 512, "codebook"),
])
def test_quantize_dequant_bit_exact(oracle_mod, N, K, kind):
    if kind == "zeros":
        W = torch.zeros((N, K), dtype=torch.bfloat16)
        W[3, 70] = 0.5                      # one non-zero block amid all-zero blocks
    elif kind == "codebook":
        _, L = oracle_mod.codebook()
        base = np.tile(np.concatenate([L, L[::-1], L, L[::-1]]), N * K // 64)
        W = torch.from_numpy((base * 0.0625).astype(np.float32).reshape(N, K)).to(torch.bfloat16)
    else:
        W = inputs.weight(7, N % 97, N, K, 0.02, outlier_frac=0.001 if kind == "outliers" else 0.0,
                          t4_mix=0.1 if kind == "t4" else 0.0)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    w = _gpu_quant(W)
    _assert_same_quant(w, q)
    Wd = ops.nf4_dequant(w)
    torch.cuda.synchronize()
    assert np.array_equal(inputs.bf16_bits(Wd), oracle_mod.dequant(q))
    if kind == "codebook":
        assert torch.equal(Wd.cpu(), W)


def test_all_zero_weight(oracle_mod):
    W = torch.zeros((16, 256), dtype=torch.bfloat16)
    w = _gpu_quant(W)
    assert torch.all(w.packed == 0x77)
    assert torch.all(w.codes == 0) and torch.all(w.scale == 0) and torch.all(w.mean == 0)
    assert torch.all(ops.nf4_dequant(w) == 0)


@pytest.mark.parametrize("wl,proj", [(1, 0), (2, 0), (2, 1), (3, 0), (3, 4), (3, 6)])
def test_workload_shapes_full(oracle_mod, wl, proj):
    w_l = inputs.WORKLOADS[wl]
    W = inputs.layer_weight(w_l, proj)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    w = _gpu_quant(W)
    _assert_same_quant(w, q)
    Wd = ops.nf4_dequant(w)
    assert np.array_equal(inputs.bf16_bits(Wd), oracle_mod.dequant(q))


@pytest.mark.parametrize("proj", [0, 1, 2])
def test_70b_shapes_sampled_groups(oracle_mod, proj):
    # full GPU quantization of the 70B-shape weights; the oracle re-quantizes
    # a sample of whole double-quant groups (16384 consecutive weights each)
    wl = inputs.WORKLOADS[4]
    p = wl.projections[proj]
    W = inputs.layer_weight(wl, proj, device="cuda")
    w = _gpu_quant(W)
    Wd = ops.nf4_dequant(w)
    torch.cuda.synchronize()
    ng = w.scale.numel()
    rng = np.random.default_rng(proj)
    groups = sorted(set(rng.choice(ng, size=48, replace=False).tolist() + [0, ng - 1]))
    flatW = W.view(-1)
    flatP = w.packed.view(-1)
    flatD = Wd.view(-1)
    for g in groups:
        lo, hi = g * 16384, min((g + 1) * 16384, p.N * p.K)
        sub = flatW[lo:hi].view(1, -1)
        q = oracle_mod.quantize_dq(inputs.bf16_bits(sub))
        assert np.array_equal(flatP[lo // 2:hi // 2].cpu().numpy(), q["packed"].reshape(-1))
        assert np.array_equal(w.codes[g * 256:g * 256 + (hi - lo) // 64].cpu().numpy(), q["codes"])
        assert w.scale[g].item() == q["scale"][0] and w.mean[g].item() == q["mean"][0]
        assert np.array_equal(inputs.bf16_bits(flatD[lo:hi]), oracle_mod.dequant(q).reshape(-1))


def test_bulk_mixture_layer_sampled(oracle_mod):
    # one layer of the bulk workload (t(4) mixture weights): 1% of the groups
    # of every projection, bit for bit
    wl = inputs.WORKLOADS[5]
    for proj in range(len(wl.projections)):
        p = wl.projections[proj]
        W = inputs.layer_weight(wl, proj, device="cuda")
        w = _gpu_quant(W)
        Wd = ops.nf4_dequant(w)
        torch.cuda.synchronize()
        ng = w.scale.numel()
        rng = np.random.default_rng(100 + proj)
        for g in rng.choice(ng, size=max(1, ng // 100), replace=False):
            lo, hi = g * 16384, (g + 1) * 16384
            q = oracle_mod.quantize_dq(inputs.bf16_bits(W.view(-1)[lo:hi].view(1, -1)))
            assert np.array_equal(w.packed.view(-1)[lo // 2:hi // 2].cpu().numpy(), q["packed"].reshape(-1))
            assert np.array_equal(w.codes[g * 256:(g + 1) * 256].cpu().numpy(), q["codes"])
            assert np.array_equal(inputs.bf16_bits(Wd.view(-1)[lo:hi]), oracle_mod.dequant(q).reshape(-1))


def test_quantize_near_thresholds(oracle_mod):
    """Weights whose normalised value w / c lies within a few ulp of an NF4
    decision threshold (and exactly on one where the division lands there):
    every bf16 weight in a window of +-1.5 % around c * m_i, for every midpoint
    m_i and block maxima c (every bf16 mantissa in [1, 2), and tiny and
    subnormal ones), each block led
    by +-c so that c is its absmax.  Bit-exact against the oracle, which
    divides in IEEE fp32 -- this is where the kernel's reciprocal-and-bucket
    fast path must hand over to the exact quotient."""
    def bits_of(v):
        return int(inputs.bf16_bits(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16))[0])

    blocks = []
    maxima = [1.0 + k / 128.0 for k in range(128)] + [0.0234375, 3.0e-3, 7.25, 1.0e-30, 1.0e-39]
    for c in maxima:
        for mi in np.asarray(oracle_mod.midpoints(), dtype=np.float64):
            centre = c * mi
            a, b = bits_of(centre * 0.985), bits_of(centre * 1.015)
            vals = np.arange(min(a, b), max(a, b) + 1, dtype=np.uint32).astype(np.uint16)
            lead = np.uint16(bits_of(c) | (0x8000 if mi < 0 else 0))
            for s0 in range(0, len(vals), 63):
                blk = np.zeros(64, dtype=np.uint16)
                blk[0] = lead
                chunk = vals[s0:s0 + 63]
                blk[1:1 + len(chunk)] = chunk
                blocks.append(blk)
    while len(blocks) % 64:                 # 8 rows of 8 blocks: N a multiple of 8
        blocks.append(np.zeros(64, dtype=np.uint16))
    bits = np.stack(blocks).reshape(-1, 512)
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    w = _gpu_quant(W)
    _assert_same_quant(w, q)
