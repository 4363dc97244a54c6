"""GPU parity of qlora_linear_fwd / qlora_linear_bwd against the fp64 oracle.

Tolerance |err| <= 1e-2 * max(1, |ref|) per element.  The weight the GPU
multiplies with is first checked to be the oracle's bit for bit (see
test_gpu_quant.py), so the oracle's W' is the exact operand.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs
from bit_nf4_quantized_quant_b200 import _ops as ops

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


def _setup(oracle_mod, M, N, K, r, seed, w_std=0.02, x_std=1.0):
    W = inputs.weight(50 + seed, 0, N, K, w_std)
    X = inputs.normal(60 + seed, (M, K), x_std)
    A = inputs.uniform(61 + seed, (r, K), 1.0 / np.sqrt(K))
    B = inputs.normal(62 + seed, (N, r), 0.01 * 10)    # larger than the workloads' so the LoRA term matters
    dY = inputs.normal(63 + seed, (M, N), 1.0)
    q = oracle_mod.quantize_dq(inputs.bf16_bits(W))
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q)).astype(np.float64)
    w = ops.nf4_quantize_dq(W.cuda())
    assert np.array_equal(w.packed.cpu().numpy(), q["packed"])
    return W, X, A, B, dY, Wd, w


CASES = [
    # M, N, K, r            small-M kernels for M <= 32, tcgen05 kernels above
    (1, 64, 64, 16),
    (3, 136, 192, 4),
    (8, 256, 1024, 16),
    (16, 512, 512, 64),
    (17, 200, 320, 24),
    (32, 1024, 1024, 16),
    (5, 4096, 4096, 16),
    (33, 128, 256, 16),
    (100, 264, 640, 8),
    (128, 256, 256, 16),
    (200, 520, 448, 24),
    (257, 384, 448, 64),
    (300, 768, 1216, 100),
    (512, 1024, 2048, 16),
    (129, 256, 512, 16),
    (640, 1280, 1024, 32),
    (1000, 520, 1088, 64),
    (2, 256, 512, 256),         # maximum rank on each path
    (64, 256, 512, 256),
    (130, 256, 512, 256),
    # more tiles than persistent CTAs (148) or SM pairs (74), so that a CTA or pair runs
    # several tiles through its double-buffered accumulator: forward tiles span N,
    # backward tiles span K
    (64, 38912, 256, 16),       # single-SM kernel: 152 forward tiles
    (100, 256, 38912, 8),       # single-SM kernel: 152 backward tiles
    (512, 11008, 1024, 16),     # SM pairs: 86 forward pair tiles
    (520, 1024, 11008, 32),     # SM pairs: 3 x 43 = 129 backward pair tiles, ragged M
    (512, 4096, 4096, 16),      # SM pairs, one token tile per step, stream-K both ways (32 tiles)
    (500, 5120, 1024, 16),      # SM pairs, one token tile, stream-K forward (40 tiles), ragged M
]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_fwd_bwd_parity(oracle_mod, M, N, K, r):
    s = 32.0 / r
    W, X, A, B, dY, Wd, w = _setup(oracle_mod, M, N, K, r, seed=M + N + K + r)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    X64, A64, B64, dY64 = (inputs.to_f64(t) for t in (X, A, B, dY))
    # the backward with T given takes T as an input: feed it the oracle's T rounded to bf16
    T_in = torch.from_numpy(X64 @ A64.T).to(torch.bfloat16)
    T_out = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = ops.qlora_linear_fwd(Xc, w, Ac, Bc, s, T_out=T_out)
    dX, dA, dB = ops.qlora_linear_bwd(Xc, dYc, w, Ac, Bc, s)
    dX2, dA2, dB2 = ops.qlora_linear_bwd(Xc, dYc, w, Ac, Bc, s, T=T_in.cuda())
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    Yr, Tr = oracle_mod.linear_fwd(X64, Wd, A64, B64, s)
    dXr, dAr, dBr = oracle_mod.linear_bwd(X64, dY64, Wd, A64, B64, s)
    _close(inputs.to_f64(Y), Yr, "Y")
    _close(inputs.to_f64(T_out), Tr, "T")
    _close(inputs.to_f64(dX), dXr, "dX")
    _close(inputs.to_f64(dA), dAr, "dA")
    _close(inputs.to_f64(dB), dBr, "dB")
    # with T supplied, the bf16 T is an input of the backward: dB = s dY^T T_given
    dBr_given = s * (dY64.T @ inputs.to_f64(T_in))
    _close(inputs.to_f64(dX2), dXr, "dX (T given)")
    _close(inputs.to_f64(dA2), dAr, "dA (T given)")
    _close(inputs.to_f64(dB2), dBr_given, "dB (T given)")
    assert ops.qlora_last_path() == (1 if M <= 32 else 2 if M <= 128 else 3)


def test_zero_B_is_plain_dequant_matmul(oracle_mod):
    M, N, K, r = 24, 512, 1024, 16
    W, X, A, B, dY, Wd, w = _setup(oracle_mod, M, N, K, r, seed=3)
    Bz = torch.zeros_like(B)
    Y = ops.qlora_linear_fwd(X.cuda(), w, A.cuda(), Bz.cuda(), 2.0)
    Wdq = ops.nf4_dequant(w)
    ref = (X.cuda().float() @ Wdq.float().T)
    torch.cuda.synchronize()
    _close(inputs.to_f64(Y), ref.double().cpu().numpy(), "Y vs torch.matmul on nf4_dequant")


def test_repeatable(oracle_mod):
    M, N, K, r = 16, 1024, 2048, 16
    W, X, A, B, dY, Wd, w = _setup(oracle_mod, M, N, K, r, seed=4)
    outs = []
    for _ in range(2):
        Y = ops.qlora_linear_fwd(X.cuda(), w, A.cuda(), B.cuda(), 2.0)
        dX, dA, dB = ops.qlora_linear_bwd(X.cuda(), dY.cuda(), w, A.cuda(), B.cuda(), 2.0)
        outs.append([t.cpu() for t in (Y, dX, dA, dB)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)        # fixed reduction orders: bit-identical reruns


@pytest.mark.parametrize("M", [1, 5, 17, 64, 200])
def test_inputs_written_just_before_each_call(M):
    """Every input of every call is written by the kernels queued right before it on the same
    stream, with no synchronisation: the weights by nf4_quantize_dq, the adapters and dY by torch
    copies, and layer 1's X is layer 0's Y.  The kernels that start before the one ahead of them
    has finished (programmatic launch) must read none of it early, so the outputs must equal, bit
    for bit, those of a run that synchronises after every call."""
    N0, K0, r, s = 512, 1024, 16, 2.0
    shapes = [(N0, K0), (K0, N0)]          # layer 1 maps layer 0's output back to K0
    W = [inputs.weight(90 + i, 0, n, k, 0.02).cuda() for i, (n, k) in enumerate(shapes)]
    X0 = inputs.normal(92, (M, K0), 1.0).cuda()
    A = [inputs.uniform(93 + i, (r, k), 1.0 / np.sqrt(k)).cuda() for i, (n, k) in enumerate(shapes)]
    B = [inputs.normal(95 + i, (n, r), 0.1).cuda() for i, (n, k) in enumerate(shapes)]
    dY = [inputs.normal(97 + i, (M, n), 1.0).cuda() for i, (n, k) in enumerate(shapes)]

    def run(sync):
        outs = []
        x = X0.clone()
        for i in range(2):
            w = ops.nf4_quantize_dq(W[i])
            a, b, dy = A[i].clone(), B[i].clone(), dY[i].clone()
            if sync:
                torch.cuda.synchronize()
            T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
            y = ops.qlora_linear_fwd(x, w, a, b, s, T_out=T)
            if sync:
                torch.cuda.synchronize()
            dx, da, db = ops.qlora_linear_bwd(x, dy, w, a, b, s, T=T)
            if sync:
                torch.cuda.synchronize()
            outs += [y, T, dx, da, db]
            x = y
        torch.cuda.synchronize()
        assert ops.qlora_device_status() == 0
        return [t.cpu() for t in outs]

    ref = run(True)
    for _ in range(3):
        got = run(False)
        for g, e in zip(got, ref):
            assert torch.equal(g, e)


@pytest.mark.parametrize("M,N0,K0", [(64, 768, 1024), (200, 768, 1024), (600, 768, 1024), (2048, 4096, 4096),
                                     (2048, 11008, 4096)])
@pytest.mark.parametrize("given_T", [True, False])
@pytest.mark.parametrize("dropout", [0.0, 0.1])
def test_layer_chain_on_one_workspace(M, N0, K0, given_T, dropout):
    """Two layers' forward, then their backward in reverse order (layer 0's dY is layer 1's dX),
    on one stream and ONE workspace, with the adapter gradients copied by torch right after the
    last call: no synchronisation anywhere.  In the backward, dB and dA run beside the fused dX
    kernel (they skip the wait on it), and every next call's kernels overwrite the workspace that
    the previous call's kernels read; the results must equal, bit for bit, a run that synchronises
    after every call -- run eagerly, and replayed as a CUDA graph.  At 2048 tokens the SM-pair
    kernel runs stream-K (partial tiles and counters in the workspace) in the forward of both
    shapes and in the backward of the 11008-wide dX."""
    r, s = 16, 2.0
    shapes = [(N0, K0), (K0, N0)]                 # layer 1 maps layer 0's output back to K0
    W = [inputs.weight(70 + i, 0, n, k, 0.02).cuda() for i, (n, k) in enumerate(shapes)]
    w = [ops.nf4_quantize_dq(Wi) for Wi in W]
    X0 = inputs.normal(72, (M, K0), 1.0).cuda()
    A = [inputs.uniform(73 + i, (r, k), 1.0 / np.sqrt(k)).cuda() for i, (n, k) in enumerate(shapes)]
    B = [inputs.normal(75 + i, (n, r), 0.1).cuda() for i, (n, k) in enumerate(shapes)]
    dY1 = inputs.normal(77, (M, K0), 1.0).cuda()
    nbytes = max((ops.qlora_dropout_workspace_bytes if dropout else ops.qlora_workspace_bytes)(M, n, k, r)
                 for n, k in shapes)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    Ts = [torch.empty((M, r), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    Ys = [torch.empty((M, n), dtype=torch.bfloat16, device="cuda") for n, k in shapes]
    dXs = [torch.empty((M, k), dtype=torch.bfloat16, device="cuda") for n, k in shapes]
    dAs = [torch.empty((r, k), dtype=torch.bfloat16, device="cuda") for n, k in shapes]
    dBs = [torch.empty((n, r), dtype=torch.bfloat16, device="cuda") for n, k in shapes]
    copies = [torch.empty_like(t) for t in dAs + dBs]

    def fwd(i, x):
        if dropout:
            ops.qlora_linear_fwd_dropout(x, w[i], A[i], B[i], s, dropout, 5, i, Y=Ys[i], T_out=Ts[i], ws=ws)
        else:
            ops.qlora_linear_fwd(x, w[i], A[i], B[i], s, Y=Ys[i], T_out=Ts[i], ws=ws)

    def bwd(i, x, dy):
        T = Ts[i] if given_T else None
        if dropout:
            ops.qlora_linear_bwd_dropout(x, dy, w[i], A[i], B[i], s, dropout, 5, i, T=T, dX=dXs[i], dA=dAs[i],
                                         dB=dBs[i], ws=ws)
        else:
            ops.qlora_linear_bwd(x, dy, w[i], A[i], B[i], s, T=T, dX=dXs[i], dA=dAs[i], dB=dBs[i], ws=ws)

    def seq(sync):
        for i, x in ((0, X0), (1, Ys[0])):
            fwd(i, x)
            if sync:
                torch.cuda.synchronize()
        for i, x, dy in ((1, Ys[0], dY1), (0, X0, dXs[1])):
            bwd(i, x, dy)
            if sync:
                torch.cuda.synchronize()
        for c, t in zip(copies, dAs + dBs):
            c.copy_(t)

    def results():
        torch.cuda.synchronize()
        assert ops.qlora_device_status() == 0
        return [t.cpu() for t in Ys + Ts + dXs + copies]

    seq(True)
    ref = results()
    for _ in range(2):
        for t in Ys + Ts + dXs + dAs + dBs + copies:
            t.zero_()
        seq(False)
        for g, e in zip(results(), ref):
            assert torch.equal(g, e)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        seq(False)
    for _ in range(2):
        for t in Ys + Ts + dXs + dAs + dBs + copies:
            t.zero_()
        g.replay()
        for gt, e in zip(results(), ref):
            assert torch.equal(gt, e)
    del g


def _sampled_rows_parity(oracle_mod, wl, proj, M, rows_n=16, bwd=True):
    p = wl.projections[proj]
    s = wl.scaling
    W = inputs.layer_weight(wl, proj, device="cuda")
    X, A, B, dY = inputs.layer_inputs(wl, proj, M, device="cuda", with_dy=bwd)
    w = ops.nf4_quantize_dq(W)
    Y = ops.qlora_linear_fwd(X, w, A, B, s)
    if bwd:
        dX, dA, dB = ops.qlora_linear_bwd(X, dY, w, A, B, s)
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    rng = np.random.default_rng(1000 * wl.index + proj + M)
    rows_m = np.unique(np.concatenate([rng.choice(M, size=min(rows_n, M), replace=False), [0, M - 1]]))
    # oracle weight rows (output features) and columns needed
    Wbits = inputs.bf16_bits(W)
    X64 = inputs.to_f64(X)
    A64, B64 = inputs.to_f64(A), inputs.to_f64(B)
    # Y rows: need the whole W'
    q_full = oracle_mod.quantize_dq(Wbits)
    Wd = oracle_mod.bf16_to_f32(oracle_mod.dequant(q_full)).astype(np.float64)
    assert np.array_equal(w.packed.cpu().numpy(), q_full["packed"])
    Yr, _ = oracle_mod.linear_fwd(X64[rows_m], Wd, A64, B64, s)
    _close(inputs.to_f64(Y)[rows_m], Yr, "Y rows")
    if bwd:
        dY64 = inputs.to_f64(dY)
        dXr, _, _ = oracle_mod.linear_bwd(X64[rows_m], dY64[rows_m], Wd, A64, B64, s)
        _close(inputs.to_f64(dX)[rows_m], dXr, "dX rows")
        # dA, dB need every row: computed in full by the oracle
        dAr, dBr = oracle_mod.linear_bwd_adapters(X64, dY64, A64, B64, s)
        _close(inputs.to_f64(dA), dAr, "dA")
        _close(inputs.to_f64(dB), dBr, "dB")


@pytest.mark.parametrize("proj", [0])
def test_workload1_full(oracle_mod, proj):
    _sampled_rows_parity(oracle_mod, inputs.WORKLOADS[1], proj, 16, rows_n=16)


@pytest.mark.parametrize("proj,M", [(0, 1), (0, 4), (1, 8), (1, 32)])
def test_workload2_decode(oracle_mod, proj, M):
    _sampled_rows_parity(oracle_mod, inputs.WORKLOADS[2], proj, M, rows_n=M, bwd=False)


@pytest.mark.parametrize("M,N,K,r", [(512, 28672, 1024, 64), (384, 1024, 11008, 16)])
def test_multi_tile_pair_kernel_repeats_bit_identically(oracle_mod, M, N, K, r):
    """Several SM-pair tiles per pair, two LoRA steps per tile (r = 64): five runs of the
    forward and backward must agree bit for bit (the reduction orders are fixed, so any
    difference is a race) and the first must match the oracle."""
    s = 16.0 / r
    W, X, A, B, dY, Wd, w = _setup(oracle_mod, M, N, K, r, seed=7)
    Xc, Ac, Bc, dYc = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    outs = []
    for _ in range(5):
        Y = ops.qlora_linear_fwd(Xc, w, Ac, Bc, s)
        dX, dA, dB = ops.qlora_linear_bwd(Xc, dYc, w, Ac, Bc, s)
        outs.append([t.cpu() for t in (Y, dX, dA, dB)])
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    assert ops.qlora_last_path() == 3
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a, b)
    X64, A64, B64, dY64 = (inputs.to_f64(t) for t in (X, A, B, dY))
    Yr, _ = oracle_mod.linear_fwd(X64, Wd, A64, B64, s)
    dXr, dAr, dBr = oracle_mod.linear_bwd(X64, dY64, Wd, A64, B64, s)
    for name, got, ref in zip(("Y", "dX", "dA", "dB"), outs[0], (Yr, dXr, dAr, dBr)):
        _close(inputs.to_f64(got), ref, name)


@pytest.mark.parametrize("M,N,K,r,bwd", [(512, 28672, 1024, 16, False),   # SM pairs, 112 tiles stream-K
                                         (512, 4096, 4096, 16, False),    # SM pairs, one token tile, stream-K
                                         (512, 4096, 4096, 16, True),
                                         (512, 4096, 11008, 64, True),    # SM pairs, backward over 11008
                                         (1024, 4096, 11008, 16, True),   # SM pairs, backward, 172 tiles stream-K
                                         (100, 38912, 256, 16, False),    # single SM, 152 tiles
                                         (64, 512, 38912, 8, True),       # single SM, backward, 152 tiles
                                         (16, 4096, 28672, 64, True)])    # small-M backward (tcgen05)
def test_fused_kernels_repeat_bit_identically(M, N, K, r, bwd):
    """Fifty back-to-back calls give bit-identical outputs.  Every reduction order is fixed,
    so a difference can only come from a race between a stage's producer and its consumers
    (this caught packed stages being released while their shared loads were in flight)."""
    s = 16.0 / r
    W = inputs.weight(57, 0, N, K, 0.02, device="cuda")
    X = inputs.normal(67, (M, K), 1.0, "cuda")
    A = inputs.uniform(68, (r, K), 1.0 / np.sqrt(K), "cuda")
    B = inputs.normal(69, (N, r), 0.1, "cuda")
    dY = inputs.normal(70, (M, N), 1.0, "cuda")
    w = ops.nf4_quantize_dq(W)
    ws = ops.workspace(M, N, K, r)
    first = None
    same = torch.ones((), dtype=torch.bool, device="cuda")
    for _ in range(50):
        if bwd:
            out = ops.qlora_linear_bwd(X, dY, w, A, B, s, ws=ws)[0]
        else:
            out = ops.qlora_linear_fwd(X, w, A, B, s, ws=ws)
        if first is None:
            first = out.clone()
        else:
            same &= torch.equal(out, first)
    torch.cuda.synchronize()
    assert ops.qlora_device_status() == 0
    assert bool(same)
