"""The data-parallel (N > 1) path of bench.py, on CPU with gloo, world size 2.

Every rank draws its own batch (bench.rank_batch), computes the adapter
gradients of its batch (here with the oracle, on the GPU with the library),
packs them into the flat buffer of bench.grad_layout and all-reduces it once.
The sum over ranks must equal the gradients of the concatenated batch, since
dA = s U^T X and dB = s dY^T T are sums over tokens; dX and Y stay rank-local.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from bit_nf4_quantized_quant_b200 import inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _small_workload():
    wl = inputs.Workload(90, "dp-test", [inputs.Projection("a", 64, 128), inputs.Projection("b", 96, 64)], [8], 4,
                         8.0, 0.02, True)
    return wl


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    wl = _small_workload()
    M, r, s = 8, wl.r, wl.scaling
    offs, total = bench.grad_layout([(p.N, p.K) for p in wl.projections], r)
    flat = torch.zeros(total, dtype=torch.float64)
    for i, p in enumerate(wl.projections):
        _, A, B, _ = inputs.layer_inputs(wl, i, M, with_dy=False)
        X, dY = bench.rank_batch(wl, i, M, rank, world, "cpu")
        dA, dB = oracle.linear_bwd_adapters(inputs.to_f64(X), inputs.to_f64(dY), inputs.to_f64(A),
                                            inputs.to_f64(B), s)
        oa, ob = offs[i]
        flat[oa:oa + dA.size] = torch.from_numpy(dA.reshape(-1))
        flat[ob:ob + dB.size] = torch.from_numpy(dB.reshape(-1))
    dist.all_reduce(flat)
    if rank == 0:
        np.save(out_path, flat.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_dp_gradient_allreduce_equals_full_batch(tmp_path, oracle_mod):
    world = 2
    out = str(tmp_path / "flat.npy")
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    flat = np.load(out)
    wl = _small_workload()
    M, r, s = 8, wl.r, wl.scaling
    offs, total = bench.grad_layout([(p.N, p.K) for p in wl.projections], r)
    assert flat.size == total
    for i, p in enumerate(wl.projections):
        _, A, B, _ = inputs.layer_inputs(wl, i, M, with_dy=False)
        Xs, dYs = zip(*(bench.rank_batch(wl, i, M, k, world, "cpu") for k in range(world)))
        X = np.concatenate([inputs.to_f64(x) for x in Xs])
        dY = np.concatenate([inputs.to_f64(y) for y in dYs])
        assert not np.array_equal(inputs.to_f64(Xs[0]), inputs.to_f64(Xs[1]))   # distinct batches
        dA, dB = oracle_mod.linear_bwd_adapters(X, dY, inputs.to_f64(A), inputs.to_f64(B), s)
        oa, ob = offs[i]
        assert np.allclose(flat[oa:oa + dA.size], dA.reshape(-1), rtol=1e-12, atol=1e-12)
        assert np.allclose(flat[ob:ob + dB.size], dB.reshape(-1), rtol=1e-12, atol=1e-12)


def _worker_bf16(rank, world, port, out_path):
    """The bench's dtype path: each rank's adapter gradients arrive in bf16 (the library
    writes dA, dB in bf16 into the flat buffer) and the flat bf16 buffer is all-reduced."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    wl = _small_workload()
    M, r, s = 8, wl.r, wl.scaling
    offs, total = bench.grad_layout([(p.N, p.K) for p in wl.projections], r)
    flat = torch.zeros(total, dtype=torch.bfloat16)
    for i, p in enumerate(wl.projections):
        _, A, B, _ = inputs.layer_inputs(wl, i, M, with_dy=False)
        X, dY = bench.rank_batch(wl, i, M, rank, world, "cpu")
        dA, dB = oracle.linear_bwd_adapters(inputs.to_f64(X), inputs.to_f64(dY), inputs.to_f64(A),
                                            inputs.to_f64(B), s)
        oa, ob = offs[i]
        flat[oa:oa + dA.size] = torch.from_numpy(dA.reshape(-1)).to(torch.bfloat16)
        flat[ob:ob + dB.size] = torch.from_numpy(dB.reshape(-1)).to(torch.bfloat16)
    dist.all_reduce(flat)
    if rank == 0:
        np.save(out_path, flat.float().numpy().astype(np.float64))
    dist.barrier()
    dist.destroy_process_group()


def test_dp_bf16_allreduce_within_the_stated_bound(tmp_path, oracle_mod):
    """bf16 gradients summed in bf16 over N ranks.  bf16 keeps 8 significant bits, so a
    round-to-nearest conversion is off by at most u = 2^-8 of the value and any faithful
    rounding of a partial sum by less than 2u.  Each rank's gradient is rounded once to
    bf16 and the sum goes through at most N - 1 roundings, so
    |sum - full-batch gradient| <= (2N - 1) 2^-8 sum_i |g_i|: the bound stated for the
    bench's all-reduce, on top of the library's own per-rank tolerance."""
    world = 2
    out = str(tmp_path / "flat_bf16.npy")
    mp.start_processes(_worker_bf16, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    flat = np.load(out)
    wl = _small_workload()
    M, r, s = 8, wl.r, wl.scaling
    offs, total = bench.grad_layout([(p.N, p.K) for p in wl.projections], r)
    for i, p in enumerate(wl.projections):
        _, A, B, _ = inputs.layer_inputs(wl, i, M, with_dy=False)
        per_rank = []
        for k in range(world):
            X, dY = bench.rank_batch(wl, i, M, k, world, "cpu")
            per_rank.append(oracle_mod.linear_bwd_adapters(inputs.to_f64(X), inputs.to_f64(dY), inputs.to_f64(A),
                                                           inputs.to_f64(B), s))
        oa, ob = offs[i]
        for j, (o, n) in enumerate(((oa, r * p.K), (ob, p.N * r))):
            ref = sum(g[j] for g in per_rank).reshape(-1)
            mag = sum(np.abs(g[j]) for g in per_rank).reshape(-1)
            err = np.abs(flat[o:o + n] - ref)
            assert np.all(err <= (2 * world - 1) * 2.0 ** -8 * mag * 1.0001 + 1e-30)
            assert err.max() > 0              # bf16 really rounds here: the bound is exercised


def test_grad_layout_disjoint():
    offs, total = bench.grad_layout([(64, 128), (96, 64), (8, 64)], 4)
    spans = []
    for (oa, ob), (N, K) in zip(offs, [(64, 128), (96, 64), (8, 64)]):
        spans += [(oa, oa + 4 * K), (ob, ob + N * 4)]
    spans.sort()
    assert spans[0][0] == 0 and spans[-1][1] == total
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
