"""Host checks of the SM-pair kernel's stream-K schedule (no GPU needed).

The library's own span iterator (the one the kernel runs, called through
qlora_pair_spans) is checked for every schedule that the benchmark workloads
and the GPU tests produce, for several pair counts:
  * every (tile, reduction step) unit is taken by exactly one pair;
  * each tile has exactly one owner span (the one ending the tile);
  * the lower pairs whose spans cover the owner's missing head are exactly
    the contiguous range the kernel's epilogue computes (pf .. pair - 1) and
    adds in that order;
  * a pair has at most one span that does not end its tile (its partial-tile
    slot is unique), and it is the pair's first span, taken first;
  * a span that adds partials is its pair's last, so its owner waits only for
    lower pairs, which computed their part first; the shared-memory staging
    the kernel uses for that fix-up is free only then.
"""
import pytest

from bit_nf4_quantized_quant_b200 import _ops as ops


def cdiv(a, b):
    return -(-a // b)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_nf4_quantized_quant_b200 import build
    build.build()


SHAPES = [  # M, N, K, r: the training workloads, the 70B shapes, and the GPU tests' multi-tile cases
    (2048, 4096, 4096, 16), (2048, 11008, 4096, 16), (2048, 4096, 11008, 16),
    (512, 8192, 8192, 64), (512, 28672, 8192, 64), (512, 8192, 28672, 64), (512, 4096, 4096, 16),
    (4096, 8192, 8192, 64), (4096, 28672, 8192, 64), (4096, 8192, 28672, 64),
    (512, 11008, 1024, 16), (520, 1024, 11008, 32), (1024, 4096, 11008, 16), (512, 28672, 1024, 16),
    (2048, 768, 1024, 16), (1000, 520, 1088, 64), (160, 512, 1024, 16),
]


def _owner_first_pair(pair, npairs, ntiles, nsteps, tile):
    """The kernel's epilogue: the lowest pair whose run reaches into this tile."""
    U = ntiles * nsteps
    tb = tile * nsteps
    pf = pair - 1
    while pf > 0 and pf * U // npairs > tb:
        pf -= 1
    return pf


@pytest.mark.parametrize("M,N,K,r", SHAPES)
@pytest.mark.parametrize("bwd", [False, True])
@pytest.mark.parametrize("pairs", [74, 73, 70, 64])
def test_stream_k_spans(M, N, K, r, bwd, pairs):
    n_out, n_red = (K, N) if bwd else (N, K)
    mt, ntiles, sk = ops.pair_schedule(M, n_out, pairs, bwd)
    assert ntiles == cdiv(M, 256 * mt) * cdiv(n_out, 256)
    if not sk:
        # whole waves, too few tiles, or whole tiles on at least 3/4 of the pairs
        assert ntiles % pairs == 0 or 3 * ntiles < pairs or 3 * pairs <= 4 * ntiles <= 4 * pairs
        return
    assert 3 * ntiles >= pairs                        # tiles split at most three ways
    rp = cdiv(r, 16) * 16
    nsteps = cdiv(n_red, 64) + cdiv(cdiv(2 * rp, 64) * 64, 64)
    taken = {}
    spans = [ops.pair_spans(ntiles, nsteps, p, pairs) for p in range(pairs)]
    partial_slot = {}
    for p, sp in enumerate(spans):
        for i, (t, s0, s1) in enumerate(sp):
            assert 0 <= t < ntiles and 0 <= s0 < s1 <= nsteps
            for s in range(s0, s1):
                assert (t, s) not in taken, (t, s)
                taken[(t, s)] = p
            if s1 < nsteps:
                assert p not in partial_slot and i == 0
                partial_slot[p] = t
    assert len(taken) == ntiles * nsteps
    for p, sp in enumerate(spans):
        for i, (t, s0, s1) in enumerate(sp):
            if s1 == nsteps and s0 > 0:
                assert i == len(sp) - 1
                pf = _owner_first_pair(p, pairs, ntiles, nsteps, t)
                contributors = sorted(q for q, tt in partial_slot.items() if tt == t)
                assert contributors == list(range(pf, p))
                assert {taken[(t, s)] for s in range(s0)} == set(contributors)
    owners = {}
    for p, sp in enumerate(spans):
        for (t, s0, s1) in sp:
            if s1 == nsteps:
                assert t not in owners
                owners[t] = p
    assert len(owners) == ntiles


def test_schedule_of_the_default_workload():
    # 7B block at 2048 tokens on 74 pairs: 4096-wide outputs are 64 two-token-tile tiles
    # (whole tiles; the backward leaves 10 pairs to dB and dA), 11008-wide ones 172
    assert ops.pair_schedule(2048, 4096, 74, False) == (2, 64, False)
    assert ops.pair_schedule(2048, 4096, 74, True) == (2, 64, False)
    assert ops.pair_schedule(2048, 11008, 74, False) == (2, 172, True)
    assert ops.pair_schedule(2048, 11008, 74, True) == (2, 172, True)
    assert ops.pair_schedule(160, 1024, 74, False)[2] is False
    # 70B 8192-wide outputs at 512 tokens: 64 one-token-tile tiles, or 32 of two; both
    # directions take two (decode-bound otherwise) with tiles split over two or three pairs
    assert ops.pair_schedule(512, 8192, 74, False) == (2, 32, True)
    assert ops.pair_schedule(512, 8192, 74, True) == (2, 32, True)
    assert ops.pair_schedule(512, 1024, 74, False) == (1, 8, False)
    # 7B 4096-wide outputs at 512 tokens: 32 one-token-tile tiles (16 of two: too few to
    # promote), dealt stream-K over all pairs in both directions
    assert ops.pair_schedule(512, 4096, 74, False) == (1, 32, True)
    assert ops.pair_schedule(512, 4096, 74, True) == (1, 32, True)


def test_bad_arguments():
    import ctypes
    with pytest.raises(ops.QLoRAError):
        ops.pair_schedule(0, 4096, 74, False)
    buf = (ctypes.c_int64 * 3)()
    assert ops.lib().qlora_pair_spans(10, 5, 3, 2, buf, 1) == ops.QLORA_ERR_VALUE     # pair >= npairs
    assert ops.lib().qlora_pair_spans(10, 5, 0, 2, None, 1) == ops.QLORA_ERR_NULL
