"""Host-side logic of bench.py (no GPU): byte and flop accounting, the
gradient layout of the data-parallel all-reduce, and the source hash that
keys the recorded DRAM-traffic figures."""
import os

import bench


def test_nf4_bytes_closed_form():
    # 4 bits per weight + one int8 code per 64 weights + fp32 scale and mean per 16384 weights
    for N, K in ((4096, 4096), (11008, 4096), (8192, 28672)):
        assert bench.nf4_bytes(N, K) * 8 == N * K * 4.12890625


def test_flops_are_the_sum_of_the_layer_products():
    M, N, K, r = 2048, 11008, 4096, 16
    mm = lambda a, b, c: 2 * a * b * c                     # an [a, c] x [c, b] product
    fwd = mm(M, N, K) + mm(M, r, K) + mm(M, N, r)           # X W'^T, T = X A^T, T B^T
    bwd = (mm(M, K, N) + mm(M, r, N) + mm(M, K, r)          # dY W', U = dY B, U A
           + mm(r, K, M) + mm(N, r, M))                     # dA = U^T X, dB = dY^T T
    assert bench.flops_fwd_bwd(M, N, K, r) == fwd + bwd


def test_traffic_entries_name_existing_sources():
    d = os.path.join(bench.ROOT, "bit_nf4_quantized_quant_b200", "csrc")
    for key, e in bench.TRAFFIC.items():
        assert e["bytes_per_launch"] > 0, key
        for f in e["files"]:
            assert os.path.exists(os.path.join(d, f)), (key, f)
        assert len(e["src"]) == 12


def test_src_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "bit_nf4_quantized_quant_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "k.cuh").write_text("int a = 1;  // one\n/* block\n comment */\nint b = 2;\n")
    h0 = bench.src_hash(["k.cuh"])
    (csrc / "k.cuh").write_text("// header\nint a = 1;\n\nint b = 2;  /* two */\n")
    assert bench.src_hash(["k.cuh"]) == h0
    (csrc / "k.cuh").write_text("int a = 1;\nint b = 3;\n")
    assert bench.src_hash(["k.cuh"]) != h0


def test_step_work_sums_the_projections():
    from bit_nf4_quantized_quant_b200 import inputs
    wl = inputs.WORKLOADS[3]
    f, b = bench.step_work(wl, 2048)
    assert f == sum(bench.flops_fwd_bwd(2048, p.N, p.K, wl.r) for p in wl.projections)
    # fwd+bwd streams every NF4 weight twice
    assert b > 2 * sum(bench.nf4_bytes(p.N, p.K) for p in wl.projections)
    wl2 = inputs.WORKLOADS[2]
    f2, b2 = bench.step_work(wl2, 1)
    assert f2 == sum(2 * p.N * p.K + 2 * wl2.r * (p.N + p.K) for p in wl2.projections)
    assert b2 == sum(bench.nf4_bytes(p.N, p.K) + 2 * (p.K + wl2.r * p.K + p.N * wl2.r + p.N)
                     for p in wl2.projections)


def test_reference_arm_runs_on_the_host(capsys):
    """The reference arm (the oracle on the host cores) prints one JSON line with the
    reference keys, on the single-linear workload."""
    import json
    import sys
    argv = sys.argv
    try:
        sys.argv = ["bench.py", "--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "0"]
        bench.main()
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
