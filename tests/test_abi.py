"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

The library must load, export every function include/qlora_nf4.h declares,
compute the same fp32 codebook as the oracle (two independent inverse-normal
methods: bisection on erfc in the library, AS 241 in the oracle), and reject
bad arguments with the documented error codes before touching a device.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_nf4_quantized_quant_b200 import _ops as ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_quant_b200 import build
    build.build()
    return ops.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    expected = {"nf4_codebook", "nf4dq_sizes", "nf4_quantize_dq", "nf4_dequant", "qlora_workspace_bytes",
                "qlora_linear_fwd", "qlora_linear_bwd", "qlora_status_string", "qlora_device_status",
                "qlora_last_path"}
    assert expected <= set(names)


def test_codebook_matches_oracle_bit_for_bit(lib, oracle_mod):
    cb = np.array(ops.nf4_codebook(), np.float32)
    _, o32 = oracle_mod.codebook()
    assert np.array_equal(cb.view(np.uint32), o32.view(np.uint32))


def test_sizes_closed_form(lib):
    assert ops.nf4dq_sizes(4096, 4096) == (8388608, 262144, 1024)
    assert ops.nf4dq_sizes(11008, 4096) == (22544384, 704512, 2752)
    assert ops.nf4dq_sizes(8192, 28672) == (117440512, 3670016, 14336)
    assert ops.nf4dq_sizes(5, 64) == (160, 5, 1)
    for N, K in [(4096, 4096), (11008, 4096), (28672, 8192)]:
        pb, nb, ng = ops.nf4dq_sizes(N, K)
        bits = (pb + nb + 8 * ng) * 8 / (N * K)
        assert bits == 4.12890625


def test_size_errors(lib):
    pb = ctypes.c_int64()
    assert lib.nf4dq_sizes(4, 96, ctypes.byref(pb), None, None) == -2
    assert lib.nf4dq_sizes(0, 64, None, None, None) == -2
    assert lib.nf4dq_sizes(4, -64, None, None, None) == -2


def test_workspace_bytes(lib):
    assert ops.qlora_workspace_bytes(16, 4096, 4096, 16) > 0
    assert ops.qlora_workspace_bytes(16, 4096, 4096, 0) == 0
    assert ops.qlora_workspace_bytes(16, 4096, 4096, 257) == 0
    assert ops.qlora_workspace_bytes(16, 4100, 4096, 16) == 0   # N % 8
    assert ops.qlora_workspace_bytes(16, 4096, 4000, 16) == 0   # K % 64
    assert ops.qlora_workspace_bytes(0, 4096, 4096, 16) == 0
    # grows with M, never shrinks
    assert ops.qlora_workspace_bytes(2048, 4096, 4096, 16) >= ops.qlora_workspace_bytes(16, 4096, 4096, 16)


def test_argument_errors_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)           # never dereferenced: every call below is rejected first
    # null pointers
    assert lib.nf4_quantize_dq(None, 64, 64, fake, fake, fake, fake, None) == -1
    assert lib.nf4_dequant(None, fake, None) == -1
    w = ops._Weight(0x1000, 0x1000, 0x1000, 0x1000, 64, 64)
    assert lib.qlora_linear_fwd(None, 4, ctypes.byref(w), fake, fake, 16, 2.0, fake, None, fake, 1 << 30, None) == -1
    # bad shapes
    assert lib.nf4_quantize_dq(fake, 64, 96, fake, fake, fake, fake, None) == -2
    wbad = ops._Weight(0x1000, 0x1000, 0x1000, 0x1000, 64, 100)
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(wbad), fake, fake, 16, 2.0, fake, None, fake, 1 << 30,
                                None) == -2
    assert lib.qlora_linear_fwd(fake, 0, ctypes.byref(w), fake, fake, 16, 2.0, fake, None, fake, 1 << 30, None) == -2
    # K beyond QLORA_MAX_K (2^21): rejected before any launch, no workspace size
    wbig = ops._Weight(0x1000, 0x1000, 0x1000, 0x1000, 64, (1 << 21) + 64)
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(wbig), fake, fake, 16, 2.0, fake, None, fake, 1 << 40,
                                None) == -2
    assert lib.qlora_linear_bwd(fake, fake, 4, ctypes.byref(wbig), fake, fake, 16, 2.0, None, fake, fake, fake, fake,
                                1 << 40, None) == -2
    assert lib.qlora_workspace_bytes(4, 64, (1 << 21) + 64, 16) == 0
    assert lib.qlora_workspace_bytes(4, 64, 1 << 21, 16) > 0
    # rank
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 0, 2.0, fake, None, fake, 1 << 30, None) == -3
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 300, 2.0, fake, None, fake, 1 << 30,
                                None) == -3
    # scaling must be finite
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 16, float("nan"), fake, None, fake, 1 << 30,
                                None) == -9
    # misaligned activations / packed weights
    mis = P(0x1002)
    assert lib.qlora_linear_fwd(mis, 4, ctypes.byref(w), fake, fake, 16, 2.0, fake, None, fake, 1 << 30, None) == -4
    wmis = ops._Weight(0x1001, 0x1000, 0x1000, 0x1000, 64, 64)
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(wmis), fake, fake, 16, 2.0, fake, None, fake, 1 << 30,
                                None) == -4
    # workspace missing
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 16, 2.0, fake, None, None, 0, None) == -5
    # backward: no gradient output may be missing
    assert lib.qlora_linear_bwd(fake, fake, 4, ctypes.byref(w), fake, fake, 16, 2.0, None, fake, fake, None, fake,
                                1 << 30, None) == -1


def test_status_strings(lib):
    for c in range(-9, 1):
        assert len(ops.status_string(c)) > 0
    assert ops.status_string(-4).startswith("pointer not 16-byte aligned")
