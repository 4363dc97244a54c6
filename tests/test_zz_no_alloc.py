"""The allocation-free forward (qlora_linear_fwd_noalloc) on the GPU.

Some callers cannot allocate device memory: another allocator already owns
the device's memory, or the call happens inside a framework callback that
forbids allocation.  For them the library offers a forward whose scratch is
a fixed static device array instead of a caller workspace.  This file runs
last (pytest collects it last by name) and must pass both alone in a fresh
process and after every other test: it checks the new entry point, called
twice in a row through the C ABI, against qlora_linear_fwd with its own
workspace.  Both run the same kernels with fixed reduction orders, so the
outputs must agree bit for bit (a stricter check than the 1e-2 tolerance of
the parity tests: a partial-sum slot read stale from an earlier call on the
shared scratch would show here).
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import _ops as ops
from bit_nf4_quantized_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,r", [(1, 11008, 4096, 16), (16, 4096, 4096, 16), (160, 1024, 2048, 64)])
def test_noalloc_forward_matches_workspace_forward(M, N, K, r):
    assert ops.qlora_workspace_bytes(M, N, K, r) <= (8 << 20)
    W = inputs.weight(40, 0, N, K, 0.02, device="cuda")
    w = ops.nf4_quantize_dq(W)
    X = inputs.normal(41, (M, K), 1.0, "cuda")
    A = inputs.uniform(42, (r, K), 1.0 / np.sqrt(K), "cuda")
    B = inputs.normal(43, (N, r), 0.1, "cuda")
    s = 32.0 / r
    ref_T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    ref = ops.qlora_linear_fwd(X, w, A, B, s, T_out=ref_T)
    for _ in range(2):                     # two calls in a row on the shared static scratch
        T = torch.empty_like(ref_T)
        Y = ops.qlora_linear_fwd_noalloc(X, w, A, B, s, T_out=T)
        torch.cuda.synchronize()
        assert ops.qlora_device_status() == 0
        assert torch.equal(Y, ref)
        assert torch.equal(T, ref_T)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = ops.lib()
    M, N, K, r = 4096, 28672, 8192, 64
    assert ops.qlora_workspace_bytes(M, N, K, r) > (8 << 20)
    fake = ctypes.c_void_p(0x1000)          # never dereferenced: the call is rejected before any launch
    wst = ops._Weight(0x1000, 0x1000, 0x1000, 0x1000, N, K)
    rc = lib.qlora_linear_fwd_noalloc(fake, M, ctypes.byref(wst), fake, fake, r, 0.25, fake, None, None)
    assert rc == -10
    assert "no-alloc" in ops.status_string(rc)
