"""GPU parity of adamw_8bit_step against the oracle: parameters (bf16), both
8-bit moment codes and their fp32 scales bit-exact after each of three chained
steps, including short last blocks, zero gradients and weight decay
("Qlora Expert", Hyperparameter Guidance: paged_adamw_8bit; the paging itself
is out of scope)."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import _ops as ops
from bit_nf4_quantized_quant_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(oracle_mod, n, seed, lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=0.01, steps=3, g_std=1e-3,
         zero_every=0):
    p = inputs.normal(seed, (n,), 0.02)
    gs = [inputs.normal(seed + 1 + k, (n,), g_std) for k in range(steps)]
    if zero_every:
        for g in gs:
            g[::zero_every] = 0
    p_dev = p.cuda()
    st = ops.AdamW8State.zeros(n)
    p_ref = inputs.bf16_bits(p).copy()
    st_ref = oracle_mod.adamw8_state(n)
    for k, g in enumerate(gs, start=1):
        ops.adamw_8bit_step(p_dev, g.cuda(), st, k, lr, b1, b2, eps, wd)
        oracle_mod.adamw8_step(p_ref, inputs.bf16_bits(g).copy(), st_ref, k, lr, b1, b2, eps, wd)
        torch.cuda.synchronize()
        assert np.array_equal(inputs.bf16_bits(p_dev), p_ref), f"p differs after step {k}"
        assert np.array_equal(st.m_code.cpu().numpy(), st_ref[0]), f"m codes differ after step {k}"
        assert np.array_equal(st.m_scale.cpu().numpy().view(np.uint32), st_ref[1].view(np.uint32))
        assert np.array_equal(st.v_code.cpu().numpy(), st_ref[2]), f"v codes differ after step {k}"
        assert np.array_equal(st.v_scale.cpu().numpy().view(np.uint32), st_ref[3].view(np.uint32))


@pytest.mark.parametrize("n", [1, 7, 8, 255, 256, 257, 1000, 4099, 65536 + 40])
def test_adamw8_bit_exact(oracle_mod, n):
    _run(oracle_mod, n, seed=n % 97)


def test_adamw8_zero_gradients_and_decay(oracle_mod):
    _run(oracle_mod, 3000, seed=11, zero_every=3, wd=0.1, lr=1e-3)


def test_adamw8_wide_gradient_range(oracle_mod):
    # gradients spanning many decades exercise the E4M3 subnormals and the saturating end
    _run(oracle_mod, 2048, seed=12, g_std=1.0, b1=0.5, b2=0.9, lr=1e-2)


def test_adamw8_7b_block_adapters(oracle_mod):
    # the flat dA/dB buffer of the 7 projections of a 7B block at r = 16
    wl = inputs.WORKLOADS[3]
    n = sum(wl.r * (p.N + p.K) for p in wl.projections)
    _run(oracle_mod, n, seed=13, steps=2)


def test_adamw8_rejects_bad_arguments():
    p = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    st = ops.AdamW8State.zeros(16)
    with pytest.raises(ops.QLoRAError) as e:
        ops.adamw_8bit_step(p, p, st, 0, 1e-3)
    assert e.value.code == -9
    with pytest.raises(ops.QLoRAError) as e:
        ops.adamw_8bit_step(p, p, st, 1, 1e-3, beta1=1.0)
    assert e.value.code == -9
