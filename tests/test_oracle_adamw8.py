"""Pins for the oracle's 8-bit AdamW step of the adapters.

"Qlora Expert", Hyperparameter Guidance: paged_adamw_8bit (8-bit Adam to cut
optimizer memory; the paging is driver behaviour and out of scope).  The
pages give no state encoding; the reading is E4M3 codes with an fp32 absmax
scale per block of 256.  Pinned against:
  * torch's float8_e4m3fn conversion (a library implementation of the same
    IEEE-style format) for every code and for round-to-nearest-even encoding;
  * torch.optim.AdamW in fp64 for the parameter update (step 1 from a zero
    state, where the stored state's quantization does not yet enter, and step
    2 started from the oracle's dequantized step-1 state);
  * the quantization's own invariants (the block maximum maps to +-448, every
    value within half a quantum, all-zero blocks, a short last block).
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_quant_b200 import inputs


def _bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_e4m3_decode_every_code_matches_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    for c in codes:
        if np.isnan(ref[c]):
            assert c in (0x7f, 0xff)
            continue
        assert oracle_mod.e4m3_to_f32(int(c)) == ref[c], c


def test_e4m3_encode_matches_torch_and_rounds_to_even(oracle_mod):
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.5, 20000),
                        [0.0, -0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 448.0, -448.0, 447.9]]).astype(np.float32)
    # exact midpoints between neighbouring codes: ties go to the even mantissa
    vals = np.array(sorted({oracle_mod.e4m3_to_f32(c) for c in range(0x7f) if c != 0x7f}), np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.f32_to_e4m3(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates(oracle_mod):
    for v in (448.0, 463.9, 464.0, 500.0, 1e30):
        assert oracle_mod.f32_to_e4m3(v) == 0x7e
        assert oracle_mod.f32_to_e4m3(-v) == 0xfe
    assert oracle_mod.e4m3_to_f32(0x7e) == 448.0


def _torch_adamw(p64, g64, lr, b1, b2, eps, wd, state=None, step=1):
    p = torch.nn.Parameter(torch.from_numpy(p64.copy()))
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p.grad = torch.from_numpy(g64.copy())
    if state is not None:
        st = opt.state[p]
        st["step"] = torch.tensor(float(step - 1), dtype=torch.float64)
        st["exp_avg"] = torch.from_numpy(state[0].astype(np.float64))
        st["exp_avg_sq"] = torch.from_numpy(state[1].astype(np.float64))
    opt.step()
    return p.detach().numpy()


def _state_values(oracle_mod, code, scale):
    table = np.array([oracle_mod.e4m3_to_f32(c) if c not in (0x7f, 0xff) else np.nan for c in range(256)], np.float32)
    blk = np.arange(code.size) // oracle_mod.ADAM_BLOCK
    return (table[code] * scale[blk]).astype(np.float32)


@pytest.mark.parametrize("n", [1, 255, 256, 1000, 4096])
def test_first_two_steps_match_torch_adamw(oracle_mod, n):
    lr, b1, b2, eps, wd = 2e-4, 0.9, 0.999, 1e-8, 0.01
    p = _bits(inputs.normal(5, (n,), 0.02).float().numpy())
    g1 = _bits(inputs.normal(6, (n,), 0.001).float().numpy())
    g2 = _bits(inputs.normal(7, (n,), 0.001).float().numpy())
    st = oracle_mod.adamw8_state(n)
    p1 = p.copy()
    oracle_mod.adamw8_step(p1, g1, st, 1, lr, b1, b2, eps, wd)
    ref1 = _torch_adamw(_f32(p).astype(np.float64), _f32(g1).astype(np.float64), lr, b1, b2, eps, wd)
    # the fp32 update then one bf16 rounding: within one bf16 ulp of the fp64 result
    ulp = np.abs(_f32(p1)).astype(np.float64) * 2.0 ** -7
    assert np.all(np.abs(_f32(p1) - ref1) <= ulp + 1e-30)
    # step 2 from the oracle's (quantized) state, fed to torch as exact values
    m1 = _state_values(oracle_mod, st[0], st[1])
    v1 = _state_values(oracle_mod, st[2], st[3])
    p2 = p1.copy()
    oracle_mod.adamw8_step(p2, g2, st, 2, lr, b1, b2, eps, wd)
    ref2 = _torch_adamw(_f32(p1).astype(np.float64), _f32(g2).astype(np.float64), lr, b1, b2, eps, wd,
                        state=(m1, v1), step=2)
    ulp = np.abs(_f32(p2)).astype(np.float64) * 2.0 ** -7
    assert np.all(np.abs(_f32(p2) - ref2) <= ulp + 1e-30)


def test_state_quantization_invariants(oracle_mod):
    n = 3 * 256 + 77
    rng = np.random.default_rng(9)
    p = _bits(rng.standard_normal(n) * 0.02)
    g = _bits(rng.standard_normal(n) * 10.0 ** rng.uniform(-6, -1, n))
    g[256:512] = 0                                          # an all-zero gradient block
    st = oracle_mod.adamw8_state(n)
    b1, b2 = 0.9, 0.999
    oracle_mod.adamw8_step(p, g, st, 1, 1e-3, b1, b2, 1e-8, 0.0)
    # from a zero state the new moments are omb * g and omb2 * g^2, omb = fl32(1 - fl32(b))
    omb1 = np.float32(1.0 - np.float64(np.float32(b1)))
    omb2 = np.float32(1.0 - np.float64(np.float32(b2)))
    m_true = (omb1 * _f32(g)).astype(np.float32)
    v_true = (omb2 * (_f32(g) * _f32(g)).astype(np.float32)).astype(np.float32)
    for code, scale, true in ((st[0], st[1], m_true), (st[2], st[3], v_true)):
        vals = _state_values(oracle_mod, code, scale)
        for b in range(scale.size):
            sl = slice(256 * b, min(n, 256 * b + 256))
            amax = np.abs(true[sl]).max()
            assert scale[b] == np.float32(amax / np.float32(448.0))
            if amax == 0:
                assert not code[sl].any()
                continue
            assert np.abs(code[sl].astype(np.int32) & 0x7f).max() == 0x7e       # the maximum maps to 448
            # E4M3: 3 mantissa bits, so half a quantum is at most 2^-4 of the value in the normal
            # range, and 2^-10 (half the subnormal step 2^-9) times the scale below it
            err = np.abs(vals[sl].astype(np.float64) - true[sl])
            bound = np.maximum(np.abs(true[sl]) * 2.0 ** -4, float(scale[b]) * 2.0 ** -10) * 1.0001
            assert np.all(err <= bound)
