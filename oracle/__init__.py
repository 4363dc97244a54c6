"""CPU oracle for the QLoRA frozen-NF4 linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` are the only callers.  The product
library never imports, links or runs anything here, and nothing here imports
the product package.

Two parts:

* ``nf4_oracle.c`` (built into ``liboracle_nf4.so`` with gcc, loaded through
  ctypes): the codebook, block absmax, NF4 encoding, double quantization and
  dequantization, bit for bit, in plain loops.
* the forward and backward of the linear layer below, written out as their
  definitions in fp64 with numpy matrix products as the only library step.

Page citations (title, section):

* "QLoRA Guide" (dataaihub.co), "How QLoRA Works / Forward pass" and its
  "Dequant + LoRA path" diagram: the input goes both through the dequantized
  frozen weight and through LoRA A then B, and the two are summed; only A and
  B get gradients, the dequantized weight is a constant for autograd.
* "QLoRA Implementation Details (2025 Edition)", "Step 4: Apply LoRA
  Adapters": the LoRA scaling is alpha / r.
* "QLORA: Efficient Finetuning of Quantized LLMs" (imaddabbura.github.io),
  "Notes": every forward/backward loads the 4-bit weights, dequantizes to
  BF16, multiplies, and computes gradients only for the adapters, which are
  stored and trained in BF16.

Parity unpinned (no value on the pages to pin against, only self-consistency
and mathematics): the codebook values themselves (reading R1), the tie rule
(R2), the nibble order (R3) and the int8 form of the double quantization
(R4).  Everything else is pinned by the tests in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_nf4.so")

NF4_BLOCK = 64
DQ_GROUP = 256


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no fused multiply-add contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.oracle_ppnd16.restype = ctypes.c_double
        L.oracle_ppnd16.argtypes = [ctypes.c_double]
        L.oracle_nf4_codebook.argtypes = [P, P]
        L.oracle_nf4_midpoints.argtypes = [P, P]
        L.oracle_nf4_encode_value.restype = ctypes.c_int
        L.oracle_nf4_encode_value.argtypes = [ctypes.c_float, P]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_block_absmax.argtypes = [P, i64, P]
        L.oracle_double_quant.argtypes = [P, i64, P, P, P]
        L.oracle_quantize_dq.restype = ctypes.c_int
        L.oracle_quantize_dq.argtypes = [P, i64, i64, P, P, P, P, P]
        L.oracle_block_constant.restype = ctypes.c_float
        L.oracle_block_constant.argtypes = [ctypes.c_int8, ctypes.c_float, ctypes.c_float]
        L.oracle_dequant.restype = ctypes.c_int
        L.oracle_dequant.argtypes = [P, P, P, P, i64, i64, P]
        L.oracle_dequant_rows.restype = ctypes.c_int
        L.oracle_dequant_rows.argtypes = [P, P, P, P, i64, i64, P, i64, P]
        i32 = ctypes.c_int
        L.oracle_fp4_codebook.argtypes = [P, P]
        L.oracle_codebook.restype = i32
        L.oracle_codebook.argtypes = [i32, P]
        L.oracle_encode_value_qt.restype = i32
        L.oracle_encode_value_qt.argtypes = [i32, ctypes.c_float]
        L.oracle_quantize_dq_qt.restype = i32
        L.oracle_quantize_dq_qt.argtypes = [i32, P, i64, i64, P, P, P, P, P]
        L.oracle_dequant_qt.restype = i32
        L.oracle_dequant_qt.argtypes = [i32, P, P, P, P, i64, i64, P, i64, P]
        L.oracle_e4m3_to_f32.restype = ctypes.c_float
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.oracle_adamw8_step.restype = i32
        L.oracle_adamw8_step.argtypes = [P, P, i64, P, P, P, P, i64, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                         ctypes.c_float, ctypes.c_float]
        L.oracle_philox4x64.argtypes = [P, P, P]
        L.oracle_dropout_mask.restype = i32
        L.oracle_dropout_mask.argtypes = [ctypes.c_uint64, ctypes.c_uint64, i64, i64, ctypes.c_float, P]
        L.oracle_dequant_merge.restype = i32
        L.oracle_dequant_merge.argtypes = [i32, P, P, P, P, i64, i64, P, P, i32, ctypes.c_float, P, i64, P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# codebook and scalar encoding
# --------------------------------------------------------------------------
def ppnd16(p: float) -> float:
    """Inverse standard normal CDF (Wichura 1988, AS 241)."""
    return lib().oracle_ppnd16(float(p))


def codebook():
    """The 16 NF4 levels: (fp64 before rounding, fp32 as used)."""
    v64 = np.zeros(16, np.float64)
    v32 = np.zeros(16, np.float32)
    lib().oracle_nf4_codebook(_ptr(v64), _ptr(v32))
    return v64, v32


def midpoints(L32: np.ndarray | None = None) -> np.ndarray:
    if L32 is None:
        L32 = codebook()[1]
    L32 = np.ascontiguousarray(L32, np.float32)
    m = np.zeros(15, np.float32)
    lib().oracle_nf4_midpoints(_ptr(L32), _ptr(m))
    return m


def encode_value(x: float, m: np.ndarray | None = None) -> int:
    if m is None:
        m = midpoints()
    m = np.ascontiguousarray(m, np.float32)
    return lib().oracle_nf4_encode_value(ctypes.c_float(float(x)), _ptr(m))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns (uint16) to fp32."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_scalar(f: float) -> int:
    return int(lib().oracle_f32_to_bf16(ctypes.c_float(f)))


# --------------------------------------------------------------------------
# quantize / double-quant / dequant
# --------------------------------------------------------------------------
def quantize_dq(W_bits: np.ndarray):
    """bf16 W [N, K] (raw uint16 bits) -> dict(packed, codes, scale, mean, absmax)."""
    W_bits = np.ascontiguousarray(W_bits, np.uint16)
    N, K = W_bits.shape
    nblocks = N * K // NF4_BLOCK
    G = (nblocks + DQ_GROUP - 1) // DQ_GROUP
    packed = np.zeros((N, K // 2), np.uint8)
    codes = np.zeros(nblocks, np.int8)
    scale = np.zeros(G, np.float32)
    mean = np.zeros(G, np.float32)
    absmax = np.zeros(nblocks, np.float32)
    rc = lib().oracle_quantize_dq(_ptr(W_bits), N, K, _ptr(packed), _ptr(codes), _ptr(scale), _ptr(mean),
                                  _ptr(absmax))
    if rc != 0:
        raise ValueError(f"oracle_quantize_dq rejected shape {W_bits.shape}")
    return dict(packed=packed, codes=codes, scale=scale, mean=mean, absmax=absmax, N=N, K=K)


def double_quant(absmax: np.ndarray):
    absmax = np.ascontiguousarray(absmax, np.float32)
    nb = absmax.size
    G = (nb + DQ_GROUP - 1) // DQ_GROUP
    codes = np.zeros(nb, np.int8)
    scale = np.zeros(G, np.float32)
    mean = np.zeros(G, np.float32)
    lib().oracle_double_quant(_ptr(absmax), nb, _ptr(codes), _ptr(scale), _ptr(mean))
    return codes, scale, mean


def block_constant(code: int, scale: float, mean: float) -> float:
    return float(lib().oracle_block_constant(ctypes.c_int8(int(code)), ctypes.c_float(scale),
                                             ctypes.c_float(mean)))


def dequant(q: dict) -> np.ndarray:
    """NF4-DQ -> bf16 W' [N, K] as raw uint16 bits."""
    N, K = q["N"], q["K"]
    out = np.zeros((N, K), np.uint16)
    rc = lib().oracle_dequant(_ptr(q["packed"]), _ptr(q["codes"]), _ptr(q["scale"]), _ptr(q["mean"]),
                              N, K, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequant rejected its arguments")
    return out


def dequant_rows(q: dict, rows) -> np.ndarray:
    N, K = q["N"], q["K"]
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    out = np.zeros((rows.size, K), np.uint16)
    rc = lib().oracle_dequant_rows(_ptr(q["packed"]), _ptr(q["codes"]), _ptr(q["scale"]), _ptr(q["mean"]),
                                   N, K, _ptr(rows), rows.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequant_rows rejected its arguments")
    return out


# --------------------------------------------------------------------------
# quant types: NF4 (the default) and the FP4 (E2M1) variant
# --------------------------------------------------------------------------
QUANT_NF4 = 0
QUANT_FP4 = 1


def codebook_qt(qt: int) -> np.ndarray:
    """The nibble-indexed 16-entry fp32 table of a quant type."""
    L = np.zeros(16, np.float32)
    if lib().oracle_codebook(int(qt), _ptr(L)) == 0:
        raise ValueError(f"unknown quant type {qt}")
    return L


def fp4_codebook():
    """The FP4 (E2M1 / 6) table: (fp64 before rounding, fp32 as used)."""
    v64 = np.zeros(16, np.float64)
    v32 = np.zeros(16, np.float32)
    lib().oracle_fp4_codebook(_ptr(v64), _ptr(v32))
    return v64, v32


def encode_value_qt(qt: int, x: float) -> int:
    return int(lib().oracle_encode_value_qt(int(qt), ctypes.c_float(float(x))))


def quantize_dq_qt(W_bits: np.ndarray, qt: int):
    """quantize_dq for any quant type (NF4 or FP4)."""
    W_bits = np.ascontiguousarray(W_bits, np.uint16)
    N, K = W_bits.shape
    nblocks = N * K // NF4_BLOCK
    G = (nblocks + DQ_GROUP - 1) // DQ_GROUP
    packed = np.zeros((N, K // 2), np.uint8)
    codes = np.zeros(nblocks, np.int8)
    scale = np.zeros(G, np.float32)
    mean = np.zeros(G, np.float32)
    absmax = np.zeros(nblocks, np.float32)
    rc = lib().oracle_quantize_dq_qt(int(qt), _ptr(W_bits), N, K, _ptr(packed), _ptr(codes), _ptr(scale),
                                     _ptr(mean), _ptr(absmax))
    if rc != 0:
        raise ValueError(f"oracle_quantize_dq_qt rejected its arguments ({rc})")
    return dict(packed=packed, codes=codes, scale=scale, mean=mean, absmax=absmax, N=N, K=K, qt=int(qt))


def dequant_qt(q: dict, rows=None) -> np.ndarray:
    """bf16 W' (raw bits) of a quantized weight of any quant type, all rows or the listed ones."""
    N, K = q["N"], q["K"]
    qt = q.get("qt", QUANT_NF4)
    if rows is None:
        out = np.zeros((N, K), np.uint16)
        rc = lib().oracle_dequant_qt(qt, _ptr(q["packed"]), _ptr(q["codes"]), _ptr(q["scale"]), _ptr(q["mean"]),
                                     N, K, None, 0, _ptr(out))
    else:
        rows = np.ascontiguousarray(np.asarray(rows, np.int64))
        out = np.zeros((rows.size, K), np.uint16)
        rc = lib().oracle_dequant_qt(qt, _ptr(q["packed"]), _ptr(q["codes"]), _ptr(q["scale"]), _ptr(q["mean"]),
                                     N, K, _ptr(rows), rows.size, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_dequant_qt rejected its arguments ({rc})")
    return out


def dequant_merge(q: dict, A_bits: np.ndarray, B_bits: np.ndarray, s: float, rows=None) -> np.ndarray:
    """Dequantize-and-merge: bf16 bits of W' + s B A, one fma per LoRA term in fp32
    (see oracle_dequant_merge), for all rows or the listed ones."""
    N, K = q["N"], q["K"]
    A_bits = np.ascontiguousarray(A_bits, np.uint16)
    B_bits = np.ascontiguousarray(B_bits, np.uint16)
    r = A_bits.shape[0]
    assert A_bits.shape == (r, K) and B_bits.shape == (N, r)
    qt = q.get("qt", QUANT_NF4)
    if rows is None:
        out = np.zeros((N, K), np.uint16)
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, np.int64))
        out = np.zeros((rows.size, K), np.uint16)
        rp, nr = _ptr(rows), rows.size
    rc = lib().oracle_dequant_merge(qt, _ptr(q["packed"]), _ptr(q["codes"]), _ptr(q["scale"]), _ptr(q["mean"]),
                                    N, K, _ptr(A_bits), _ptr(B_bits), r, ctypes.c_float(s), rp, nr, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_dequant_merge rejected its arguments ({rc})")
    return out


# --------------------------------------------------------------------------
# 8-bit AdamW step of the adapters (E4M3 states, blocks of 256)
# --------------------------------------------------------------------------
ADAM_BLOCK = 256


def e4m3_to_f32(code: int) -> float:
    return float(lib().oracle_e4m3_to_f32(ctypes.c_uint8(int(code))))


def f32_to_e4m3(x: float) -> int:
    return int(lib().oracle_f32_to_e4m3(ctypes.c_float(float(x))))


def adamw8_state(n: int):
    """Zero 8-bit moment states for n parameters: (m_code, m_scale, v_code, v_scale)."""
    nb = (n + ADAM_BLOCK - 1) // ADAM_BLOCK
    return (np.zeros(n, np.uint8), np.zeros(nb, np.float32), np.zeros(n, np.uint8), np.zeros(nb, np.float32))


def adamw8_step(p_bits: np.ndarray, g_bits: np.ndarray, state, step: int, lr: float, b1: float, b2: float,
                eps: float, wd: float):
    """One AdamW step in place: p_bits (bf16 bits, updated), state (updated)."""
    m_code, m_scale, v_code, v_scale = state
    for a in (p_bits, g_bits, m_code, m_scale, v_code, v_scale):
        assert a.flags["C_CONTIGUOUS"]
    n = p_bits.size
    assert g_bits.size == n and m_code.size == n and v_code.size == n
    rc = lib().oracle_adamw8_step(_ptr(p_bits), _ptr(g_bits), n, _ptr(m_code), _ptr(m_scale), _ptr(v_code),
                                  _ptr(v_scale), int(step), ctypes.c_float(lr), ctypes.c_float(b1),
                                  ctypes.c_float(b2), ctypes.c_float(eps), ctypes.c_float(wd))
    if rc != 0:
        raise ValueError(f"oracle_adamw8_step rejected its arguments ({rc})")


# --------------------------------------------------------------------------
# LoRA dropout: Philox4x64-10 keep mask of the LoRA branch's input
# --------------------------------------------------------------------------
def philox4x64(counter, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(counter, np.uint64))
    k = np.ascontiguousarray(np.asarray(key, np.uint64))
    out = np.zeros(4, np.uint64)
    lib().oracle_philox4x64(_ptr(c), _ptr(k), _ptr(out))
    return out


def dropout_mask(seed: int, offset: int, M: int, K: int, p: float) -> np.ndarray:
    """Keep mask [M, K] (bool) of the LoRA dropout with rate p."""
    keep = np.zeros((M, K), np.uint8)
    rc = lib().oracle_dropout_mask(ctypes.c_uint64(seed), ctypes.c_uint64(offset), M, K, ctypes.c_float(p),
                                   _ptr(keep))
    if rc != 0:
        raise ValueError("oracle_dropout_mask rejected its arguments")
    return keep.astype(bool)


def dropout_scale(p: float) -> float:
    """The scale of kept values, fl32(1 / (1 - p)) for the fp32 rate p."""
    return float(np.float32(1.0 / (1.0 - float(np.float32(p)))))


# --------------------------------------------------------------------------
# linear layer forward / backward, fp64 definitions
# --------------------------------------------------------------------------
def lora_scaling(r: int, alpha: float) -> float:
    """LoRA scaling alpha / r ("Step 4: Apply LoRA Adapters": r=64, alpha=16 -> 0.25)."""
    return float(alpha) / float(r)


def linear_fwd(X, Wd, A, B, s):
    """Y = X W'^T + s (X A^T) B^T and T = X A^T, all fp64.

    X [M, K], Wd = W' [N, K] (already dequantized), A [r, K], B [N, r].
    """
    X = np.asarray(X, np.float64)
    T = X @ np.asarray(A, np.float64).T
    Y = X @ np.asarray(Wd, np.float64).T + s * (T @ np.asarray(B, np.float64).T)
    return Y, T


def linear_bwd(X, dY, Wd, A, B, s):
    """Gradients of <Y, dY> for the layer above; the frozen W' gets none.

    U = dY B, dX = dY W' + s U A, dA = s U^T X, dB = s dY^T T with T = X A^T.
    """
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    T = X @ A.T
    U = dY @ B
    dX = dY @ np.asarray(Wd, np.float64) + s * (U @ A)
    dA = s * (U.T @ X)
    dB = s * (dY.T @ T)
    return dX, dA, dB


def linear_bwd_adapters(X, dY, A, B, s):
    """The adapter gradients alone (dA, dB) of linear_bwd, without dX."""
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    T = X @ np.asarray(A, np.float64).T
    U = dY @ np.asarray(B, np.float64)
    return s * (U.T @ X), s * (dY.T @ T)


def linear_fwd_dropout(X, Wd, A, B, s, keep, c):
    """Forward with LoRA dropout on the branch input: Y = X W'^T + s (Xd A^T) B^T,
    Xd = X * keep * c (keep the mask, c the scale of kept values); returns (Y, T)."""
    X = np.asarray(X, np.float64)
    Xd = X * np.asarray(keep, np.float64) * c
    T = Xd @ np.asarray(A, np.float64).T
    Y = X @ np.asarray(Wd, np.float64).T + s * (T @ np.asarray(B, np.float64).T)
    return Y, T


def linear_bwd_dropout(X, dY, Wd, A, B, s, keep, c):
    """Gradients of <Y, dY> for linear_fwd_dropout with the mask held fixed:
    U = dY B, dX = dY W' + s (U A) * keep * c, dA = s U^T Xd, dB = s dY^T T."""
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    km = np.asarray(keep, np.float64) * c
    Xd = X * km
    T = Xd @ A.T
    U = dY @ B
    dX = dY @ np.asarray(Wd, np.float64) + s * (U @ A) * km
    dA = s * (U.T @ Xd)
    dB = s * (dY.T @ T)
    return dX, dA, dB

