"""Thin ctypes binding of libqlora_nf4.so (argument marshalling only).

Every function has the name of the C entry point it calls (see
``include/qlora_nf4.h``) and takes torch tensors for the device buffers, whose
pointers and the current CUDA stream are passed through unchanged.  All
computation happens in the library's CUDA kernels; if the library cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_NULL = -1
QLORA_ERR_TIMEOUT = -8
QLORA_ERR_VALUE = -9

_lib = None


class QLoRAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


QLORA_QUANT_NF4 = 0
QLORA_QUANT_FP4 = 1


class _Weight(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("quant_type", ctypes.c_int32)]


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libqlora_nf4.so not found at {LIB_PATH}; run "
                               "`python -m bit_nf4_quantized_quant_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        u64 = ctypes.c_uint64
        WP = ctypes.POINTER(_Weight)
        sig = {
            "nf4_codebook": (i32, [P]),
            "quant4_codebook": (i32, [i32, P]),
            "quant4_quantize_dq": (i32, [P, i64, i64, i32, P, P, P, P, P]),
            "nf4_dequant_merge": (i32, [WP, P, P, i32, f32, P, P]),
            "adamw_8bit_step": (i32, [P, P, i64, P, P, P, P, i64, f32, f32, f32, f32, f32, P]),
            "qlora_dropout_workspace_bytes": (ctypes.c_size_t, [i64, i64, i64, i32]),
            "qlora_linear_fwd_dropout": (i32, [P, i64, WP, P, P, i32, f32, f32, u64, u64, P, P, P,
                                               ctypes.c_size_t, P]),
            "qlora_linear_bwd_dropout": (i32, [P, P, i64, WP, P, P, i32, f32, f32, u64, u64, P, P, P, P, P,
                                               ctypes.c_size_t, P]),
            "nf4dq_sizes": (i32, [i64, i64, P, P, P]),
            "nf4_quantize_dq": (i32, [P, i64, i64, P, P, P, P, P]),
            "nf4_dequant": (i32, [WP, P, P]),
            "qlora_workspace_bytes": (ctypes.c_size_t, [i64, i64, i64, i32]),
            "qlora_linear_fwd": (i32, [P, i64, WP, P, P, i32, f32, P, P, P, ctypes.c_size_t, P]),
            "qlora_linear_bwd": (i32, [P, P, i64, WP, P, P, i32, f32, P, P, P, P, P, ctypes.c_size_t, P]),
            "qlora_status_string": (ctypes.c_char_p, [i32]),
            "qlora_device_status": (i32, [i32]),
            "qlora_last_path": (i32, []),
            "qlora_pair_schedule": (i32, [i64, i64, i32, i32, P, P, P]),
            "qlora_pair_spans": (i32, [i64, i32, i32, i32, P, i32]),
            "qlora_launch_count": (ctypes.c_longlong, []),
            "qlora_set_kernel_events": (i32, [P, P]),
            "qlora_linear_fwd_noalloc": (i32, [P, i64, WP, P, P, i32, f32, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().qlora_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != QLORA_OK:
        raise QLoRAError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bits(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype == torch.bfloat16, t.dtype
    assert t.is_contiguous()
    return t


# --------------------------------------------------------------------------
@dataclass
class NF4Weight:
    """A quantized frozen weight: device tensors plus its logical shape."""
    packed: torch.Tensor   # uint8 [N, K/2]
    codes: torch.Tensor    # int8 [N*K/64]
    scale: torch.Tensor    # fp32 [G]
    mean: torch.Tensor     # fp32 [G]
    N: int
    K: int
    quant_type: int = QLORA_QUANT_NF4

    def c_struct(self) -> _Weight:
        return _Weight(self.packed.data_ptr(), self.codes.data_ptr(), self.scale.data_ptr(),
                       self.mean.data_ptr(), self.N, self.K, self.quant_type)

    @staticmethod
    def empty(N: int, K: int, device="cuda", quant_type: int = QLORA_QUANT_NF4) -> "NF4Weight":
        pb, nb, ng = nf4dq_sizes(N, K)
        return NF4Weight(torch.empty((N, K // 2), dtype=torch.uint8, device=device),
                         torch.empty(nb, dtype=torch.int8, device=device),
                         torch.empty(ng, dtype=torch.float32, device=device),
                         torch.empty(ng, dtype=torch.float32, device=device), N, K, quant_type)


def nf4_codebook() -> list:
    out = (ctypes.c_float * 16)()
    _check("nf4_codebook", lib().nf4_codebook(out))
    return list(out)


def quant4_codebook(quant_type: int) -> list:
    out = (ctypes.c_float * 16)()
    _check("quant4_codebook", lib().quant4_codebook(int(quant_type), out))
    return list(out)


def nf4dq_sizes(N: int, K: int):
    pb, nb, ng = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check("nf4dq_sizes", lib().nf4dq_sizes(N, K, ctypes.byref(pb), ctypes.byref(nb), ctypes.byref(ng)))
    return pb.value, nb.value, ng.value


def nf4_quantize_dq(W: torch.Tensor, out: NF4Weight | None = None, stream=None) -> NF4Weight:
    """bf16 W [N, K] (device) -> NF4Weight."""
    W = _bits(W)
    N, K = W.shape
    if out is None:
        out = NF4Weight.empty(N, K, W.device)
    _check("nf4_quantize_dq", lib().nf4_quantize_dq(_ptr(W), N, K, _ptr(out.packed), _ptr(out.codes),
                                                    _ptr(out.scale), _ptr(out.mean), _stream(stream)))
    return out


def quant4_quantize_dq(W: torch.Tensor, quant_type: int, out: NF4Weight | None = None, stream=None) -> NF4Weight:
    """bf16 W [N, K] (device) -> NF4Weight of the given quant type (NF4 or FP4)."""
    W = _bits(W)
    N, K = W.shape
    if out is None:
        out = NF4Weight.empty(N, K, W.device, quant_type)
    out.quant_type = int(quant_type)
    _check("quant4_quantize_dq", lib().quant4_quantize_dq(_ptr(W), N, K, int(quant_type), _ptr(out.packed),
                                                          _ptr(out.codes), _ptr(out.scale), _ptr(out.mean),
                                                          _stream(stream)))
    return out


def nf4_dequant_merge(w: NF4Weight, A, B, scaling: float, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Dense bf16 W' + scaling * B A (the merged weight of the adapted layer)."""
    if out is None:
        out = torch.empty((w.N, w.K), dtype=torch.bfloat16, device=w.packed.device)
    st = w.c_struct()
    _check("nf4_dequant_merge", lib().nf4_dequant_merge(ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)),
                                                        A.shape[0], float(scaling), _ptr(out), _stream(stream)))
    return out


QLORA_ADAM_BLOCK = 256


@dataclass
class AdamW8State:
    """8-bit moment states of n parameters (E4M3 codes + one fp32 scale per 256)."""
    m_code: torch.Tensor   # uint8 [n]
    m_scale: torch.Tensor  # fp32 [ceil(n / 256)]
    v_code: torch.Tensor   # uint8 [n]
    v_scale: torch.Tensor  # fp32 [ceil(n / 256)]

    @staticmethod
    def zeros(n: int, device="cuda") -> "AdamW8State":
        nb = (n + QLORA_ADAM_BLOCK - 1) // QLORA_ADAM_BLOCK
        return AdamW8State(torch.zeros(n, dtype=torch.uint8, device=device),
                           torch.zeros(nb, dtype=torch.float32, device=device),
                           torch.zeros(n, dtype=torch.uint8, device=device),
                           torch.zeros(nb, dtype=torch.float32, device=device))


def adamw_8bit_step(p: torch.Tensor, g: torch.Tensor, state: AdamW8State, step: int, lr: float,
                    beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                    stream=None) -> None:
    """In-place AdamW step of the bf16 parameters p with gradient g and 8-bit states."""
    p, g = _bits(p), _bits(g)
    _check("adamw_8bit_step", lib().adamw_8bit_step(
        _ptr(p), _ptr(g), p.numel(), _ptr(state.m_code), _ptr(state.m_scale), _ptr(state.v_code),
        _ptr(state.v_scale), int(step), float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
        _stream(stream)))


def nf4_dequant(w: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((w.N, w.K), dtype=torch.bfloat16, device=w.packed.device)
    st = w.c_struct()
    _check("nf4_dequant", lib().nf4_dequant(ctypes.byref(st), _ptr(out), _stream(stream)))
    return out


def qlora_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes(M, N, K, r))


def workspace(M: int, N: int, K: int, r: int, device="cuda") -> torch.Tensor:
    n = qlora_workspace_bytes(M, N, K, r)
    if n == 0:
        raise QLoRAError("qlora_workspace_bytes", -2)
    return torch.empty(n, dtype=torch.uint8, device=device)


def qlora_linear_fwd(X, w: NF4Weight, A, B, scaling: float, Y=None, T_out=None, ws=None, stream=None):
    """Y = X W'^T + s (X A^T) B^T; returns Y (and fills T_out when given)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = workspace(M, w.N, w.K, A.shape[0], X.device)
    st = w.c_struct()
    _check("qlora_linear_fwd", lib().qlora_linear_fwd(
        _ptr(_bits(X)), M, ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)), A.shape[0], float(scaling),
        _ptr(Y), _ptr(T_out), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def qlora_linear_bwd(X, dY, w: NF4Weight, A, B, scaling: float, T=None, dX=None, dA=None, dB=None, ws=None,
                     stream=None):
    """Returns (dX, dA, dB); the frozen weight gets no gradient."""
    M = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if dX is None:
        dX = torch.empty((M, w.K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, w.K), dtype=torch.bfloat16, device=dev)
    if dB is None:
        dB = torch.empty((w.N, r), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = workspace(M, w.N, w.K, r, dev)
    st = w.c_struct()
    _check("qlora_linear_bwd", lib().qlora_linear_bwd(
        _ptr(_bits(X)), _ptr(_bits(dY)), M, ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)), r, float(scaling),
        _ptr(T), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream(stream)))
    return dX, dA, dB


def qlora_dropout_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_dropout_workspace_bytes(M, N, K, r))


def dropout_workspace(M: int, N: int, K: int, r: int, device="cuda") -> torch.Tensor:
    n = qlora_dropout_workspace_bytes(M, N, K, r)
    if n == 0:
        raise QLoRAError("qlora_dropout_workspace_bytes", -2)
    return torch.empty(n, dtype=torch.uint8, device=device)


def qlora_linear_fwd_dropout(X, w: NF4Weight, A, B, scaling: float, dropout_p: float, seed: int, offset: int,
                             Y=None, T_out=None, ws=None, stream=None):
    """qlora_linear_fwd with LoRA dropout on the branch input (mask from (seed, offset))."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = dropout_workspace(M, w.N, w.K, A.shape[0], X.device)
    st = w.c_struct()
    _check("qlora_linear_fwd_dropout", lib().qlora_linear_fwd_dropout(
        _ptr(_bits(X)), M, ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)), A.shape[0], float(scaling),
        float(dropout_p), int(seed), int(offset), _ptr(Y), _ptr(T_out), _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def qlora_linear_bwd_dropout(X, dY, w: NF4Weight, A, B, scaling: float, dropout_p: float, seed: int, offset: int,
                             T=None, dX=None, dA=None, dB=None, ws=None, stream=None):
    """qlora_linear_bwd under the same LoRA dropout mask as the forward; returns (dX, dA, dB)."""
    M = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if dX is None:
        dX = torch.empty((M, w.K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, w.K), dtype=torch.bfloat16, device=dev)
    if dB is None:
        dB = torch.empty((w.N, r), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = dropout_workspace(M, w.N, w.K, r, dev)
    st = w.c_struct()
    _check("qlora_linear_bwd_dropout", lib().qlora_linear_bwd_dropout(
        _ptr(_bits(X)), _ptr(_bits(dY)), M, ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)), r, float(scaling),
        float(dropout_p), int(seed), int(offset), _ptr(T), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
        _stream(stream)))
    return dX, dA, dB


def qlora_device_status(reset: bool = True) -> int:
    return int(lib().qlora_device_status(1 if reset else 0))


def qlora_last_path() -> int:
    return int(lib().qlora_last_path())


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_set_kernel_events(before, after) -> None:
    """Record torch.cuda.Event `before`/`after` around the next fused dequant-GEMM launch on this thread."""
    b = ctypes.c_void_p(before.cuda_event) if before is not None else None
    a = ctypes.c_void_p(after.cuda_event) if after is not None else None
    _check("qlora_set_kernel_events", lib().qlora_set_kernel_events(b, a))


def qlora_linear_fwd_noalloc(X, w: NF4Weight, A, B, scaling: float, Y=None, T_out=None, stream=None):
    """qlora_linear_fwd on the library's fixed static scratch (no workspace argument)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    st = w.c_struct()
    _check("qlora_linear_fwd_noalloc", lib().qlora_linear_fwd_noalloc(
        _ptr(_bits(X)), M, ctypes.byref(st), _ptr(_bits(A)), _ptr(_bits(B)), A.shape[0], float(scaling),
        _ptr(Y), _ptr(T_out), _stream(stream)))
    return Y


def pair_schedule(M: int, n_out: int, pairs: int, bwd: bool):
    """(token tiles per weight stage, tile count, stream-K) of the SM-pair kernel."""
    mt, nt, sk = ctypes.c_int(0), ctypes.c_int64(0), ctypes.c_int(0)
    _check("qlora_pair_schedule", lib().qlora_pair_schedule(M, n_out, pairs, int(bwd), ctypes.byref(mt),
                                                            ctypes.byref(nt), ctypes.byref(sk)))
    return mt.value, nt.value, bool(sk.value)


def pair_spans(ntiles: int, nsteps: int, pair: int, npairs: int):
    """The stream-K spans [(tile, first step, end step), ...] of one pair, in the order it takes them."""
    buf = (ctypes.c_int64 * 3 * 64)()
    n = lib().qlora_pair_spans(ntiles, nsteps, pair, npairs, buf, 64)
    if n < 0:
        _check("qlora_pair_spans", n)
    assert n <= 64
    return [(buf[i][0], buf[i][1], buf[i][2]) for i in range(n)]
