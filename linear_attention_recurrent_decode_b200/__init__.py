"""B200-native recurrent Kimi Delta Attention (KDA) decode.

Thin Python binding of the C ABI in ``include/kda_decode.h`` (library
``libkda_decode.so``, built in-tree by ``build.py``).  The functions here only
marshal torch tensors into pointers and sizes; every step of the decode runs
in the library's sm_100a kernels.  There is no fallback: if the library is
missing or the device is not sm_100a, the call raises.

    from linear_attention_recurrent_decode_b200 import kda_decode
    out = kda_decode(q, k, v, g, beta, state_pool, slot_idx)       # state updated in place

Tensor layouts (contiguous, on the current CUDA device):
    q, k bf16 [N,T,HV,K]; v bf16 [N,T,HV,V]; g fp32 [N,T,HV,K] (log-decay);
    beta fp32 [N,T,HV]; state_pool fp32 or bf16 [num_slots,HV,K,V]; slot_idx int32 [N]
    (negative = inactive row); out bf16 [N,T,HV,V]; gate bf16 [N,T,HV,V];
    norm_weight bf16 [V].
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = ["kda_decode", "kda_decode_gated_rmsnorm", "KdaError", "library", "status_string",
           "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_ALIAS",
           "KDA_ERR_MISALIGNED", "KDA_ERR_DEVICE", "KDA_ERR_CUDA", "LIBRARY_PATH", "EXPORTED_SYMBOLS"]

LIBRARY_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda_decode.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_ALIAS = 3
KDA_ERR_MISALIGNED = 4
KDA_ERR_DEVICE = 5
KDA_ERR_CUDA = 6

# Every symbol include/kda_decode.h declares, with its ctypes signature.
_P, _I, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
EXPORTED_SYMBOLS = {
    "kda_decode": ([_P] * 8 + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_gated_rmsnorm": ([_P] * 9 + [_F, _P] + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_bf16_state": ([_P] * 8 + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_gated_rmsnorm_bf16_state": ([_P] * 9 + [_F, _P] + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "kda_abi_version": ([], ctypes.c_int32),
}

_lock = threading.Lock()
_lib = None


class KdaError(RuntimeError):
    """A non-zero status from the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {status_string(status)}")


def library() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIBRARY_PATH):
                raise RuntimeError(
                    f"{LIBRARY_PATH} is missing: build it with "
                    "`python -m linear_attention_recurrent_decode_b200.build` (no fallback exists)")
            lib = ctypes.CDLL(LIBRARY_PATH)
            for name, (argtypes, restype) in EXPORTED_SYMBOLS.items():
                fn = getattr(lib, name)
                fn.argtypes = argtypes
                fn.restype = restype
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().kda_status_string(int(status)).decode()


def _stream_handle(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t, name, dtype, shape=None):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _common(q, k, v, g, beta, state_pool, slot_idx, out):
    import torch

    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [N, T, HV, K|V]")
    N, T, HV, K = q.shape
    V = v.shape[-1]
    _check(q, "q", torch.bfloat16)
    _check(k, "k", torch.bfloat16, (N, T, HV, K))
    _check(v, "v", torch.bfloat16, (N, T, HV, V))
    _check(g, "g", torch.float32, (N, T, HV, K))
    _check(beta, "beta", torch.float32, (N, T, HV))
    _check(slot_idx, "slot_idx", torch.int32, (N,))
    if state_pool.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"state_pool must be float32 or bfloat16, got {state_pool.dtype}")
    _check(state_pool, "state_pool", state_pool.dtype)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (HV, K, V):
        raise ValueError(f"state_pool must be [num_slots, {HV}, {K}, {V}]")
    if out is None:
        out = torch.empty((N, T, HV, V), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", torch.bfloat16, (N, T, HV, V))
    return N, T, HV, K, V, out


def kda_decode(q, k, v, g, beta, state_pool, slot_idx, out=None, scale: float | None = None,
               stream=None):
    """Recurrent KDA decode step on the caller's stream; updates ``state_pool`` in
    place and returns ``out`` (allocated if not given).  ``scale`` defaults to
    1/sqrt(K).  A bf16 ``state_pool`` runs the bf16-state entry point (fp32
    math, state rounded to bf16 once per call)."""
    import torch

    N, T, HV, K, V, out = _common(q, k, v, g, beta, state_pool, slot_idx, out)
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    name = "kda_decode_bf16_state" if state_pool.dtype == torch.bfloat16 else "kda_decode"
    st = getattr(library(), name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                                  state_pool.data_ptr(), slot_idx.data_ptr(), out.data_ptr(),
                                  N, T, HV, K, V, float(scale), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, name)
    return out


def kda_decode_gated_rmsnorm(q, k, v, g, beta, state_pool, slot_idx, gate, norm_weight,
                             eps: float = 1e-6, out=None, scale: float | None = None, stream=None):
    """Decode step fused with the gated RMS norm over V:
    out = bf16(o / sqrt(mean(o^2) + eps) * norm_weight * sigmoid(gate))."""
    import torch

    N, T, HV, K, V, out = _common(q, k, v, g, beta, state_pool, slot_idx, out)
    _check(gate, "gate", torch.bfloat16, (N, T, HV, V))
    _check(norm_weight, "norm_weight", torch.bfloat16, (V,))
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    name = ("kda_decode_gated_rmsnorm_bf16_state" if state_pool.dtype == torch.bfloat16
            else "kda_decode_gated_rmsnorm")
    st = getattr(library(), name)(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(), state_pool.data_ptr(),
        slot_idx.data_ptr(), gate.data_ptr(), norm_weight.data_ptr(), float(eps), out.data_ptr(),
        N, T, HV, K, V, float(scale), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, name)
    return out
