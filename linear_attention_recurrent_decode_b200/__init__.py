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

import torch

__all__ = ["kda_decode", "kda_decode_gated_rmsnorm", "kda_decode_ex", "HostStep", "HostPipeline", "MappedStep",
           "host_memory_is_mapped", "device_error", "kda_prefill",
           "prefill_workspace_bytes", "KdaError", "library", "status_string",
           "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_ALIAS",
           "KDA_ERR_MISALIGNED", "KDA_ERR_DEVICE", "KDA_ERR_CUDA", "KDA_ERR_SCRATCH_LIMIT", "KDA_STATE_FP32",
           "KDA_STATE_BF16",
           "KDA_LAYOUT_KV", "KDA_LAYOUT_VK", "LIBRARY_PATH", "EXPORTED_SYMBOLS"]

LIBRARY_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda_decode.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_ALIAS = 3
KDA_ERR_MISALIGNED = 4
KDA_ERR_DEVICE = 5
KDA_ERR_CUDA = 6
KDA_ERR_SCRATCH_LIMIT = 7

_P, _I, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float


class DecodeArgs(ctypes.Structure):
    """ctypes mirror of ``kda_decode_args`` (include/kda_decode.h)."""
    _fields_ = [
        ("q", _P), ("q_row_stride", _I),
        ("k", _P), ("k_row_stride", _I),
        ("v", _P), ("v_row_stride", _I),
        ("g", _P), ("g_row_stride", _I),
        ("beta", _P), ("beta_row_stride", _I),
        ("raw_gate", _P), ("A_log", _P), ("dt_bias", _P), ("raw_beta", _P),
        ("state_pool", _P), ("state_dtype", ctypes.c_int32), ("state_layout", ctypes.c_int32),
        ("slot_idx", _P),
        ("gate", _P), ("gate_row_stride", _I),
        ("norm_weight", _P),
        ("eps", _F),
        ("out", _P),
        ("N", _I), ("T", _I), ("HV", _I), ("K", _I), ("V", _I),
        ("scale", _F),
        ("num_slots", _I), ("status", _P),
    ]


KDA_STATE_FP32 = 0
KDA_STATE_BF16 = 1
KDA_LAYOUT_KV = 0
KDA_LAYOUT_VK = 1

# Every symbol include/kda_decode.h and include/kda_prefill.h declare, with its ctypes signature.
EXPORTED_SYMBOLS = {
    "kda_decode": ([_P] * 8 + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_gated_rmsnorm": ([_P] * 9 + [_F, _P] + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_bf16_state": ([_P] * 8 + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_gated_rmsnorm_bf16_state": ([_P] * 9 + [_F, _P] + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_decode_ex": ([ctypes.POINTER(DecodeArgs), _P], ctypes.c_int),
    "kda_decode_host": ([ctypes.POINTER(DecodeArgs), _P, _P, _I, _P, _P], ctypes.c_int),
    "kda_decode_host_pipelined": ([ctypes.POINTER(DecodeArgs), _P, _P, _I, _P, _P, _P, _P, _P], ctypes.c_int),
    "kda_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "kda_host_memory_is_mapped": ([_P, _I], ctypes.c_int32),
    "kda_abi_version": ([], ctypes.c_int32),
    "kda_decode_device_error": ([_P, ctypes.c_int32], ctypes.c_int),
    # include/kda_prefill.h
    "kda_prefill_workspace_bytes": ([_I] * 5, ctypes.c_int64),
    "kda_prefill": ([_P] * 9 + [_I] * 6 + [_F, _P], ctypes.c_int),
    "kda_prefill_no_alloc": ([_P] * 8 + [_I] * 5 + [_F, _P], ctypes.c_int),
    "kda_prefill_stage": ([ctypes.c_int32] + [_P] * 9 + [_I] * 6 + [_F, _P], ctypes.c_int),
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
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
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
    """The raw handle of ``stream`` (default: the current stream), which must
    belong to the current device: the library launches on the current device."""
    if stream is None:
        stream = torch.cuda.current_stream()
    if hasattr(stream, "cuda_stream"):
        if stream.device_index != torch.cuda.current_device():
            raise ValueError(f"stream is on cuda:{stream.device_index}, the current device is "
                             f"cuda:{torch.cuda.current_device()}")
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(t, name, dtype, shape=None, device=None):
    # one combined test on the per-call path; the detailed reason only on failure.
    # ``device`` is the current device index: the library launches there, so a
    # tensor on another GPU would be reached through peer addressing.
    if (not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda or not t.is_contiguous()
            or (shape is not None and t.shape != shape) or (device is not None and t.get_device() != device)):
        _check_failed(t, name, dtype, shape, device)


def _check_failed(t, name, dtype, shape, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if device is not None and t.get_device() != device:
        raise ValueError(f"{name} is on cuda:{t.get_device()}, the current device is cuda:{device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _common(q, k, v, g, beta, state_pool, slot_idx, out):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [N, T, HV, K|V]")
    N, T, HV, K = q.shape
    V = v.shape[-1]
    dev = torch.cuda.current_device() if q.is_cuda else None  # a CPU q is refused by _check
    _check(q, "q", torch.bfloat16, None, dev)
    _check(k, "k", torch.bfloat16, (N, T, HV, K), dev)
    _check(v, "v", torch.bfloat16, (N, T, HV, V), dev)
    _check(g, "g", torch.float32, (N, T, HV, K), dev)
    _check(beta, "beta", torch.float32, (N, T, HV), dev)
    _check(slot_idx, "slot_idx", torch.int32, (N,), dev)
    if state_pool.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"state_pool must be float32 or bfloat16, got {state_pool.dtype}")
    _check(state_pool, "state_pool", state_pool.dtype, None, dev)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (HV, K, V):
        raise ValueError(f"state_pool must be [num_slots, {HV}, {K}, {V}]")
    if out is None:
        out = torch.empty((N, T, HV, V), dtype=torch.bfloat16, device=q.device)
    _check(out, "out", torch.bfloat16, (N, T, HV, V), dev)
    return N, T, HV, K, V, out


def kda_decode(q, k, v, g, beta, state_pool, slot_idx, out=None, scale: float | None = None,
               stream=None):
    """Recurrent KDA decode step on the caller's stream; updates ``state_pool`` in
    place and returns ``out`` (allocated if not given).  ``scale`` defaults to
    1/sqrt(K).  A bf16 ``state_pool`` runs the bf16-state entry point (fp32
    math, state rounded to bf16 once per call)."""
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


def _rows(t, name, dtype, N, T, inner):
    """Validate a [N, T, ...inner] view whose (n, t) rows are uniformly strided and
    whose per-row part is dense; return its row stride in elements (0 for None)."""
    if t is None:
        return 0
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if tuple(t.shape) != (N, T, *inner):
        raise ValueError(f"{name} must have shape {(N, T, *inner)}, got {tuple(t.shape)}")
    want = 1
    for d in range(t.dim() - 1, 1, -1):  # the per-row part must be dense
        if t.shape[d] > 1 and t.stride(d) != want:
            raise ValueError(f"{name}: each (n, t) row must be contiguous")
        want *= t.shape[d]
    rs = t.stride(1) if T > 1 else t.stride(0)
    if N > 1 and T > 1 and t.stride(0) != T * t.stride(1):
        raise ValueError(f"{name}: (n, t) rows must be evenly strided (stride(0) == T * stride(1))")
    return rs if (N * T) > 1 else max(rs, want)


def _ex_args(q, k, v, state_pool, slot_idx, *, g=None, beta=None, raw_gate=None, A_log=None,
                  dt_bias=None, raw_beta=None, gate=None, norm_weight=None, eps: float = 1e-6, out=None,
                  scale: float | None = None, state_layout: str = "kv", num_slots: int | None = None,
                  status=None):
    """The kda_decode_args of a call (and its output tensor); see kda_decode_ex."""
    N, T, HV, K = q.shape
    V = v.shape[-1]
    bf, f32 = torch.bfloat16, torch.float32
    dev = torch.cuda.current_device() if q.is_cuda else -1  # CPU tensors are refused below
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("raw_gate", raw_gate),
                    ("A_log", A_log), ("dt_bias", dt_bias), ("raw_beta", raw_beta), ("state_pool", state_pool),
                    ("slot_idx", slot_idx), ("gate", gate), ("norm_weight", norm_weight), ("out", out),
                    ("status", status)):
        if isinstance(t, torch.Tensor) and t.is_cuda and t.get_device() != dev:
            raise ValueError(f"{name} is on cuda:{t.get_device()}, the current device is cuda:{dev}")
    a = DecodeArgs()
    a.q, a.q_row_stride = q.data_ptr(), _rows(q, "q", bf, N, T, (HV, K))
    a.k, a.k_row_stride = k.data_ptr(), _rows(k, "k", bf, N, T, (HV, K))
    a.v, a.v_row_stride = v.data_ptr(), _rows(v, "v", bf, N, T, (HV, V))
    if raw_gate is not None:
        a.raw_gate, a.g_row_stride = raw_gate.data_ptr(), _rows(raw_gate, "raw_gate", bf, N, T, (HV, K))
        a.raw_beta, a.beta_row_stride = raw_beta.data_ptr(), _rows(raw_beta, "raw_beta", bf, N, T, (HV,))
        _check(A_log, "A_log", f32, (HV,))
        _check(dt_bias, "dt_bias", f32, (HV, K))
        a.A_log, a.dt_bias = A_log.data_ptr(), dt_bias.data_ptr()
    else:
        a.g, a.g_row_stride = g.data_ptr(), _rows(g, "g", f32, N, T, (HV, K))
        a.beta, a.beta_row_stride = beta.data_ptr(), _rows(beta, "beta", f32, N, T, (HV,))
    if state_pool.dtype not in (f32, bf):
        raise TypeError("state_pool must be float32 or bfloat16")
    _check(state_pool, "state_pool", state_pool.dtype)
    if state_layout not in ("kv", "vk"):
        raise ValueError("state_layout must be 'kv' or 'vk'")
    block = (K, V) if state_layout == "kv" else (V, K)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (HV, *block):
        raise ValueError(f"state_pool must be [num_slots, {HV}, {block[0]}, {block[1]}]")
    a.state_pool = state_pool.data_ptr()
    a.state_layout = KDA_LAYOUT_KV if state_layout == "kv" else KDA_LAYOUT_VK
    a.state_dtype = KDA_STATE_BF16 if state_pool.dtype == bf else KDA_STATE_FP32
    _check(slot_idx, "slot_idx", torch.int32, (N,))
    a.slot_idx = slot_idx.data_ptr()
    if gate is not None:
        a.gate, a.gate_row_stride = gate.data_ptr(), _rows(gate, "gate", bf, N, T, (HV, V))
        _check(norm_weight, "norm_weight", bf, (V,))
        a.norm_weight = norm_weight.data_ptr()
    a.eps = float(eps)
    if out is None:
        out = torch.empty((N, T, HV, V), dtype=bf, device=q.device)
    _check(out, "out", bf, (N, T, HV, V))
    a.out = out.data_ptr()
    a.N, a.T, a.HV, a.K, a.V = N, T, HV, K, V
    a.scale = float(1.0 / math.sqrt(K) if scale is None else scale)
    a.num_slots = int(state_pool.shape[0] if num_slots is None else num_slots)
    if a.num_slots < 0 or a.num_slots > state_pool.shape[0]:
        raise ValueError(f"num_slots must be in [0, {state_pool.shape[0]}] (0 = unchecked)")
    if status is not None:
        _check(status, "status", torch.int32, None, dev)
        if status.numel() < 1:
            raise ValueError("status must hold at least one int32")
        a.status = status.data_ptr()
    return a, out


def kda_decode_ex(q, k, v, state_pool, slot_idx, *, g=None, beta=None, raw_gate=None, A_log=None,
                  dt_bias=None, raw_beta=None, gate=None, norm_weight=None, eps: float = 1e-6, out=None,
                  scale: float | None = None, stream=None, state_layout: str = "kv",
                  num_slots: int | None = None, status=None):
    """General decode step (``kda_decode_ex`` of the C ABI).

    q, k [N,T,HV,K], v [N,T,HV,V] (bf16) may be strided views, e.g. slices of
    one packed ``mixed_qkv`` row buffer; so may g / raw_gate [N,T,HV,K] and
    beta / raw_beta [N,T,HV] and gate [N,T,HV,V].  Give either ``g`` and
    ``beta`` (fp32) or the serving form ``raw_gate``, ``A_log`` [HV],
    ``dt_bias`` [HV,K] (fp32) and ``raw_beta`` (bf16).  ``gate`` with
    ``norm_weight`` selects the fused gated RMS norm.  The pool may be fp32 or
    bf16, with blocks [K, V] (``state_layout="kv"``: pool [num_slots,HV,K,V])
    or [V, K] (``"vk"``: pool [num_slots,HV,V,K], key index fastest).

    Slots are checked against ``num_slots`` (default: the pool's first
    dimension; 0 = unchecked): an active row naming a slot at or beyond it gets
    a zero output, leaves the pool untouched and, when ``status`` (a device
    int32 tensor the caller zeroes) is given, sets ``status[0]`` to 1.
    Returns ``out`` (dense bf16 [N,T,HV,V])."""
    a, out = _ex_args(q, k, v, state_pool, slot_idx, g=g, beta=beta, raw_gate=raw_gate, A_log=A_log,
                      dt_bias=dt_bias, raw_beta=raw_beta, gate=gate, norm_weight=norm_weight, eps=eps, out=out,
                      scale=scale, state_layout=state_layout, num_slots=num_slots, status=status)
    st = library().kda_decode_ex(ctypes.byref(a), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_ex")
    return out


class HostStep:
    """One decode step run from host memory (``kda_decode_host`` of the C ABI),
    bound once and run many times, as a serving loop with static buffers does.

    ``host_in`` (pinned uint8) is copied to ``dev_in`` (device uint8) each
    call; the tensors given for the step's inputs must be views into
    ``dev_in``.  The output goes to ``out`` on the device and is copied to
    ``host_out`` (pinned, same shape and dtype).  Keyword arguments are those of
    :func:`kda_decode_ex`.  Calling the object enqueues the copy in, the step
    and the copy out on ``stream``: one call into the library per step.
    """

    def __init__(self, q, k, v, state_pool, slot_idx, *, host_in, dev_in, host_out, out, stream=None, **kw):

        for name, t in (("host_in", host_in), ("host_out", host_out)):
            if t.is_cuda or not t.is_pinned():
                raise ValueError(f"{name} must be pinned host memory")
        if not dev_in.is_cuda or not dev_in.is_contiguous() or not host_in.is_contiguous():
            raise ValueError("dev_in must be a contiguous device tensor, host_in contiguous")
        nbytes = host_in.numel() * host_in.element_size()
        if dev_in.numel() * dev_in.element_size() < nbytes:
            raise ValueError("dev_in is smaller than host_in")
        if host_out.shape != out.shape or host_out.dtype != out.dtype or not host_out.is_contiguous():
            raise ValueError("host_out must match out")
        lo, hi = dev_in.data_ptr(), dev_in.data_ptr() + nbytes
        for name, t in (("q", q), ("k", k), ("v", v), ("slot_idx", slot_idx)):
            if not lo <= t.data_ptr() < hi:
                raise ValueError(f"{name} must be a view into dev_in")
        self.args, self.out = _ex_args(q, k, v, state_pool, slot_idx, out=out, **kw)
        self._keep = (q, k, v, state_pool, slot_idx, host_in, dev_in, host_out, out, kw)
        self._ptrs = (host_in.data_ptr(), dev_in.data_ptr(), nbytes, host_out.data_ptr())
        self._torch_stream = stream if stream is not None else torch.cuda.current_stream()
        self._stream = _stream_handle(self._torch_stream)
        self._fn = library().kda_decode_host
        self._ref = ctypes.byref(self.args)

    def __call__(self):
        st = self._fn(self._ref, *self._ptrs, self._stream)
        if st != KDA_OK:
            raise KdaError(st, "kda_decode_host")


class HostPipeline:
    """Steps run from host memory with each step's copy in overlapping the
    previous step's kernel and copy out (``kda_decode_host_pipelined`` of the C
    ABI).

    ``steps`` are :class:`HostStep` objects bound to the same ``stream`` and
    state pool, each with its own staging buffers (``host_in``, ``dev_in``,
    ``host_out``); calling the pipeline runs the next one in turn, its copy in
    enqueued on ``copy_stream``.  Two staging sets let step i+1's inputs travel
    while step i computes; the events that order a set's reuse are made here,
    once.  A step's output is in its ``host_out`` once ``stream`` has passed it.
    """

    def __init__(self, steps, copy_stream):
        if len(steps) < 1 or len({id(s._torch_stream) for s in steps}) != 1:
            raise ValueError("steps must share one stream")
        self._steps = list(steps)
        self._copy = copy_stream
        self._copy_handle = _stream_handle(copy_stream)
        stream = steps[0]._torch_stream
        if copy_stream.cuda_stream == stream.cuda_stream:
            raise ValueError("copy_stream must differ from the steps' stream")
        self._events = []
        for _ in self._steps:  # torch creates an event's handle on its first record
            ready, free = torch.cuda.Event(), torch.cuda.Event()
            ready.record(copy_stream)
            free.record(stream)
            self._events.append((ready, free))
        torch.cuda.synchronize()
        self._handles = [(ctypes.c_void_p(r.cuda_event), ctypes.c_void_p(f.cuda_event)) for r, f in self._events]
        self._fn = library().kda_decode_host_pipelined
        self._next = 0

    def rearm(self):
        """Record every staging set's "free" event on the steps' stream now, so
        that the next wait on it refers to this point.  Call it first when
        capturing steps into a CUDA graph (inside the capture, after forking the
        copy stream from the steps' stream): a captured wait must refer to a
        record made inside the same capture."""
        stream = self._steps[0]._torch_stream
        for _, free in self._events:
            free.record(stream)

    def __call__(self):
        i = self._next
        st = self._steps[i]
        rc = self._fn(st._ref, *st._ptrs, st._stream, self._copy_handle, *self._handles[i])
        if rc != KDA_OK:
            raise KdaError(rc, "kda_decode_host_pipelined")
        self._next = (i + 1) % len(self._steps)
        return st


def device_error(clear: bool = False) -> int:
    """The decode kernels' device-side error word on the current device (1 if a
    kernel gave up a bounded wait since the last clear, else 0); ``clear``
    resets it.  Waits for the device's work in flight."""
    word = ctypes.c_int32(0)
    status = library().kda_decode_device_error(ctypes.byref(word), 1 if clear else 0)
    if status != KDA_OK:
        raise KdaError(status, "kda_decode_device_error")
    return int(word.value)


def host_memory_is_mapped(t) -> bool:
    """Whether the current device reads and writes the page-locked host tensor
    ``t`` at its host address (``kda_host_memory_is_mapped`` of the C ABI)."""
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
        return False
    return bool(library().kda_host_memory_is_mapped(t.data_ptr(), t.numel() * t.element_size()))


class MappedStep:
    """One decode step read from and written to page-locked host memory directly:
    ``kda_decode_ex`` given host pointers the device reaches at the same address
    (checked once, here, with :func:`host_memory_is_mapped`).  The kernel reads
    the step's inputs across PCIe and writes ``out`` back to host memory in its
    one launch, so a step costs no separate copies and no stream dependencies.

    ``host_in`` is the pinned buffer the input tensors are views of; ``out`` a
    pinned bf16 [N, T, HV, V] tensor; the state pool stays on the device.
    Keyword arguments are those of :func:`kda_decode_ex` (g/beta or the raw
    form, gate, norm_weight, eps, scale, state_layout, num_slots, status)."""

    def __init__(self, q, k, v, state_pool, slot_idx, *, host_in, out, stream=None, **kw):
        for name, t in (("host_in", host_in), ("out", out)):
            if not host_memory_is_mapped(t):
                raise ValueError(f"{name} is not page-locked host memory the current device maps at its address")
        lo, hi = host_in.data_ptr(), host_in.data_ptr() + host_in.numel() * host_in.element_size()
        views = {"q": q, "k": k, "v": v, "slot_idx": slot_idx,
                 **{key: t for key, t in kw.items() if isinstance(t, torch.Tensor) and not t.is_cuda}}
        for name, t in views.items():
            if not (lo <= t.data_ptr() and t.data_ptr() + t.numel() * t.element_size() <= hi):
                raise ValueError(f"{name} must be a view into host_in")
        if out.dtype != torch.bfloat16 or not out.is_contiguous():
            raise ValueError("out must be a contiguous bf16 tensor")
        if not state_pool.is_cuda:
            raise ValueError("state_pool must be on the device")
        self.args = _mapped_args(q, k, v, state_pool, slot_idx, out, kw)
        self._keep = (q, k, v, state_pool, slot_idx, host_in, out, kw)
        self._torch_stream = stream if stream is not None else torch.cuda.current_stream()
        self._stream = _stream_handle(self._torch_stream)
        self._fn = library().kda_decode_ex
        self._ref = ctypes.byref(self.args)
        self.out = out

    def __call__(self):
        st = self._fn(self._ref, self._stream)
        if st != KDA_OK:
            raise KdaError(st, "kda_decode_ex")


def _mapped_args(q, k, v, state_pool, slot_idx, out, kw):
    """kda_decode_args for host-resident (mapped) inputs and output: the same
    marshalling as _ex_args, with the device checks applied to the pool only."""
    N, T, HV, K = q.shape
    V = v.shape[-1]
    a = DecodeArgs()
    bf, f32 = torch.bfloat16, torch.float32

    def rows(t, name, dtype, inner):
        if t is None:
            return 0
        if t.dtype != dtype or tuple(t.shape) != (N, T, *inner):
            raise ValueError(f"{name} must be {dtype} {(N, T, *inner)}")
        return t.stride(1) if T > 1 else t.stride(0)

    a.q, a.q_row_stride = q.data_ptr(), rows(q, "q", bf, (HV, K))
    a.k, a.k_row_stride = k.data_ptr(), rows(k, "k", bf, (HV, K))
    a.v, a.v_row_stride = v.data_ptr(), rows(v, "v", bf, (HV, V))
    if kw.get("raw_gate") is not None:
        a.raw_gate, a.g_row_stride = kw["raw_gate"].data_ptr(), rows(kw["raw_gate"], "raw_gate", bf, (HV, K))
        a.raw_beta, a.beta_row_stride = kw["raw_beta"].data_ptr(), rows(kw["raw_beta"], "raw_beta", bf, (HV,))
        a.A_log, a.dt_bias = kw["A_log"].data_ptr(), kw["dt_bias"].data_ptr()
    else:
        a.g, a.g_row_stride = kw["g"].data_ptr(), rows(kw["g"], "g", f32, (HV, K))
        a.beta, a.beta_row_stride = kw["beta"].data_ptr(), rows(kw["beta"], "beta", f32, (HV,))
    layout = kw.get("state_layout", "kv")
    a.state_pool = state_pool.data_ptr()
    a.state_layout = KDA_LAYOUT_KV if layout == "kv" else KDA_LAYOUT_VK
    a.state_dtype = KDA_STATE_BF16 if state_pool.dtype == bf else KDA_STATE_FP32
    a.slot_idx = slot_idx.data_ptr()
    if kw.get("gate") is not None:
        a.gate, a.gate_row_stride = kw["gate"].data_ptr(), rows(kw["gate"], "gate", bf, (HV, V))
        a.norm_weight = kw["norm_weight"].data_ptr()
    a.eps = float(kw.get("eps", 1e-6))
    if tuple(out.shape) != (N, T, HV, V):
        raise ValueError(f"out must be [{N}, {T}, {HV}, {V}]")
    a.out = out.data_ptr()
    a.N, a.T, a.HV, a.K, a.V = N, T, HV, K, V
    scale = kw.get("scale")
    a.scale = float(1.0 / math.sqrt(K) if scale is None else scale)
    a.num_slots = int(state_pool.shape[0] if kw.get("num_slots") is None else kw["num_slots"])
    return a


# ---------------------------------------------------------------- chunked prefill
def prefill_workspace_bytes(N: int, T: int, HV: int, K: int = 128, V: int = 128) -> int:
    """Device workspace ``kda_prefill`` needs for these sizes (bytes)."""
    n = library().kda_prefill_workspace_bytes(N, T, HV, K, V)
    if n < 0:
        raise ValueError(f"kda_prefill does not support N={N}, T={T}, HV={HV}, K={K}, V={V}")
    return n


def kda_prefill(q, k, v, g, beta, state_pool, slot_idx, out=None, scale: float | None = None, workspace=None,
                stream=None, stage: int | None = None):
    """Chunked prefill (``kda_prefill`` of the C ABI): the decode recurrence over
    all T tokens of each sequence, taken in chunks of 64 tokens; updates
    ``state_pool`` (fp32 [num_slots, HV, K, V]) in place and returns ``out``
    (bf16 [N, T, HV, V]).  ``workspace``: a device uint8 tensor of at least
    :func:`prefill_workspace_bytes` bytes (allocated here if not given).
    ``stage`` 0, 1 or 2 runs only that kernel (``kda_prefill_stage``: chunk
    preparation, state recurrence, chunk outputs; a caller keeps their order
    and passes the same workspace to all three)."""
    N, T, HV, K, V, out = _common(q, k, v, g, beta, state_pool, slot_idx, out)
    if state_pool.dtype != torch.float32:
        raise TypeError("kda_prefill takes an fp32 state pool")
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    need = prefill_workspace_bytes(N, T, HV, K, V)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8, None, torch.cuda.current_device())
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(), state_pool.data_ptr(),
            slot_idx.data_ptr(), out.data_ptr(), workspace.data_ptr(), workspace.numel(), N, T, HV, K, V,
            float(scale), _stream_handle(stream))
    if stage is None:
        st = library().kda_prefill(*args)
    else:
        st = library().kda_prefill_stage(int(stage), *args)
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill" if stage is None else "kda_prefill_stage")
    return out
