"""fp64 CPU oracle of the recurrent KDA decode step (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it and
shares no code with it: the oracle is the plain C loop in ``kda_oracle.c``
(compiled here with gcc), wrapped by ctypes.

What the oracle computes, and which page each step follows, is stated at the
top of ``kda_oracle.c``.  Every function here only marshals arrays; all the
arithmetic of the method lives in the C file.

Parity status of each entry point (what pins it, see ``tests/test_oracle_pins.py``):
  * ``kda_decode_ref``                    -- pinned by closed forms and a hand-worked
                                             K=V=4 case.
  * ``kda_decode_ref`` with ``gate``/``norm_weight`` (gated RMS norm) -- pinned by
                                             closed forms (rank-1 readout, unit
                                             gate limit).
  * ``round_bf16`` (bf16 state write-back) -- pinned by the format's definition
                                             and torch's conversion.
  * ``activate`` (raw gate / raw beta)  -- PARITY UNPINNED by the sources: no page
                                             prints the activation.  The tests pin only
                                             properties every softplus-style gate and
                                             logistic beta has (g <= 0, monotone in the
                                             raw gate, its two limits, the dt_bias shift;
                                             beta in (0,1), increasing, symmetric), not
                                             the formula taken as the reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libkda_oracle.so`` with gcc (IEEE fp64,
    no contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Load an oracle shared object built from ``kda_oracle.c`` (or an edited
    copy of it, as the mutation tests do) and declare its signature."""
    lib = ctypes.CDLL(path)
    f = lib.kda_oracle_decode_units
    P = ctypes.c_void_p
    I = ctypes.c_int64
    D = ctypes.c_double
    f.argtypes = [P, P, P, P, P, P, P, P, I, P, P, I, I, I, I, I, D, D, I, I, P, P]
    f.restype = ctypes.c_int
    r = lib.kda_oracle_round_bf16
    r.argtypes = [P, P, I]
    r.restype = None
    a = lib.kda_oracle_activate
    a.argtypes = [P, P, P, P, P, P, I, I, I]
    a.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _as_bf16_bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 bit pattern array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16, x.dtype
        return np.ascontiguousarray(x)
    import torch  # only for the dtype reinterpretation of a CPU tensor

    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _as_np(x, dtype) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(x, dtype=dtype)


def _is_f64(x) -> bool:
    return str(x.dtype) in ("float64", "torch.float64")


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def round_bf16(x) -> np.ndarray:
    """Doubles rounded to bf16 (nearest, ties to even) by the oracle's own C
    routine; returned as float64 values."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    bits = np.empty(a.shape, dtype=np.uint16)
    _load().kda_oracle_round_bf16(_ptr(a), _ptr(bits), a.size)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def activate(raw_gate, A_log, dt_bias, raw_beta):
    """Gate and beta of the serving input form, in double (see
    ``kda_oracle_activate`` in kda_oracle.c; the formula is a reading, not fixed
    by the sources).  raw_gate bf16 [N,T,HV,K], A_log fp32 [HV], dt_bias fp32
    [HV,K], raw_beta bf16 [N,T,HV] -> (g fp64 [N,T,HV,K], beta fp64 [N,T,HV])."""
    rg = _as_bf16_bits(raw_gate)
    N, T, HV, K = rg.shape
    rb = _as_bf16_bits(raw_beta).reshape(N, T, HV)
    al = _as_np(A_log, np.float32).reshape(HV)
    db = _as_np(dt_bias, np.float32).reshape(HV, K)
    g = np.empty((N, T, HV, K), np.float64)
    beta = np.empty((N, T, HV), np.float64)
    _load().kda_oracle_activate(_ptr(rg), _ptr(al), _ptr(db), _ptr(rb), _ptr(g), _ptr(beta), N * T, HV, K)
    return g, beta


def kda_decode_ref(q, k, v, g, beta, state_pool, slot_idx, scale: float,
                   gate=None, norm_weight=None, eps: float = 1e-6,
                   threads: int = 1, units: tuple[int, int] | None = None,
                   state_inplace: np.ndarray | None = None):
    """Run the oracle on one call.

    q, k: bf16 [N,T,HV,K]; v: bf16 [N,T,HV,V]; g: fp32 or fp64 [N,T,HV,K];
    beta: fp32 or fp64 [N,T,HV]; state_pool: fp32 or fp64 [num_slots,HV,K,V];
    slot_idx: int32 [N] (negative = inactive row); gate: bf16 [N,T,HV,V] and
    norm_weight: bf16 [V] for the gated RMS-norm variant (both or neither).

    Returns ``(out, state)``: ``out`` fp64 [N,T,HV,V] (unrounded) and the updated
    pool in fp64.  ``units=(begin, end)`` restricts the work to units
    ``n*HV + h`` in that range (the rest of ``out`` stays zero); ``threads``
    splits the units over host threads (ctypes releases the GIL).  If
    ``state_inplace`` (an fp64 pool) is given it is updated in place and
    ``state_pool`` is ignored.
    """
    lib = _load()
    qb, kb, vb = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v)
    N, T, HV, K = qb.shape
    V = vb.shape[-1]
    assert kb.shape == (N, T, HV, K) and vb.shape == (N, T, HV, V)
    # g and beta are widened exactly to double (fp32 inputs) or taken as given (fp64)
    gn = _as_np(g, np.float64 if _is_f64(g) else np.float32).astype(np.float64).reshape(N, T, HV, K)
    bn = _as_np(beta, np.float64 if _is_f64(beta) else np.float32).astype(np.float64).reshape(N, T, HV)
    sn = _as_np(slot_idx, np.int32).reshape(N)
    if (gate is None) != (norm_weight is None):
        raise ValueError("gate and norm_weight go together")
    zb = None if gate is None else _as_bf16_bits(gate).reshape(N, T, HV, V)
    wb = None if norm_weight is None else _as_bf16_bits(norm_weight).reshape(V)
    bf16_state = False
    if state_inplace is not None:
        st = state_inplace
        assert st.dtype == np.float64 and st.flags.c_contiguous
    elif isinstance(state_pool, np.ndarray) and state_pool.dtype == np.uint16 or (
            not isinstance(state_pool, np.ndarray) and str(state_pool.dtype) == "torch.bfloat16"):
        bf16_state = True
        st = (_as_bf16_bits(state_pool).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    else:
        st = _as_np(state_pool, np.float64).copy()
    num_slots = st.shape[0]
    assert st.shape == (num_slots, HV, K, V), st.shape
    out = np.zeros((N, T, HV, V), dtype=np.float64)

    total = N * HV
    b0, b1 = (0, total) if units is None else (max(0, units[0]), min(total, units[1]))

    def run(lo, hi):
        rk = np.empty(V, dtype=np.float64)
        u = np.empty(V, dtype=np.float64)
        rc = lib.kda_oracle_decode_units(
            _ptr(qb), _ptr(kb), _ptr(vb), _ptr(gn), _ptr(bn), _ptr(zb), _ptr(wb), _ptr(st),
            num_slots, _ptr(sn), _ptr(out), N, T, HV, K, V, float(scale), float(eps),
            lo, hi, _ptr(rk), _ptr(u))
        if rc != 0:
            raise ValueError("oracle rejected the call (slot index >= num_slots or bad size)")

    threads = max(1, int(threads))
    active = sn[sn >= 0]
    # Units touch disjoint states only when active slots are distinct; with a
    # repeated slot the rows must run in sequence order, so stay on one thread.
    if threads == 1 or b1 - b0 <= 1 or len(np.unique(active)) != len(active):
        run(b0, b1)
    else:
        bounds = sorted(set(int(b) for b in np.linspace(b0, b1, threads + 1)))
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda ab: run(*ab), zip(bounds[:-1], bounds[1:])))
    if bf16_state:
        st = round_bf16(st)
    return out, st
