"""Seeded synthetic inputs for the KDA decode step.

This module draws random numbers and nothing else: it holds none of the
decode step's arithmetic, so both the CUDA path and the fp64 oracle can take
their inputs from it without sharing any computation.  All tensors are made on
the CPU with ``torch.Generator`` (seeded) and may then be copied to a device.

Input recipe (every configuration, unless stated otherwise):
  * state pool fp32 ``[num_slots, HV, K, V]`` ~ N(0, 0.02^2) (0.02 is the std);
    for a bf16 pool the same draw is rounded to bf16;
  * q, k, v drawn fp32 ~ N(0, 1); q and k are L2-normalised over K per
    (n, t, h) in fp32 and then all three are rounded to bf16;
  * g fp32 ``[N, T, HV, K]`` = -softplus(N(0, 1)) per key channel (log-decay);
  * beta fp32 ``[N, T, HV]`` = sigmoid(N(0, 1));
  * slot_idx int32 ``[N]``: distinct slots drawn by a random permutation;
  * gated variant: gate z bf16 ``[N, T, HV, V]`` ~ N(0, 1), RMS-norm weight
    bf16 ``[V]`` ~ N(1, 0.1^2), eps = 1e-6;
  * scale = 1/sqrt(K).

The shapes follow the serving shapes of the pages: K = V = 128 and 8 local
value heads with N = 32 sequences dominating decode graphs (vLLM #57585,
"Retained baseline trace attribution"), T = 4 for speculative decode
(vLLM #57585, "Microbenchmark and earlier serving limits"), a gated RMS norm
after the decode kernel (b12x #249, sequence diagram).  No public dataset is
involved; these draws stand in for the activations of a KDA layer.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass
class Workload:
    name: str
    N: int
    T: int
    HV: int
    K: int
    V: int
    num_slots: int
    gated: bool
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    state: torch.Tensor
    slot_idx: torch.Tensor
    scale: float
    gate: torch.Tensor | None = None
    norm_weight: torch.Tensor | None = None
    eps: float = 1e-6
    # Serving form: raw gate / beta (then g and beta are None).
    raw: "RawGate | None" = None
    # q, k, v read as slices of one packed row buffer (the serving form does).
    packed: bool = False
    # Block layout of the state pool: "kv" [num_slots, HV, K, V] or "vk"
    # [num_slots, HV, V, K] (key index fastest).
    state_layout: str = "kv"

    def state_kv(self) -> torch.Tensor:
        """The state pool as [num_slots, HV, K, V] (a transposed view for "vk")."""
        return self.state if self.state_layout == "kv" else self.state.transpose(-1, -2)

    def tensors(self):
        """Dict of the call's tensors (gate/norm_weight only when gated; the raw
        gate inputs instead of g and beta in the serving form)."""
        d = dict(q=self.q, k=self.k, v=self.v, state=self.state, slot_idx=self.slot_idx)
        if self.raw is None:
            d.update(g=self.g, beta=self.beta)
        else:
            d.update(raw_gate=self.raw.raw_gate, A_log=self.raw.A_log, dt_bias=self.raw.dt_bias,
                     raw_beta=self.raw.raw_beta)
        if self.gated:
            d.update(gate=self.gate, norm_weight=self.norm_weight)
        return d

    def to(self, device, state_too: bool = True) -> "Workload":
        """Copy of the workload with its tensors on ``device``."""
        upd = {}
        for key, t in self.tensors().items():
            if key == "state" and not state_too:
                continue
            upd[key] = t.to(device)
        raw = None
        if self.raw is not None:
            raw = RawGate(*(upd.pop(k) for k in ("raw_gate", "A_log", "dt_bias", "raw_beta")))
        return dataclasses.replace(self, raw=raw, **upd)

    def io_bytes(self) -> int:
        """Bytes of per-call inputs and outputs other than the state pool."""
        t = self.tensors()
        return sum(x.numel() * x.element_size() for key, x in t.items() if key != "state") + \
            self.N * self.T * self.HV * self.V * 2

    def state_bytes_touched(self) -> int:
        """State bytes one call reads (it writes the same amount back)."""
        active = int((self.slot_idx >= 0).sum())
        return active * self.HV * self.K * self.V * self.state.element_size()


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def make(N: int, T: int, HV: int, K: int = 128, V: int = 128, num_slots: int | None = None,
         gated: bool = False, seed: int = 0, name: str = "custom",
         decay: str = "softplus", inactive: int = 0, state_std: float = 0.02,
         state_dtype: str = "fp32", serving: bool = False, packed: bool | None = None,
         state_layout: str = "kv") -> Workload:
    """Draw one call's inputs.

    ``decay``: ``"softplus"`` (g = -softplus(N(0,1))) or ``"uniform"``
    (exp(g) ~ U[0.5, 1)).  ``inactive``: how many rows (the last ones) get a
    negative slot index, as CUDA-graph padding rows do.  ``serving``: raw gate
    and beta inputs instead of g and beta.  ``packed``: q, k, v to be passed as
    slices of one packed row buffer (default: as ``serving``).  ``state_layout``:
    "kv" or "vk" (the same draw, stored with the key index fastest).
    """
    gen = torch.Generator().manual_seed(seed)
    if num_slots is None:
        num_slots = max(1, 2 * N)
    if N > num_slots:
        raise ValueError("need N <= num_slots for distinct slots")

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = randn(N, T, HV, K)
    k = randn(N, T, HV, K)
    v = randn(N, T, HV, V)
    q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    if decay == "softplus":
        g = -torch.nn.functional.softplus(randn(N, T, HV, K))
    elif decay == "uniform":
        g = torch.log(0.5 + 0.5 * torch.rand(N, T, HV, K, generator=gen, dtype=torch.float32))
    else:
        raise ValueError(decay)
    beta = torch.sigmoid(randn(N, T, HV))
    state = randn(num_slots, HV, K, V) * state_std
    if state_dtype == "bf16":
        state = state.to(torch.bfloat16)
    elif state_dtype != "fp32":
        raise ValueError(state_dtype)
    if state_layout == "vk":
        state = state.transpose(-1, -2)
    elif state_layout != "kv":
        raise ValueError(state_layout)
    slot_idx = torch.randperm(num_slots, generator=gen)[:N].to(torch.int32)
    if inactive:
        slot_idx[N - inactive:] = -1
    gate = norm_weight = None
    if gated:
        gate = _bf16(randn(N, T, HV, V))
        norm_weight = _bf16(1.0 + 0.1 * randn(V))
    raw = raw_gate_inputs(N, T, HV, K, seed=seed) if serving else None
    return Workload(name=name, N=N, T=T, HV=HV, K=K, V=V, num_slots=num_slots, gated=gated,
                    q=_bf16(q), k=_bf16(k), v=_bf16(v),
                    g=None if serving else g.contiguous(), beta=None if serving else beta.contiguous(),
                    state=state.contiguous(), slot_idx=slot_idx.contiguous(),
                    scale=1.0 / math.sqrt(K), gate=gate, norm_weight=norm_weight, raw=raw,
                    packed=serving if packed is None else packed, state_layout=state_layout)


# The five workloads: name -> keyword arguments of ``make``.
CONFIGS = {
    "n1_t1_hv8": dict(N=1, T=1, HV=8, num_slots=1),
    "n32_t1_hv8": dict(N=32, T=1, HV=8, num_slots=64),
    "n32_t1_hv16_gated": dict(N=32, T=1, HV=16, num_slots=128, gated=True),
    "n32_t1_hv16": dict(N=32, T=1, HV=16, num_slots=128),  # the gated workload without the norm
    "n1_t4_hv8": dict(N=1, T=4, HV=8, num_slots=2),
    "n8_t4_hv8": dict(N=8, T=4, HV=8, num_slots=16),
    "n32_t4_hv8": dict(N=32, T=4, HV=8, num_slots=64),
    "n256_t1_hv32": dict(N=256, T=1, HV=32, num_slots=1024, decay="uniform"),
    # bf16 state pool (the state traffic halves)
    "n32_t1_hv8_bf16state": dict(N=32, T=1, HV=8, num_slots=64, state_dtype="bf16"),
    "n32_t1_hv16_gated_bf16state": dict(N=32, T=1, HV=16, num_slots=128, gated=True, state_dtype="bf16"),
    "n32_t4_hv8_bf16state": dict(N=32, T=4, HV=8, num_slots=64, state_dtype="bf16"),
    "n256_t1_hv32_bf16state": dict(N=256, T=1, HV=32, num_slots=1024, decay="uniform", state_dtype="bf16"),
    # serving input form: q, k, v packed in one row buffer, raw gate and beta activated in-kernel
    "n32_t1_hv8_raw": dict(N=32, T=1, HV=8, num_slots=64, serving=True),
    "n32_t1_hv16_gated_raw_bf16state": dict(N=32, T=1, HV=16, num_slots=128, gated=True, serving=True,
                                            state_dtype="bf16"),
    "n32_t4_hv8_raw": dict(N=32, T=4, HV=8, num_slots=64, serving=True),
    # q, k, v packed in one row buffer, activated g and beta (row-strided kernels)
    "n32_t1_hv8_packed": dict(N=32, T=1, HV=8, num_slots=64, packed=True),
    "n32_t4_hv8_packed": dict(N=32, T=4, HV=8, num_slots=64, packed=True),
    # [V, K] state blocks (key index fastest)
    "n32_t1_hv8_vk": dict(N=32, T=1, HV=8, num_slots=64, state_layout="vk"),
    "n32_t1_hv8_bf16state_vk": dict(N=32, T=1, HV=8, num_slots=64, state_dtype="bf16", state_layout="vk"),
    "n32_t4_hv8_vk": dict(N=32, T=4, HV=8, num_slots=64, state_layout="vk"),
    # general shapes: K outside {64, 128, 256}, V not a multiple of 32 (masked form)
    "n32_t1_hv8_k192_v130": dict(N=32, T=1, HV=8, K=192, V=130, num_slots=64),
    "n32_t4_hv8_k96_v100": dict(N=32, T=4, HV=8, K=96, V=100, num_slots=64),
}


# Long token runs for the chunked prefill (kda_prefill): one prompt of 64, 1000
# (a ragged last chunk) and 8192 tokens at 8 heads, and a batch of 8 prompts of
# 1024 tokens.  The pages give no prefill shapes; these take the decode
# serving shapes' 8 local heads and K = V = 128 (vLLM #57585, "Retained
# baseline trace attribution") with prompt lengths of the long-context
# serving runs it reports (2048-token and mixed 2048/32768-token inputs,
# "Follow-up serving validation").
PREFILL_CONFIGS = {
    "prefill_n1_t64_hv8": dict(N=1, T=64, HV=8, num_slots=2),
    "prefill_n1_t1000_hv8": dict(N=1, T=1000, HV=8, num_slots=2),
    "prefill_n1_t8192_hv8": dict(N=1, T=8192, HV=8, num_slots=2),
    "prefill_n8_t1024_hv8": dict(N=8, T=1024, HV=8, num_slots=16),
}


def config(name: str, seed: int = 0) -> Workload:
    """One of the named workloads (K = V = 128 unless the name says), drawn with ``seed``."""
    kw = CONFIGS[name] if name in CONFIGS else PREFILL_CONFIGS[name]
    return make(name=name, seed=seed, **kw)


@dataclasses.dataclass
class RawGate:
    """Serving-form decay and beta inputs: raw bf16 gate and beta, per-head
    A_log, per-head per-key-channel dt_bias."""
    raw_gate: torch.Tensor  # bf16 [N, T, HV, K]
    A_log: torch.Tensor     # fp32 [HV]
    dt_bias: torch.Tensor   # fp32 [HV, K]
    raw_beta: torch.Tensor  # bf16 [N, T, HV]

    def to(self, device) -> "RawGate":
        return RawGate(*(t.to(device) for t in (self.raw_gate, self.A_log, self.dt_bias, self.raw_beta)))


def raw_gate_inputs(N: int, T: int, HV: int, K: int, seed: int = 0) -> RawGate:
    """Draws in the ranges a KDA layer is initialised to: raw gate and raw beta
    ~ N(0, 1); A_log = log U[1, 16); dt_bias = softplus^-1(dt) with
    dt ~ U[0.001, 0.1) (so the decay rates sit mostly in (0.8, 1))."""
    gen = torch.Generator().manual_seed(seed + 999_983)
    raw_gate = torch.randn(N, T, HV, K, generator=gen).to(torch.bfloat16)
    raw_beta = torch.randn(N, T, HV, generator=gen).to(torch.bfloat16)
    A_log = torch.log(1.0 + 15.0 * torch.rand(HV, generator=gen))
    dt = 0.001 + 0.099 * torch.rand(HV, K, generator=gen)
    dt_bias = torch.log(torch.expm1(dt))
    return RawGate(raw_gate, A_log.float(), dt_bias.float(), raw_beta)


def pack_rows(parts, pad: int = 8):
    """One buffer whose (n, t) rows hold the given [N, T, ...] tensors side by
    side (as a packed ``mixed_qkv`` row holds q, k and v), each row padded by
    ``pad`` elements so the row stride exceeds the row width.  Returns the
    buffer and views of it shaped like the parts."""
    N, T = parts[0].shape[:2]
    widths = [p[0, 0].numel() for p in parts]
    buf = torch.zeros(N, T, sum(widths) + pad, dtype=parts[0].dtype, device=parts[0].device)
    views, off = [], 0
    for p, wd in zip(parts, widths):
        view = buf[:, :, off:off + wd].unflatten(-1, tuple(p.shape[2:]))
        view.copy_(p)
        views.append(view)
        off += wd
    return buf, views
