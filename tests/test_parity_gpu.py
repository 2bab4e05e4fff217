"""Parity of the CUDA path with the fp64 oracle, through the C ABI.

Every test draws seeded inputs from ``workloads`` (shared with the oracle),
runs the library on the GPU, runs the oracle on the CPU on the same inputs and
compares element by element with the tolerances of ``tests/parity.py``:
outputs within 1 bf16 ulp (and 2e-3 normwise), state within 1e-5 relative,
untouched slots bit-identical.
"""
import ctypes
import dataclasses
import os

import numpy as np
import pytest
import torch

import linear_attention_recurrent_decode_b200 as kda
import oracle
from linear_attention_recurrent_decode_b200 import workloads
from tests.parity import check_out, check_state, check_state_bf16

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))


def run_gpu(w, dev, out=None, stream=None):
    """Run one call on ``dev``; returns (out_fp64, pool_after_gpu, pool_before_gpu)."""
    d = w.to(dev)
    before = d.state.clone()
    if w.gated:
        o = kda.kda_decode_gated_rmsnorm(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, d.gate,
                                         d.norm_weight, eps=w.eps, scale=w.scale, out=out, stream=stream)
    else:
        o = kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, scale=w.scale, out=out,
                           stream=stream)
    torch.cuda.synchronize()
    return o, d.state, before


def run_oracle(w, rows=None):
    """Oracle on all rows, or on the listed rows only (with a compact pool of their slots)."""
    if rows is None:
        kw = dict(gate=w.gate, norm_weight=w.norm_weight, eps=w.eps) if w.gated else {}
        return oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale,
                                     threads=THREADS, **kw)
    rows = torch.as_tensor(rows)
    slots = w.slot_idx[rows]
    compact = w.state[slots.clamp_min(0).long()]
    local = torch.where(slots >= 0, torch.arange(len(rows), dtype=torch.int32), slots)
    kw = dict(gate=w.gate[rows], norm_weight=w.norm_weight, eps=w.eps) if w.gated else {}
    return oracle.kda_decode_ref(w.q[rows], w.k[rows], w.v[rows], w.g[rows], w.beta[rows], compact,
                                 local, w.scale, threads=THREADS, **kw)


def assert_parity(w, o_gpu, pool_gpu, pool_before, rows=None):
    out_ref, st_ref = run_oracle(w, rows)
    sel = slice(None) if rows is None else torch.as_tensor(rows)
    check_out(o_gpu[sel].float().cpu().numpy(), out_ref)
    slots = w.slot_idx if rows is None else w.slot_idx[torch.as_tensor(rows)]
    for i, s in enumerate(slots.tolist()):
        if s < 0:
            continue
        ref = st_ref[s] if rows is None else st_ref[i]
        if pool_gpu.dtype == torch.bfloat16:
            check_state_bf16(pool_gpu[s].float().cpu().numpy(), ref, what=f"bf16 state slot {s}")
        else:
            check_state(pool_gpu[s].cpu().numpy(), ref, what=f"state slot {s}")
    # every slot that no active row names is bit-identical
    touched = torch.zeros(w.num_slots, dtype=torch.bool, device=pool_gpu.device)
    act = w.slot_idx[w.slot_idx >= 0].long().to(pool_gpu.device)
    touched[act] = True
    assert torch.equal(pool_gpu[~touched], pool_before[~touched]), "an untouched slot changed"
    if len(act):
        changed = (pool_gpu[act] != pool_before[act]).flatten(1).any(dim=1)
        assert bool(changed.all()), "an active slot was not written"


SMALL_CONFIGS = ["n1_t1_hv8", "n32_t1_hv8", "n32_t1_hv16_gated", "n1_t4_hv8", "n8_t4_hv8", "n32_t4_hv8",
                 "n32_t1_hv8_k192_v130", "n32_t4_hv8_k96_v100",
                 "n32_t1_hv8_bf16state", "n32_t1_hv16_gated_bf16state", "n32_t4_hv8_bf16state"]


@pytest.mark.parametrize("name", SMALL_CONFIGS)
def test_named_workload_parity(name, cuda_device):
    w = workloads.config(name)
    o, pool, before = run_gpu(w, cuda_device)
    assert_parity(w, o, pool, before)


@pytest.mark.parametrize("name", ["n256_t1_hv32", "n256_t1_hv32_bf16state"])
def test_large_batch_parity_sampled(name, cuda_device):
    """N=256, T=1, HV=32, 1024-slot pool (2 GiB fp32 / 1 GiB bf16): sampled rows
    against the oracle, including the rows whose slots sit furthest into the
    pool, every other slot checked bit-exact on the GPU."""
    w = workloads.config(name)
    o, pool, before = run_gpu(w, cuda_device)
    order = torch.argsort(w.slot_idx, descending=True)
    rows = sorted(set(order[:8].tolist()) | set(range(0, 256, 9)))
    assert int(w.slot_idx[rows].max()) >= 1000
    assert_parity(w, o, pool, before, rows=rows)


@pytest.mark.parametrize("gated", [False, True])
def test_pool_offsets_beyond_32_bits(gated, cuda_device):
    """Slots whose element offsets exceed 2^31 (a 8.6 GB pool): the kernel's
    64-bit slot arithmetic lands every row in its own slot.  Only the active
    slots hold drawn states; the rest of the pool is zero and must stay zero."""
    HV, K, V = 2, 128, 128
    num_slots = 66_000  # 66000 * 2 * 128 * 128 = 2.16e9 elements > 2^31
    w = workloads.make(N=4, T=2, HV=HV, K=K, V=V, num_slots=4, gated=gated, seed=21)
    big_slots = torch.tensor([65_999, 32_768, 65_537, 7], dtype=torch.int32)
    assert int(big_slots.max()) * HV * K * V > 2 ** 31
    pool = torch.zeros(num_slots, HV, K, V, dtype=torch.float32, device=cuda_device)
    pool[big_slots.long().to(cuda_device)] = w.state[w.slot_idx.long()].to(cuda_device)
    d = w.to(cuda_device, state_too=False)
    big_idx = big_slots.to(cuda_device)
    if gated:
        o = kda.kda_decode_gated_rmsnorm(d.q, d.k, d.v, d.g, d.beta, pool, big_idx, d.gate, d.norm_weight,
                                         eps=w.eps, scale=w.scale)
    else:
        o = kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, pool, big_idx, scale=w.scale)
    torch.cuda.synchronize()
    kw = dict(gate=w.gate, norm_weight=w.norm_weight, eps=w.eps) if gated else {}
    out_ref, st_ref = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale, **kw)
    check_out(o.float().cpu().numpy(), out_ref)
    for n in range(w.N):
        check_state(pool[int(big_slots[n])].cpu().numpy(), st_ref[int(w.slot_idx[n])])
    mask = torch.ones(num_slots, dtype=torch.bool, device=cuda_device)
    mask[big_slots.long().to(cuda_device)] = False
    assert int(torch.count_nonzero(pool[mask])) == 0
    del pool


CASES = [
    # N, T, HV, K, V, gated, inactive
    (1, 1, 1, 128, 32, False, 0),
    (3, 1, 3, 128, 96, False, 0),       # 3 tiles: ragged V
    (5, 2, 2, 64, 160, False, 1),
    (4, 3, 1, 256, 64, False, 0),
    (2, 5, 2, 128, 128, False, 0),
    (7, 1, 5, 128, 128, False, 2),      # padding rows
    (2, 8, 1, 64, 32, False, 0),
    (1, 1, 1, 128, 32, True, 0),        # cluster of 1
    (3, 1, 3, 128, 96, True, 0),
    (2, 3, 2, 64, 256, True, 1),        # cluster of 8 (largest)
    (4, 2, 2, 256, 128, True, 0),
    (6, 4, 2, 128, 224, True, 2),
    # more tokens than one shared-memory chunk: prefetch of the next chunk, ragged last chunk
    (3, 9, 2, 128, 128, False, 0),
    (2, 17, 3, 64, 96, False, 1),
    (2, 20, 2, 256, 64, False, 0),
    (3, 9, 2, 128, 128, True, 1),
    (2, 17, 1, 64, 256, True, 0),
    # widest supported shapes: 8 value tiles with K = 256 (plain and one cluster of 8), many heads
    (2, 1, 2, 256, 256, False, 0),
    (2, 2, 2, 256, 256, True, 0),
    (1, 1, 64, 128, 128, False, 0),
    (1, 5, 48, 128, 128, True, 0),
    (3, 1, 1, 128, 512, False, 0),
]


@pytest.mark.parametrize("N,T,HV,K,V,gated,inactive", CASES)
def test_shapes_parity(N, T, HV, K, V, gated, inactive, cuda_device):
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=2 * N + 1, gated=gated,
                       inactive=inactive, seed=N * 1000 + T * 100 + V)
    o, pool, before = run_gpu(w, cuda_device)
    assert_parity(w, o, pool, before)
    if inactive:
        assert torch.all(o[N - inactive:] == 0)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("T", [4, 12])
def test_t_steps_equal_successive_single_steps(gated, T, cuda_device):
    w = workloads.make(N=6, T=T, HV=3, K=128, V=128, num_slots=9, gated=gated, seed=11)
    d = w.to(cuda_device)
    pool_a = d.state.clone()
    pool_b = d.state.clone()
    fn = kda.kda_decode_gated_rmsnorm if gated else kda.kda_decode
    extra = (lambda sl: (d.gate[:, sl].contiguous(), d.norm_weight)) if gated else (lambda sl: ())
    out_a = fn(d.q, d.k, d.v, d.g, d.beta, pool_a, d.slot_idx, *extra(slice(None)))
    outs = []
    for t in range(w.T):
        sl = slice(t, t + 1)
        outs.append(fn(d.q[:, sl].contiguous(), d.k[:, sl].contiguous(), d.v[:, sl].contiguous(),
                       d.g[:, sl].contiguous(), d.beta[:, sl].contiguous(), pool_b, d.slot_idx,
                       *extra(sl)))
    torch.cuda.synchronize()
    # The multi-token kernel regroups the same arithmetic by chunks of tokens,
    # so the two paths agree to rounding, not bit for bit.
    check_out(out_a.float().cpu().numpy(), torch.cat(outs, dim=1).float().cpu().numpy(), what="T-call vs T calls")
    for s_ in w.slot_idx.tolist():
        check_state(pool_a[s_].cpu().numpy(), pool_b[s_].cpu().numpy(), what=f"slot {s_}")
    untouched = torch.ones(w.num_slots, dtype=torch.bool, device=cuda_device)
    untouched[w.slot_idx.long().to(cuda_device)] = False
    assert torch.equal(pool_a[untouched], pool_b[untouched])


def test_empty_batch_is_noop(cuda_device):
    w = workloads.make(N=2, T=1, HV=2, K=128, V=128, num_slots=3)
    d = w.to(cuda_device)
    before = d.state.clone()
    kda.kda_decode(d.q[:0], d.k[:0], d.v[:0], d.g[:0], d.beta[:0], d.state, d.slot_idx[:0])
    kda.kda_decode(d.q[:, :0], d.k[:, :0], d.v[:, :0], d.g[:, :0], d.beta[:, :0], d.state, d.slot_idx)
    torch.cuda.synchronize()
    assert torch.equal(d.state, before)


def test_all_rows_inactive(cuda_device):
    w = workloads.make(N=3, T=2, HV=2, K=128, V=64, num_slots=4, inactive=3, gated=True)
    o, pool, before = run_gpu(w, cuda_device, out=torch.full((3, 2, 2, 64), 7.0, dtype=torch.bfloat16,
                                                              device=cuda_device))
    assert torch.all(o == 0)
    assert torch.equal(pool, before)


def test_side_stream_and_graph_replay(cuda_device):
    """A call captured in a CUDA graph on a side stream replays to the eager result."""
    w = workloads.config("n32_t1_hv8")
    d = w.to(cuda_device)
    pool_eager = d.state.clone()
    pool_graph = d.state.clone()
    out_eager = kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, pool_eager, d.slot_idx)
    out_graph = torch.empty_like(out_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, pool_graph, d.slot_idx, out=out_graph, stream=s)
    torch.cuda.synchronize()
    assert torch.equal(pool_graph, d.state), "capture must not execute the kernel"
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_graph, out_eager)
    assert torch.equal(pool_graph, pool_eager)
    graph.replay()  # a second step advances the state again, like the eager path
    kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, pool_eager, d.slot_idx)
    torch.cuda.synchronize()
    assert torch.equal(pool_graph, pool_eager)
    del graph


def test_rejections_with_real_buffers(cuda_device):
    w = workloads.make(N=2, T=1, HV=2, K=128, V=128, num_slots=3)
    d = w.to(cuda_device)
    lib = kda.library()
    s = torch.cuda.current_stream().cuda_stream
    before = d.state.clone()

    def call(q=None, out=None, state=None, K=128):
        return lib.kda_decode(q or d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), d.g.data_ptr(),
                              d.beta.data_ptr(), state or d.state.data_ptr(), d.slot_idx.data_ptr(),
                              out or d.q.data_ptr() + 64, 2, 1, 2, K, 128, 0.1, s)

    out = torch.empty(2, 1, 2, 128, dtype=torch.bfloat16, device=cuda_device)
    assert call() == kda.KDA_ERR_ALIAS                             # out inside q
    assert call(out=d.state.data_ptr()) == kda.KDA_ERR_ALIAS       # out = pool
    assert call(out=out.data_ptr() + 2) == kda.KDA_ERR_MISALIGNED
    assert call(out=out.data_ptr(), K=300) == kda.KDA_ERR_UNSUPPORTED
    assert call(out=out.data_ptr(), q=d.q.data_ptr() + 8) == kda.KDA_ERR_MISALIGNED
    torch.cuda.synchronize()
    assert torch.equal(d.state, before)
    assert call(out=out.data_ptr()) == kda.KDA_OK
    with pytest.raises(kda.KdaError):
        kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, out=d.v)
    torch.cuda.synchronize()


@pytest.mark.parametrize("gated", [False, True])
def test_back_to_back_calls_see_prior_writes(gated, cuda_device):
    """Calls are launched with programmatic stream serialization; each call must
    still see everything earlier in the stream: the previous call's state write
    and a torch kernel that rewrites the next call's inputs in place."""
    w = workloads.make(N=8, T=1, HV=4, K=128, V=128, num_slots=16, gated=gated, seed=31)
    d = w.to(cuda_device)
    fn = kda.kda_decode_gated_rmsnorm if gated else kda.kda_decode
    extra = (d.gate, d.norm_weight) if gated else ()
    outs = []
    for step in range(3):
        outs.append(fn(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, *extra).clone())
        d.v.mul_(-0.5)          # foreign kernels on the same stream between calls
        d.g.add_(-0.25)
    torch.cuda.synchronize()
    state = w.state.double().numpy().copy()
    v, g = w.v.clone(), w.g.clone()
    kw = dict(gate=w.gate, norm_weight=w.norm_weight, eps=w.eps) if gated else {}
    for step in range(3):
        ref, state = oracle.kda_decode_ref(w.q, w.k, v, g, w.beta, state, w.slot_idx, w.scale, **kw)
        check_out(outs[step].float().cpu().numpy(), ref, what=f"step {step}")
        v = (v.float() * -0.5).to(torch.bfloat16)
        g = g + -0.25
    for s in w.slot_idx.tolist():
        check_state(d.state[s].cpu().numpy(), state[s], what=f"slot {s}")


def test_random_shapes_against_oracle(cuda_device):
    """Seeded sweep of small random shapes (all K, V multiples of 32 up to 256,
    T up to 11, random padding rows, plain and gated) against the oracle."""
    rng = np.random.default_rng(20261202)
    for case in range(24):
        K = int(rng.choice([64, 128, 256]))
        gated = bool(rng.integers(0, 2))
        V = 32 * int(rng.integers(1, 9))
        N = int(rng.integers(1, 6))
        T = int(rng.integers(1, 12))
        HV = int(rng.integers(1, 5))
        inactive = int(rng.integers(0, N))
        w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=N + int(rng.integers(0, 4)), gated=gated,
                           inactive=inactive, seed=1000 + case,
                           decay=str(rng.choice(["softplus", "uniform"])))
        o, pool, before = run_gpu(w, cuda_device)
        try:
            assert_parity(w, o, pool, before)
        except AssertionError as e:
            raise AssertionError(f"case {case}: N={N} T={T} HV={HV} K={K} V={V} gated={gated} "
                                 f"inactive={inactive}: {e}") from e


BF16_CASES = [
    # N, T, HV, K, V, gated, inactive
    (3, 1, 3, 128, 96, False, 0),
    (5, 2, 2, 64, 160, False, 1),
    (2, 9, 2, 128, 128, False, 0),
    (4, 1, 2, 256, 128, True, 1),
    (2, 6, 2, 128, 256, True, 0),
]


@pytest.mark.parametrize("N,T,HV,K,V,gated,inactive", BF16_CASES)
def test_bf16_state_shapes_parity(N, T, HV, K, V, gated, inactive, cuda_device):
    """bf16 state pool: fp32 math, state rounded to bf16 once per call."""
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=2 * N + 1, gated=gated, inactive=inactive,
                       seed=7000 + N * 100 + T, state_dtype="bf16")
    o, pool, before = run_gpu(w, cuda_device)
    assert pool.dtype == torch.bfloat16
    assert_parity(w, o, pool, before)


def test_bf16_state_beta0_g0_is_bit_identical(cuda_device):
    """beta = 0 and g = 0 leave a bf16 pool bit for bit (widening and rounding are exact)."""
    w = workloads.make(N=4, T=3, HV=2, K=128, V=128, num_slots=6, seed=77, state_dtype="bf16")
    w.beta.zero_()
    w.g.zero_()
    o, pool, before = run_gpu(w, cuda_device)
    assert torch.equal(pool, before)


# ---------------------------------------------------------------------------
# kda_decode_ex: strided / packed inputs and the raw serving form
# ---------------------------------------------------------------------------
def test_ex_dense_equals_fixed_entry_points(cuda_device):
    for gated in (False, True):
        w = workloads.make(N=5, T=3, HV=2, K=128, V=96, num_slots=7, gated=gated, seed=41)
        d = w.to(cuda_device)
        p1, p2 = d.state.clone(), d.state.clone()
        extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if gated else {}
        o1 = kda.kda_decode_ex(d.q, d.k, d.v, p1, d.slot_idx, g=d.g, beta=d.beta, **extra)
        fn = kda.kda_decode_gated_rmsnorm if gated else kda.kda_decode
        o2 = fn(d.q, d.k, d.v, d.g, d.beta, p2, d.slot_idx, *((d.gate, d.norm_weight) if gated else ()))
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(p1, p2)


@pytest.mark.parametrize("T,gated,state", [(1, False, "fp32"), (1, True, "fp32"), (5, False, "fp32"),
                                           (1, False, "bf16"), (6, True, "bf16")])
def test_ex_packed_mixed_qkv_and_strided_gate(T, gated, state, cuda_device):
    """q, k, v as slices of one padded packed row; g and beta as strided slices too."""
    w = workloads.make(N=4, T=T, HV=3, K=128, V=128, num_slots=6, gated=gated, seed=43, state_dtype=state)
    d = w.to(cuda_device)
    _, (q, k, v) = workloads.pack_rows([d.q, d.k, d.v], pad=24)
    _, (g, beta) = workloads.pack_rows([d.g, d.beta.unsqueeze(-1)], pad=5)  # 392 floats: 16-byte rows
    beta = beta.squeeze(-1)
    assert not q.is_contiguous() and q.stride(0) == T * (2 * 3 * 128 + 3 * 128 + 24)
    before = d.state.clone()
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if gated else {}
    o = kda.kda_decode_ex(q, k, v, d.state, d.slot_idx, g=g, beta=beta, **extra)
    torch.cuda.synchronize()
    assert_parity(w, o, d.state, before)


@pytest.mark.parametrize("N,T,HV,K,V,gated,state", [
    (4, 1, 2, 128, 128, False, "fp32"),
    (32, 1, 8, 128, 128, False, "fp32"),
    (3, 1, 2, 128, 128, True, "fp32"),
    (3, 4, 2, 128, 128, False, "fp32"),
    (2, 9, 2, 64, 96, True, "fp32"),
    (3, 1, 2, 256, 64, False, "bf16"),
    (2, 5, 2, 128, 128, True, "bf16"),
])
def test_ex_raw_gate_form_against_the_reading(N, T, HV, K, V, gated, state, cuda_device):
    """Raw gate / beta activated in the kernel, inputs packed like mixed_qkv;
    against the oracle's activation feeding its recurrence.  The activation
    formula is a reading no page prints (parity unpinned): this checks the
    kernel against that reading, not against the pages."""
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=N + 3, gated=gated, seed=50 + N + T,
                       state_dtype=state, inactive=1 if N > 2 else 0)
    rg = workloads.raw_gate_inputs(N, T, HV, K, seed=51)
    d, r = w.to(cuda_device), rg.to(cuda_device)
    _, (q, k, v) = workloads.pack_rows([d.q, d.k, d.v], pad=8)
    before = d.state.clone()
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if gated else {}
    o = kda.kda_decode_ex(q, k, v, d.state, d.slot_idx, raw_gate=r.raw_gate, A_log=r.A_log,
                          dt_bias=r.dt_bias, raw_beta=r.raw_beta, **extra)
    torch.cuda.synchronize()
    g, beta = oracle.activate(rg.raw_gate, rg.A_log, rg.dt_bias, rg.raw_beta)
    w_ref = dataclasses.replace(w, g=torch.from_numpy(g), beta=torch.from_numpy(beta))
    assert_parity(w_ref, o, d.state, before)


SERVING_CONFIGS = [n for n in workloads.CONFIGS if "_raw" in n or "_packed" in n or n.endswith("_vk")]


@pytest.mark.parametrize("name", SERVING_CONFIGS)
def test_named_serving_workload_parity(name, cuda_device):
    """The packed, serving-form and [V, K]-pool workloads, called as the
    benchmark calls them (kda_decode_ex; q, k, v packed in one row buffer when
    the workload says so; raw gate and beta, or activated ones).  For the
    ``*_raw*`` workloads the reference is the oracle's activation reading
    (parity unpinned by the pages), not a formula the pages print."""
    w = workloads.config(name)
    d = w.to(cuda_device)
    q, k, v = d.q, d.k, d.v
    if w.packed:
        _, (q, k, v) = workloads.pack_rows([d.q, d.k, d.v], pad=8)
    before = d.state_kv().clone()
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if w.gated else {}
    if w.raw is not None:
        extra.update(raw_gate=d.raw.raw_gate, A_log=d.raw.A_log, dt_bias=d.raw.dt_bias, raw_beta=d.raw.raw_beta)
    else:
        extra.update(g=d.g, beta=d.beta)
    o = kda.kda_decode_ex(q, k, v, d.state, d.slot_idx, scale=w.scale, state_layout=w.state_layout, **extra)
    torch.cuda.synchronize()
    if w.raw is not None:
        g, beta = oracle.activate(w.raw.raw_gate, w.raw.A_log, w.raw.dt_bias, w.raw.raw_beta)
        w = dataclasses.replace(w, g=torch.from_numpy(g), beta=torch.from_numpy(beta))
    assert_parity(dataclasses.replace(w, state=w.state_kv()), o, d.state_kv(), before)


@pytest.mark.parametrize("T,gated,state", [(1, False, "fp32"), (1, True, "bf16"), (4, False, "fp32"),
                                           (7, True, "fp32")])
def test_strided_form_bit_identical_to_dense(T, gated, state, cuda_device):
    """The strided-input kernels differ from the dense ones only in addressing:
    the same values laid out in packed rows give bit-identical outputs and state."""
    w = workloads.make(N=6, T=T, HV=4, K=128, V=128, num_slots=9, gated=gated, seed=60 + T,
                       state_dtype=state, inactive=1)
    d = w.to(cuda_device)
    p_dense, p_strided = d.state.clone(), d.state.clone()
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if gated else {}
    o_dense = kda.kda_decode_ex(d.q, d.k, d.v, p_dense, d.slot_idx, g=d.g, beta=d.beta, **extra)
    _, (q, k, v) = workloads.pack_rows([d.q, d.k, d.v], pad=16)
    _, (g, beta) = workloads.pack_rows([d.g, d.beta.unsqueeze(-1)], pad=4)  # 520 floats: 16-byte rows
    if gated:
        _, (z,) = workloads.pack_rows([d.gate], pad=8)
        extra["gate"] = z
    o_strided = kda.kda_decode_ex(q, k, v, p_strided, d.slot_idx, g=g, beta=beta.squeeze(-1), **extra)
    torch.cuda.synchronize()
    assert torch.equal(o_dense, o_strided)
    assert torch.equal(p_dense, p_strided)


VK_CASES = [  # N, T, HV, K, V, gated, state dtype, input form
    (5, 1, 3, 128, 128, False, "fp32", "dense"),
    (5, 1, 3, 128, 128, True, "fp32", "dense"),
    (4, 1, 2, 64, 96, False, "fp32", "dense"),
    (3, 1, 2, 256, 64, True, "fp32", "dense"),
    (5, 4, 3, 128, 128, False, "fp32", "dense"),
    (3, 9, 2, 128, 160, True, "fp32", "dense"),
    (4, 1, 3, 128, 128, False, "bf16", "dense"),
    (4, 1, 3, 64, 128, True, "bf16", "dense"),
    (3, 6, 2, 256, 128, False, "bf16", "dense"),
    (4, 1, 3, 128, 128, False, "fp32", "raw"),
    (3, 5, 2, 128, 128, True, "bf16", "raw"),
]


def _vk_call(w, d, pool, layout, form):
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if w.gated else {}
    if form == "raw":
        r = d.raw
        extra.update(raw_gate=r.raw_gate, A_log=r.A_log, dt_bias=r.dt_bias, raw_beta=r.raw_beta)
    else:
        extra.update(g=d.g, beta=d.beta)
    return kda.kda_decode_ex(d.q, d.k, d.v, pool, d.slot_idx, scale=w.scale, state_layout=layout, **extra)


@pytest.mark.parametrize("N,T,HV,K,V,gated,state,form", VK_CASES)
def test_vk_layout_parity(N, T, HV, K, V, gated, state, form, cuda_device):
    """[V, K] state blocks: against the oracle on the same state read as [K, V],
    and bit-identical to the [K, V] pool (the same arithmetic, another address
    map).  The ``raw`` cases check against the oracle's activation reading
    (parity unpinned by the pages)."""
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=N + 3, gated=gated, seed=70 + N + T + K,
                       state_dtype=state, inactive=1, serving=form == "raw", packed=False)
    d = w.to(cuda_device)
    pool_kv = d.state.clone()
    pool_vk = d.state.transpose(-1, -2).contiguous()
    before = d.state.clone()
    o_kv = _vk_call(w, d, pool_kv, "kv", form)
    o_vk = _vk_call(w, d, pool_vk, "vk", form)
    torch.cuda.synchronize()
    assert torch.equal(o_kv, o_vk), "outputs differ between the [K, V] and [V, K] pools"
    assert torch.equal(pool_kv, pool_vk.transpose(-1, -2)), "states differ between the [K, V] and [V, K] pools"
    if form == "raw":
        g, beta = oracle.activate(w.raw.raw_gate, w.raw.A_log, w.raw.dt_bias, w.raw.raw_beta)
        w = dataclasses.replace(w, g=torch.from_numpy(g), beta=torch.from_numpy(beta))
    assert_parity(w, o_vk, pool_vk.transpose(-1, -2), before)


def test_vk_layout_rejects_wrong_pool_shape(cuda_device):
    w = workloads.make(N=2, T=1, HV=2, K=128, V=64, num_slots=3, seed=5)
    d = w.to(cuda_device)
    with pytest.raises(ValueError):
        kda.kda_decode_ex(d.q, d.k, d.v, d.state, d.slot_idx, g=d.g, beta=d.beta, state_layout="vk")


@pytest.mark.parametrize("name", ["n32_t1_hv8", "n32_t1_hv16_gated", "n8_t4_hv8", "n32_t1_hv8_raw"])
def test_host_step_equals_device_call(name, cuda_device):
    """HostStep (kda_decode_host): inputs staged in pinned host memory, copied in,
    decoded and the output copied back by one library call per step.  Two
    steps on one pool give the same outputs and state as two kda_decode_ex
    calls on device tensors."""
    w = workloads.config(name)
    inputs = {key: t for key, t in w.tensors().items() if key != "state"}
    nbytes = sum((t.numel() * t.element_size() + 15) // 16 * 16 for t in inputs.values())
    host_in = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty(nbytes, dtype=torch.uint8, device=cuda_device)
    hv, dv, off = {}, {}, 0
    for key, t in inputs.items():
        b = t.numel() * t.element_size()
        hv[key] = host_in[off:off + b].view(t.dtype).view(t.shape)
        dv[key] = dev_in[off:off + b].view(t.dtype).view(t.shape)
        hv[key].copy_(t)
        off += (b + 15) // 16 * 16
    extra = dict(gate=dv["gate"], norm_weight=dv["norm_weight"], eps=w.eps) if w.gated else {}
    if w.raw is not None:
        extra.update(raw_gate=dv["raw_gate"], A_log=dv["A_log"], dt_bias=dv["dt_bias"], raw_beta=dv["raw_beta"])
    else:
        extra.update(g=dv["g"], beta=dv["beta"])
    pool_h = w.state.to(cuda_device)
    out_d = torch.empty(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16, device=cuda_device)
    host_out = torch.empty(out_d.shape, dtype=torch.bfloat16).pin_memory()
    step = kda.HostStep(dv["q"], dv["k"], dv["v"], pool_h, dv["slot_idx"], host_in=host_in, dev_in=dev_in,
                        host_out=host_out, out=out_d, scale=w.scale, **extra)
    d = w.to(cuda_device)
    pool_ref = d.state.clone()
    ref_extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if w.gated else {}
    if w.raw is not None:
        ref_extra.update(raw_gate=d.raw.raw_gate, A_log=d.raw.A_log, dt_bias=d.raw.dt_bias, raw_beta=d.raw.raw_beta)
    else:
        ref_extra.update(g=d.g, beta=d.beta)
    for _ in range(2):
        dev_in.zero_()  # the step must bring its own inputs in
        step()
        torch.cuda.synchronize()
        ref = kda.kda_decode_ex(d.q, d.k, d.v, pool_ref, d.slot_idx, scale=w.scale, **ref_extra)
        torch.cuda.synchronize()
        assert torch.equal(host_out, ref.cpu())
        assert torch.equal(pool_h, pool_ref)


def test_host_step_rejects_views_outside_the_staging_buffer(cuda_device):
    w = workloads.make(N=2, T=1, HV=2, K=128, V=64, num_slots=3, seed=9)
    d = w.to(cuda_device)
    host_in = torch.empty(1 << 16, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty(1 << 16, dtype=torch.uint8, device=cuda_device)
    out = torch.empty(2, 1, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    host_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(ValueError):
        kda.HostStep(d.q, d.k, d.v, d.state, d.slot_idx, host_in=host_in, dev_in=dev_in, host_out=host_out,
                     out=out, g=d.g, beta=d.beta)


@pytest.mark.parametrize("N,T,HV,K,V,gated,state,layout,form", [
    # long token runs: many chunks, a ragged last chunk, every input form and pool format
    (2, 37, 2, 128, 128, False, "fp32", "kv", "dense"),
    (2, 37, 2, 128, 96, True, "fp32", "vk", "dense"),
    (2, 33, 2, 64, 128, False, "bf16", "vk", "raw"),
    (2, 23, 2, 256, 64, True, "bf16", "kv", "raw"),
    (3, 13, 2, 128, 128, True, "fp32", "vk", "raw"),
    (2, 29, 3, 256, 128, False, "fp32", "vk", "dense"),
])
def test_long_token_runs_every_form(N, T, HV, K, V, gated, state, layout, form, cuda_device):
    """T up to 37 tokens in one call (ten chunks of four with a ragged tail),
    across pool dtypes, pool layouts and input forms, against the oracle (the
    ``raw`` cases against its activation reading, parity unpinned by the
    pages)."""
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=N + 2, gated=gated, seed=80 + T + K,
                       state_dtype=state, inactive=1 if N > 2 else 0, serving=form == "raw", packed=False,
                       decay="uniform")
    d = w.to(cuda_device)
    before = d.state.clone()
    pool = d.state.clone() if layout == "kv" else d.state.transpose(-1, -2).contiguous()
    o = _vk_call(w, d, pool, layout, form)
    torch.cuda.synchronize()
    if form == "raw":
        g, beta = oracle.activate(w.raw.raw_gate, w.raw.A_log, w.raw.dt_bias, w.raw.raw_beta)
        w = dataclasses.replace(w, g=torch.from_numpy(g), beta=torch.from_numpy(beta))
    assert_parity(w, o, pool if layout == "kv" else pool.transpose(-1, -2), before)


# ---------------------------------------------------------------------------
# checked slots (kda_decode_args.num_slots / status)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,gated,state,form", [
    (1, False, "fp32", "dense"), (1, True, "bf16", "dense"), (1, False, "fp32", "raw"),
    (6, True, "fp32", "dense"), (5, False, "bf16", "raw"),
])
def test_checked_slots_skip_rows_beyond_the_declared_pool(T, gated, state, form, cuda_device):
    """With the pool's size declared, a row naming a slot at or past it is
    skipped like a padding row (zero output, pool untouched) and raises the
    status word.  The pool is allocated with two slots more than declared, so
    the out-of-range slots still lie inside the allocation: a guard that failed
    would change those slots (checked bit for bit) but could not fault."""
    declared = 6
    w = workloads.make(N=4, T=T, HV=2, K=128, V=128, num_slots=declared + 2, gated=gated, seed=90 + T,
                       state_dtype=state, serving=form == "raw", packed=False)
    w.slot_idx.copy_(torch.tensor([0, declared, 3, declared + 1], dtype=torch.int32))
    d = w.to(cuda_device)
    before = d.state.clone()
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    extra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if gated else {}
    if form == "raw":
        r = d.raw
        extra.update(raw_gate=r.raw_gate, A_log=r.A_log, dt_bias=r.dt_bias, raw_beta=r.raw_beta)
    else:
        extra.update(g=d.g, beta=d.beta)
    o = kda.kda_decode_ex(d.q, d.k, d.v, d.state, d.slot_idx, scale=w.scale, num_slots=declared,
                          status=status, **extra)
    torch.cuda.synchronize()
    assert int(status.item()) == 1, "an out-of-range slot did not raise the status word"
    ref = dataclasses.replace(w, slot_idx=torch.tensor([0, -1, 3, -1], dtype=torch.int32))
    if form == "raw":
        g, beta = oracle.activate(w.raw.raw_gate, w.raw.A_log, w.raw.dt_bias, w.raw.raw_beta)
        ref = dataclasses.replace(ref, g=torch.from_numpy(g), beta=torch.from_numpy(beta))
    assert_parity(ref, o, d.state, before)
    assert torch.equal(d.state[declared:], before[declared:])

    # every slot in range: the status word stays as the caller left it (zero)
    status.zero_()
    d.slot_idx.copy_(torch.tensor([0, 5, 3, -1], dtype=torch.int32, device=cuda_device))
    kda.kda_decode_ex(d.q, d.k, d.v, d.state, d.slot_idx, scale=w.scale, num_slots=declared,
                      status=status, **extra)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_checked_slots_equal_unchecked_when_in_range(cuda_device):
    """Declaring the pool's size changes nothing for in-range slots: the checked
    call (row-strided kernels) is bit-identical to the unchecked dense one."""
    w = workloads.make(N=8, T=1, HV=4, K=128, V=128, num_slots=12, seed=95, inactive=2)
    d1, d2 = w.to(cuda_device), w.to(cuda_device)
    o1 = kda.kda_decode_ex(d1.q, d1.k, d1.v, d1.state, d1.slot_idx, g=d1.g, beta=d1.beta, num_slots=0)
    o2 = kda.kda_decode_ex(d2.q, d2.k, d2.v, d2.state, d2.slot_idx, g=d2.g, beta=d2.beta, num_slots=12)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(d1.state, d2.state)


# ---------------------------------------------------------------------------
# general K and V (masked, element-wise form)
# ---------------------------------------------------------------------------
GENERAL_CASES = [
    (3, 1, 2, 96, 100, False, "fp32", 1),
    (3, 1, 2, 192, 130, True, "fp32", 1),
    (2, 5, 2, 96, 130, False, "fp32", 0),
    (3, 7, 3, 192, 100, True, "bf16", 1),
    (2, 1, 2, 48, 17, False, "bf16", 0),
    (3, 6, 1, 200, 33, True, "fp32", 1),
    (3, 3, 2, 128, 100, False, "fp32", 1),   # K of the vectorised set, V ragged
    (2, 1, 2, 80, 128, True, "fp32", 0),     # V of the vectorised set, K ragged
    (2, 9, 2, 1, 1, False, "fp32", 0),       # one key channel, one value column
    (2, 13, 2, 256, 250, True, "bf16", 1),   # eight value tiles, the last ragged
]


@pytest.mark.parametrize("N,T,HV,K,V,gated,state,inactive", GENERAL_CASES)
def test_general_shapes_parity(N, T, HV, K, V, gated, state, inactive, cuda_device):
    """K outside {64, 128, 256} (rows padded, masked) and V not a multiple of 32
    (last value tile masked), through the fixed entry points, against the oracle;
    padding rows included."""
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=N + 2, gated=gated, seed=400 + K + V + T,
                       state_dtype=state, inactive=inactive)
    o, pool, before = run_gpu(w, cuda_device)
    assert_parity(w, o, pool, before)


@pytest.mark.parametrize("T,gated", [(1, False), (1, True), (6, False), (5, True)])
def test_general_shapes_strided_rows(T, gated, cuda_device):
    """The general form with q, k, v as slices of one packed row buffer whose
    row stride is odd (rows of no particular alignment), bit-identical to the
    dense call."""
    w = workloads.make(N=3, T=T, HV=2, K=96, V=100, num_slots=5, gated=gated, seed=450 + T, inactive=1)
    d1, d2 = w.to(cuda_device), w.to(cuda_device)
    _, (q, k, v) = workloads.pack_rows([d2.q, d2.k, d2.v], pad=3)
    assert (q.stride(1) if T > 1 else q.stride(0)) % 2 == 1  # rows two bytes apart from alignment
    extra1 = dict(gate=d1.gate, norm_weight=d1.norm_weight, eps=w.eps) if gated else {}
    extra2 = dict(gate=d2.gate, norm_weight=d2.norm_weight, eps=w.eps) if gated else {}
    o1 = kda.kda_decode_ex(d1.q, d1.k, d1.v, d1.state, d1.slot_idx, g=d1.g, beta=d1.beta, **extra1)
    o2 = kda.kda_decode_ex(q, k, v, d2.state, d2.slot_idx, g=d2.g, beta=d2.beta, **extra2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(d1.state, d2.state)
    before = w.to(cuda_device).state
    assert_parity(w, o2, d2.state, before)


# ---------------------------------------------------------------------------
# pipelined host steps (kda_decode_host_pipelined)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["n32_t1_hv8", "n32_t1_hv16_gated", "n8_t4_hv8"])
def test_host_pipeline_equals_device_calls(name, cuda_device):
    """Four steps through two alternating staging sets, copies in on a second
    stream, equal four device calls on the same inputs bit for bit (outputs read
    from pinned host memory, final state)."""
    w = workloads.config(name)
    steps_in = [workloads.config(name, seed=60 + i) for i in range(4)]
    for x in steps_in:
        x.slot_idx.copy_(w.slot_idx)
    d_ref = w.to(cuda_device)
    pool = d_ref.state.clone()
    stream = torch.cuda.Stream(device=cuda_device)
    copy_stream = torch.cuda.Stream(device=cuda_device)
    sets = []
    for _ in range(2):
        inputs = {k: t for k, t in w.tensors().items() if k != "state"}
        nbytes = sum((t.numel() * t.element_size() + 15) // 16 * 16 for t in inputs.values())
        host_in = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        dev_in = torch.empty(nbytes, dtype=torch.uint8, device=cuda_device)
        host_views, dev_views, off = {}, {}, 0
        for k, t in inputs.items():
            n = t.numel() * t.element_size()
            host_views[k] = host_in[off:off + n].view(t.dtype).view(t.shape)
            dev_views[k] = dev_in[off:off + n].view(t.dtype).view(t.shape)
            off += (n + 15) // 16 * 16
        out_d = torch.empty(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16, device=cuda_device)
        host_out = torch.empty(out_d.shape, dtype=torch.bfloat16).pin_memory()
        extra = dict(gate=dev_views["gate"], norm_weight=dev_views["norm_weight"], eps=w.eps) if w.gated else {}
        step = kda.HostStep(dev_views["q"], dev_views["k"], dev_views["v"], pool, dev_views["slot_idx"],
                            host_in=host_in, dev_in=dev_in, host_out=host_out, out=out_d, stream=stream,
                            g=dev_views["g"], beta=dev_views["beta"], scale=w.scale, **extra)
        sets.append((step, host_views, host_out))
    pipe = kda.HostPipeline([s[0] for s in sets], copy_stream)
    got = []
    for i, x in enumerate(steps_in):
        step, host_views, host_out = sets[i % 2]
        if i >= 2:  # the set's previous output must be read before it is reused
            stream.synchronize()
            got.append(host_out.clone())
        for k, t in x.tensors().items():
            if k != "state":
                host_views[k].copy_(t)
        pipe()
    stream.synchronize()
    got += [sets[0][2].clone(), sets[1][2].clone()]
    # reference: the same four steps as device calls
    for i, x in enumerate(steps_in):
        d = x.to(cuda_device)
        if w.gated:
            ref = kda.kda_decode_gated_rmsnorm(d.q, d.k, d.v, d.g, d.beta, d_ref.state, d.slot_idx, d.gate,
                                               d.norm_weight, eps=w.eps, scale=w.scale)
        else:
            ref = kda.kda_decode(d.q, d.k, d.v, d.g, d.beta, d_ref.state, d.slot_idx, scale=w.scale)
        torch.cuda.synchronize()
        assert torch.equal(got[i], ref.cpu()), f"step {i}: output differs"
    assert torch.equal(pool, d_ref.state)


# ---------------------------------------------------------------------------
# steps read from and written to mapped page-locked host memory (MappedStep)
# ---------------------------------------------------------------------------
def _pinned_views(tensors):
    nbytes = sum((t.numel() * t.element_size() + 15) // 16 * 16 for t in tensors.values())
    buf = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    views, off = {}, 0
    for key, t in tensors.items():
        n = t.numel() * t.element_size()
        views[key] = buf[off:off + n].view(t.dtype).view(t.shape)
        views[key].copy_(t)
        off += (n + 15) // 16 * 16
    return buf, views


@pytest.mark.parametrize("name", ["n32_t1_hv8", "n32_t1_hv16_gated", "n8_t4_hv8", "n32_t1_hv8_raw"])
def test_mapped_host_step_equals_device_call(name, cuda_device):
    """Inputs in page-locked host memory and the output written straight back
    to it by the kernel: bit-identical to the same step on device buffers.  The
    buffers are checked to be mapped at their host address before any launch."""
    w = workloads.config(name)
    inputs = {k: t for k, t in w.tensors().items() if k != "state"}
    host_in, hv = _pinned_views(inputs)
    out_h = torch.zeros(w.N, w.T, w.HV, w.V, dtype=torch.bfloat16).pin_memory()
    if not (kda.host_memory_is_mapped(host_in) and kda.host_memory_is_mapped(out_h)):
        pytest.skip("page-locked host memory is not mapped at its host address on this machine")
    pool = w.state.to(cuda_device)
    extra = dict(gate=hv["gate"], norm_weight=hv["norm_weight"], eps=w.eps) if w.gated else {}
    if w.raw is not None:
        extra.update(raw_gate=hv["raw_gate"], A_log=hv["A_log"], dt_bias=hv["dt_bias"], raw_beta=hv["raw_beta"])
    else:
        extra.update(g=hv["g"], beta=hv["beta"])
    step = kda.MappedStep(hv["q"], hv["k"], hv["v"], pool, hv["slot_idx"], host_in=host_in, out=out_h,
                          scale=w.scale, **extra)
    step()
    torch.cuda.synchronize()
    d = w.to(cuda_device)
    dextra = dict(gate=d.gate, norm_weight=d.norm_weight, eps=w.eps) if w.gated else {}
    if w.raw is not None:
        dextra.update(raw_gate=d.raw.raw_gate, A_log=d.raw.A_log, dt_bias=d.raw.dt_bias, raw_beta=d.raw.raw_beta)
    else:
        dextra.update(g=d.g, beta=d.beta)
    ref = kda.kda_decode_ex(d.q, d.k, d.v, d.state, d.slot_idx, scale=w.scale, **dextra)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu()) and torch.equal(pool, d.state)


def test_no_kernel_gave_up_a_bounded_wait(cuda_device):
    """The multi-token kernels' state-tile copy and the gated kernels' output
    hand-over end in bounded waits; after a plain, a gated and a multi-token
    call (and everything this file ran before) none of them gave up."""
    kda.device_error(clear=False)
    for name in ("n32_t4_hv8", "n32_t1_hv16_gated"):
        w = workloads.config(name).to(cuda_device)
        if w.gated:
            kda.kda_decode_gated_rmsnorm(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.gate, w.norm_weight,
                                         eps=w.eps, scale=w.scale)
        else:
            kda.kda_decode(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, scale=w.scale)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    assert kda.device_error() == 0
