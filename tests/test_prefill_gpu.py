"""Parity of the chunked prefill (``kda_prefill``, through the C ABI) with the
fp64 oracle.

The prefill computes the same recurrence as the decode step over all T tokens
of a call, so the oracle is the same token-by-token loop; outputs and states
are held to the decode step's tolerances (``tests/parity.py``): outputs within
1 bf16 ulp (and 2e-3 normwise), states within 1e-5 relative, untouched slots
bit-identical.  The shapes span one chunk, a ragged last chunk, many chunks,
inactive rows, the exact path taken for extreme decays, and the named prefill
workloads (the 8192-token prompt at full size).
"""
import os

import numpy as np
import pytest
import torch

import linear_attention_recurrent_decode_b200 as kda
import oracle
from linear_attention_recurrent_decode_b200 import workloads
from tests.parity import check_out, check_state

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))


def run_prefill(w, dev):
    d = w.to(dev)
    before = d.state.clone()
    o = kda.kda_prefill(d.q, d.k, d.v, d.g, d.beta, d.state, d.slot_idx, scale=w.scale)
    torch.cuda.synchronize()
    return o, d.state, before


def assert_prefill_parity(w, o, pool, before):
    ref_out, ref_state = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale,
                                               threads=THREADS)
    check_out(o.float().cpu().numpy(), ref_out)
    active = [s for s in w.slot_idx.tolist() if s >= 0]
    for s in active:
        check_state(pool[s].cpu().numpy(), ref_state[s], what=f"state slot {s}")
    untouched = [s for s in range(w.num_slots) if s not in active]
    if untouched:
        idx = torch.tensor(untouched, device=pool.device)
        assert torch.equal(pool[idx], before[idx]), "an untouched slot changed"


@pytest.mark.parametrize("N,T,HV,inactive,decay", [
    (1, 1, 2, 0, "softplus"),      # a single token: one chunk holding one row
    (1, 63, 2, 0, "softplus"),     # one ragged chunk
    (2, 64, 3, 0, "softplus"),     # exactly one chunk
    (3, 130, 2, 1, "softplus"),    # three chunks, the last ragged, an inactive row
    (2, 257, 4, 0, "uniform"),     # five chunks, mild decays (exp(g) in [0.5, 1))
    (4, 200, 1, 2, "softplus"),    # two inactive rows
    (3, 130, 4, 1, "softplus"),    # 12 heads: the state chain's 16-column tiles
    (4, 100, 6, 0, "softplus"),    # 24 heads: 32-column tiles
    (5, 96, 8, 1, "uniform"),      # 40 heads: 64-column tiles of 512 threads
])
def test_prefill_shapes(N, T, HV, inactive, decay, cuda_device):
    w = workloads.make(N=N, T=T, HV=HV, num_slots=N + 2, seed=300 + T + N, inactive=inactive, decay=decay)
    o, pool, before = run_prefill(w, cuda_device)
    assert_prefill_parity(w, o, pool, before)


@pytest.mark.parametrize("name", sorted(workloads.PREFILL_CONFIGS))
def test_prefill_named_workloads(name, cuda_device):
    """Every named prefill workload at full size, element by element."""
    w = workloads.config(name)
    o, pool, before = run_prefill(w, cuda_device)
    assert_prefill_parity(w, o, pool, before)


def test_prefill_extreme_decay_takes_the_exact_path(cuda_device):
    """Channels that decay by e^-3 per token exceed the factored path's range
    within half a chunk; those chunks take the exact path and still match."""
    w = workloads.make(N=2, T=150, HV=2, num_slots=4, seed=333)
    w.g[:, :, :, :16] = -3.0
    w.g[0, 70:90, 1, 40:48] = -6.0
    o, pool, before = run_prefill(w, cuda_device)
    assert_prefill_parity(w, o, pool, before)


def test_prefill_equals_decode_calls(cuda_device):
    """The prefill and the decode kernel compute the same recurrence: a prefill
    over T tokens and one decode call over the same T tokens agree to fp32
    rounding (both are checked against the oracle elsewhere)."""
    w = workloads.make(N=2, T=96, HV=2, num_slots=3, seed=341)
    d1, d2 = w.to(cuda_device), w.to(cuda_device)
    o1 = kda.kda_prefill(d1.q, d1.k, d1.v, d1.g, d1.beta, d1.state, d1.slot_idx)
    o2 = kda.kda_decode(d2.q, d2.k, d2.v, d2.g, d2.beta, d2.state, d2.slot_idx)
    torch.cuda.synchronize()
    diff = (o1.float() - o2.float()).abs()
    assert float(diff.max()) <= float(o2.float().abs().max()) * 2 ** -7
    for s in w.slot_idx.tolist():
        a, b = d1.state[s].double(), d2.state[s].double()
        assert float((a - b).norm() / b.norm()) < 2e-6


def test_prefill_back_to_back_calls_continue_the_state(cuda_device):
    """Two prefills of T1 and T2 tokens equal one of T1 + T2 tokens (the state
    written back by the first is the second's start state)."""
    w = workloads.make(N=2, T=160, HV=2, num_slots=3, seed=351)
    d = w.to(cuda_device)
    ws = torch.empty(kda.prefill_workspace_bytes(2, 160, 2), dtype=torch.uint8, device=cuda_device)
    o_a = kda.kda_prefill(d.q[:, :70].contiguous(), d.k[:, :70].contiguous(), d.v[:, :70].contiguous(),
                          d.g[:, :70].contiguous(), d.beta[:, :70].contiguous(), d.state, d.slot_idx, workspace=ws)
    o_b = kda.kda_prefill(d.q[:, 70:].contiguous(), d.k[:, 70:].contiguous(), d.v[:, 70:].contiguous(),
                          d.g[:, 70:].contiguous(), d.beta[:, 70:].contiguous(), d.state, d.slot_idx, workspace=ws)
    torch.cuda.synchronize()
    ref_out, ref_state = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale)
    check_out(torch.cat([o_a, o_b], dim=1).float().cpu().numpy(), ref_out)
    for s in w.slot_idx.tolist():
        check_state(d.state[s].cpu().numpy(), ref_state[s])


def test_prefill_stages_in_order_equal_one_call(cuda_device):
    """kda_prefill_stage 0, 1, 2 on one stream compute exactly what kda_prefill
    does (the same kernels with the same launch shapes): bit-identical outputs
    and final states."""
    w = workloads.make(N=3, T=150, HV=4, num_slots=5, seed=371, inactive=1)
    a, b = w.to(cuda_device), w.to(cuda_device)
    ws = torch.empty(kda.prefill_workspace_bytes(3, 150, 4), dtype=torch.uint8, device=cuda_device)
    o_all = kda.kda_prefill(a.q, a.k, a.v, a.g, a.beta, a.state, a.slot_idx, scale=w.scale, workspace=ws)
    ws2 = torch.empty_like(ws)
    o_st = torch.empty_like(o_all)
    for stage in (0, 1, 2):
        kda.kda_prefill(b.q, b.k, b.v, b.g, b.beta, b.state, b.slot_idx, out=o_st, scale=w.scale, workspace=ws2,
                        stage=stage)
    torch.cuda.synchronize()
    assert torch.equal(o_all, o_st)
    assert torch.equal(a.state, b.state)
    with pytest.raises(kda.KdaError):
        kda.kda_prefill(b.q, b.k, b.v, b.g, b.beta, b.state, b.slot_idx, out=o_st, workspace=ws2, stage=3)


def test_prefill_rejections(cuda_device):
    w = workloads.make(N=2, T=70, HV=2, num_slots=3, seed=361)
    d = w.to(cuda_device)
    lib = kda.library()
    need = kda.prefill_workspace_bytes(2, 70, 2)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    out = torch.empty(2, 70, 2, 128, dtype=torch.bfloat16, device=cuda_device)

    def call(K=128, V=128, wsb=need, out_ptr=None, ws_ptr=None):
        return lib.kda_prefill(d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), d.g.data_ptr(), d.beta.data_ptr(),
                               d.state.data_ptr(), d.slot_idx.data_ptr(), out_ptr or out.data_ptr(),
                               ws_ptr or ws.data_ptr(), wsb, 2, 70, 2, K, V, 0.1, None)

    assert call(K=64) == kda.KDA_ERR_UNSUPPORTED
    assert call(V=96) == kda.KDA_ERR_UNSUPPORTED
    assert call(wsb=need - 16) == kda.KDA_ERR_INVALID_ARG
    assert call(out_ptr=d.q.data_ptr()) == kda.KDA_ERR_ALIAS
    assert call(ws_ptr=out.data_ptr()) == kda.KDA_ERR_ALIAS
    assert call(ws_ptr=ws.data_ptr() + 8) == kda.KDA_ERR_MISALIGNED
    assert lib.kda_prefill_workspace_bytes(2, 70, 2, 64, 128) == -1
    assert lib.kda_prefill_workspace_bytes(0, 70, 2, 128, 128) == 0
    torch.cuda.synchronize()
    assert np.array_equal(d.state.cpu().numpy(), w.state.numpy()), "a rejected call touched the pool"
