"""kda_prefill_no_alloc: the chunked prefill without a caller-provided
workspace, for callers that cannot allocate device memory (a serving process
whose allocator owns the GPU's memory, a framework plugin, code recording CUDA
graphs).  It runs the same kernels on a fixed scratch array inside the library.

Called through the C ABI and compared with kda_prefill (the entry point that
takes a workspace) on the same inputs, within the parity tolerances of the
other GPU tests, over two calls in a row (the second starts from the state the
first left, and reuses the scratch the first one wrote).  This file runs last:
it works alone in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import linear_attention_recurrent_decode_b200 as kda
from linear_attention_recurrent_decode_b200 import workloads
from tests.parity import check_out, check_state

pytestmark = pytest.mark.gpu


def _call_no_alloc(lib, d, out, N, T):
    return lib.kda_prefill_no_alloc(d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), d.g.data_ptr(),
                                    d.beta.data_ptr(), d.state.data_ptr(), d.slot_idx.data_ptr(), out.data_ptr(),
                                    N, T, d.HV, d.K, d.V, ctypes.c_float(d.scale), None)


def _call_with_workspace(lib, d, out, ws, N, T):
    return lib.kda_prefill(d.q.data_ptr(), d.k.data_ptr(), d.v.data_ptr(), d.g.data_ptr(), d.beta.data_ptr(),
                           d.state.data_ptr(), d.slot_idx.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(),
                           N, T, d.HV, d.K, d.V, ctypes.c_float(d.scale), None)


def test_no_alloc_prefill_matches_the_workspace_entry_point(cuda_device):
    lib = kda.library()
    # 1000 tokens at 8 heads (16 chunks each, a ragged last one) and a padding row
    first = workloads.make(N=2, T=1000, HV=4, num_slots=4, seed=501, inactive=1)
    second = workloads.make(N=2, T=300, HV=4, num_slots=4, seed=502)
    second.slot_idx.copy_(first.slot_idx)
    a1, b1 = first.to(cuda_device), first.to(cuda_device)   # a: no-alloc, b: workspace
    a2, b2 = second.to(cuda_device), second.to(cuda_device)
    b2.state = b1.state
    a2.state = a1.state
    ws = torch.empty(kda.prefill_workspace_bytes(2, 1000, 4), dtype=torch.uint8, device=cuda_device)
    outs = []
    for a, b, T in ((a1, b1, 1000), (a2, b2, 300)):
        oa = torch.empty(2, T, 4, 128, dtype=torch.bfloat16, device=cuda_device)
        ob = torch.empty_like(oa)
        assert _call_no_alloc(lib, a, oa, 2, T) == kda.KDA_OK
        assert _call_with_workspace(lib, b, ob, ws, 2, T) == kda.KDA_OK
        outs.append((oa, ob))
    torch.cuda.synchronize()
    for oa, ob in outs:
        check_out(oa.float().cpu().numpy(), ob.double().cpu().numpy(), what="no-alloc output")
    for s in first.slot_idx.tolist():
        if s >= 0:
            check_state(a1.state[s].cpu().numpy(), b1.state[s].double().cpu().numpy(), what=f"no-alloc state {s}")


def test_no_alloc_prefill_refuses_sizes_beyond_its_scratch(cuda_device):
    lib = kda.library()
    w = workloads.make(N=1, T=2048, HV=8, num_slots=2, seed=503)  # 256 chunks of workspace > 136
    d = w.to(cuda_device)
    before = d.state.clone()
    out = torch.zeros(1, 2048, 8, 128, dtype=torch.bfloat16, device=cuda_device)
    assert kda.prefill_workspace_bytes(1, 2048, 8) > (32 << 20)
    assert _call_no_alloc(lib, d, out, 1, 2048) == kda.KDA_ERR_SCRATCH_LIMIT
    assert kda.status_string(kda.KDA_ERR_SCRATCH_LIMIT).startswith("sizes need more scratch")
    torch.cuda.synchronize()
    assert torch.equal(d.state, before) and not out.any()
