"""The seeded input generators (CPU): shapes, determinism, layouts and the
packed-row views the serving-form tests and the bench rely on."""
import math

import pytest
import torch

from linear_attention_recurrent_decode_b200 import workloads


def test_same_seed_same_draw_other_seed_other_draw():
    a = workloads.make(N=3, T=2, HV=2, K=64, V=64, seed=5)
    b = workloads.make(N=3, T=2, HV=2, K=64, V=64, seed=5)
    c = workloads.make(N=3, T=2, HV=2, K=64, V=64, seed=6)
    for key, t in a.tensors().items():
        assert torch.equal(t, b.tensors()[key]), key
    assert not torch.equal(a.q, c.q)


def test_shapes_dtypes_and_ranges():
    w = workloads.make(N=4, T=3, HV=2, K=128, V=96, num_slots=9, gated=True, seed=1, inactive=1)
    assert w.q.shape == w.k.shape == (4, 3, 2, 128) and w.v.shape == (4, 3, 2, 96)
    assert w.q.dtype == w.k.dtype == w.v.dtype == torch.bfloat16
    assert w.g.dtype == w.beta.dtype == w.state.dtype == torch.float32
    assert w.state.shape == (9, 2, 128, 96)
    assert bool((w.g < 0).all()) and bool(((w.beta > 0) & (w.beta < 1)).all())
    norms = w.k.float().norm(dim=-1)
    assert torch.allclose(norms, torch.ones_like(norms), atol=2e-2)  # L2-normalised before the bf16 rounding
    assert w.slot_idx[-1] == -1 and len(set(w.slot_idx[:-1].tolist())) == 3
    assert w.scale == pytest.approx(1 / math.sqrt(128))


def test_vk_layout_is_the_same_draw_transposed():
    kv = workloads.make(N=2, T=1, HV=3, K=64, V=32, seed=3)
    vk = workloads.make(N=2, T=1, HV=3, K=64, V=32, seed=3, state_layout="vk")
    assert vk.state.shape == (kv.num_slots, 3, 32, 64) and vk.state.is_contiguous()
    assert torch.equal(vk.state_kv(), kv.state)
    with pytest.raises(ValueError):
        workloads.make(N=1, T=1, HV=1, state_layout="kk")


def test_bf16_pool_is_the_fp32_draw_rounded():
    f = workloads.make(N=2, T=1, HV=2, K=64, V=64, seed=4)
    b = workloads.make(N=2, T=1, HV=2, K=64, V=64, seed=4, state_dtype="bf16")
    assert b.state.dtype == torch.bfloat16 and torch.equal(b.state, f.state.to(torch.bfloat16))


def test_serving_form_replaces_g_and_beta():
    w = workloads.make(N=2, T=3, HV=4, K=64, V=64, seed=2, serving=True)
    assert w.g is None and w.beta is None and w.packed
    t = w.tensors()
    assert "g" not in t and "beta" not in t
    assert t["raw_gate"].shape == (2, 3, 4, 64) and t["raw_gate"].dtype == torch.bfloat16
    assert t["A_log"].shape == (4,) and t["dt_bias"].shape == (4, 64) and t["raw_beta"].shape == (2, 3, 4)
    # dt_bias = softplus^-1(dt) with dt in [0.001, 0.1)
    dt = torch.nn.functional.softplus(t["dt_bias"].double())
    assert bool(((dt >= 0.001 - 1e-9) & (dt < 0.1 + 1e-9)).all())


def test_pack_rows_views_hold_the_parts_with_a_padded_row_stride():
    w = workloads.make(N=3, T=2, HV=2, K=64, V=32, seed=8)
    buf, (q, k, v) = workloads.pack_rows([w.q, w.k, w.v], pad=8)
    width = 2 * 64 + 2 * 64 + 2 * 32
    assert buf.shape == (3, 2, width + 8)
    assert torch.equal(q, w.q) and torch.equal(k, w.k) and torch.equal(v, w.v)
    assert q.stride(1) == k.stride(1) == v.stride(1) == width + 8
    assert k.data_ptr() - q.data_ptr() == 2 * 64 * 2 and v.data_ptr() - k.data_ptr() == 2 * 64 * 2


def test_named_configs_draw():
    for name in workloads.CONFIGS:
        if name.startswith("n256"):
            continue  # 2 GiB pools: drawn by the GPU tests and the bench
        w = workloads.config(name)
        assert w.name == name and w.q.shape[:3] == (w.N, w.T, w.HV)
