"""Pins of the fp64 oracle to facts other than itself.

Each test holds the oracle to something the pages or the mathematics fix:
closed forms of special cases, invariants of the delta rule, exact retrieval
from orthonormal keys, a hand-worked K=V=4 case (tests/golden), and library
routines (numpy matmul, scipy's expit) where a special case reduces to one.
The cases are chosen so that a plausible slip in the oracle -- a dropped
decay, decaying columns instead of key rows, the readout taken before the
update, a sign error in the correction, a wrong token/head stride, sigmoid(-z),
eps outside the square root -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from linear_attention_recurrent_decode_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def bf16_exact(x):
    """bf16 tensor holding x, asserting x is exactly representable."""
    t = bf16(x)
    assert np.array_equal(t.float().numpy(), np.asarray(x, dtype=np.float32)), "not bf16-exact"
    return t


def bf16_vals(t):
    return t.float().numpy().astype(np.float64)


def rand_case(N=2, T=3, HV=2, K=8, V=8, num_slots=5, seed=0, state_std=0.5):
    w = workloads.make(N=N, T=T, HV=HV, K=K, V=V, num_slots=num_slots, seed=seed,
                       state_std=state_std)
    return w


def run(w, **kw):
    return oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale, **kw)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def test_beta0_g0_leaves_state_and_reads_out_library_matmul():
    w = rand_case(T=2)
    w.beta.zero_()
    w.g.zero_()
    out, st = run(w)
    s0 = w.state.double().numpy()
    assert np.array_equal(st, s0), "beta=0, g=0 must leave the state bit-identical"
    q = bf16_vals(w.q)
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            for t in range(w.T):
                ref = w.scale * (s0[slot, h].T @ q[n, t, h])
                np.testing.assert_allclose(out[n, t, h], ref, rtol=1e-13, atol=1e-15)


def test_beta0_decay_closed_form_over_steps():
    """beta=0: S_T = Diag(exp(sum_t g_t)) S_0, and o_t reads Diag(exp(sum_{<=t} g)) S_0."""
    w = rand_case(T=5, K=6, V=7)
    w.beta.zero_()
    out, st = run(w)
    s0 = w.state.double().numpy()
    g = w.g.double().numpy()
    q = bf16_vals(w.q)
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            cum = np.zeros(w.K)
            for t in range(w.T):
                cum = cum + g[n, t, h]
                st_t = np.exp(cum)[:, None] * s0[slot, h]
                np.testing.assert_allclose(out[n, t, h], w.scale * (st_t.T @ q[n, t, h]),
                                           rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(st[slot, h], np.exp(cum)[:, None] * s0[slot, h],
                                       rtol=1e-12, atol=1e-300)


def test_single_step_from_zero_state():
    """S=0: S = beta k v^T and o = scale beta (q.k) v."""
    w = rand_case(T=1, K=8, V=5)
    w.state.zero_()
    out, st = run(w)
    q, k, v = bf16_vals(w.q), bf16_vals(w.k), bf16_vals(w.v)
    b = w.beta.double().numpy()
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            np.testing.assert_allclose(st[slot, h], b[n, 0, h] * np.outer(k[n, 0, h], v[n, 0, h]),
                                       rtol=1e-14, atol=1e-300)
            np.testing.assert_allclose(
                out[n, 0, h], w.scale * b[n, 0, h] * np.dot(q[n, 0, h], k[n, 0, h]) * v[n, 0, h],
                rtol=1e-13, atol=1e-300)


def test_delta_rule_write_invariant():
    """For any S, g, beta: S_new^T k = (1 - beta |k|^2) S'^T k + beta |k|^2 v with S' the decayed
    state; in particular beta = 1 and |k| = 1 store v exactly under key k."""
    w = rand_case(T=1, K=8, V=6, N=3, HV=2, num_slots=3)
    out, st = run(w)
    s0 = w.state.double().numpy()
    g = w.g.double().numpy()
    k, v = bf16_vals(w.k), bf16_vals(w.v)
    b = w.beta.double().numpy()
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            sp = np.exp(g[n, 0, h])[:, None] * s0[slot, h]
            kk = np.dot(k[n, 0, h], k[n, 0, h])
            lhs = st[slot, h].T @ k[n, 0, h]
            rhs = (1 - b[n, 0, h] * kk) * (sp.T @ k[n, 0, h]) + b[n, 0, h] * kk * v[n, 0, h]
            np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-14)

    # beta = 1 with an exactly unit key (four entries of 1/2): the write is exact.
    K, V = 8, 6
    key = bf16_exact([0.5, 0, 0.5, 0, 0.5, 0, 0.5, 0]).reshape(1, 1, 1, K)
    val = bf16(RNG.standard_normal(V)).reshape(1, 1, 1, V)
    state = torch.as_tensor(RNG.standard_normal((1, 1, K, V)), dtype=torch.float32)
    g1 = torch.as_tensor(-np.abs(RNG.standard_normal((1, 1, 1, K))), dtype=torch.float32)
    out, st = oracle.kda_decode_ref(key, key, val, g1, torch.ones(1, 1, 1), state,
                                    torch.zeros(1, dtype=torch.int32), 1.0)
    np.testing.assert_allclose(st[0, 0].T @ bf16_vals(key)[0, 0, 0], bf16_vals(val)[0, 0, 0],
                               rtol=0, atol=1e-14)
    # q = k: the readout returns exactly what was just written (readout after the update).
    np.testing.assert_allclose(out[0, 0, 0], bf16_vals(val)[0, 0, 0], rtol=0, atol=1e-14)


def test_orthonormal_keys_store_and_retrieve_exactly():
    """g=0, beta=1, S=0, keys = unit basis vectors: every stored v comes back exactly."""
    K, V, T = 6, 5, 6
    perm = RNG.permutation(K)
    keys = np.zeros((1, T, 1, K), np.float32)
    for t in range(T):
        keys[0, t, 0, perm[t]] = 1.0
    vals = bf16(RNG.standard_normal((1, T, 1, V)))
    # query the key stored two steps earlier (or the current one for t < 2)
    qs = np.zeros((1, T, 1, K), np.float32)
    for t in range(T):
        qs[0, t, 0, perm[max(0, t - 2)]] = 1.0
    out, st = oracle.kda_decode_ref(bf16_exact(qs), bf16_exact(keys), vals,
                                    torch.zeros(1, T, 1, K), torch.ones(1, T, 1),
                                    torch.zeros(1, 1, K, V), torch.zeros(1, dtype=torch.int32), 0.25)
    vv = bf16_vals(vals)
    for t in range(T):
        assert np.array_equal(out[0, t, 0], 0.25 * vv[0, max(0, t - 2), 0])
    for t in range(T):
        assert np.array_equal(st[0, 0, perm[t]], vv[0, t, 0])


def test_t_steps_equal_successive_single_steps():
    w = rand_case(T=4, N=3, HV=2, K=8, V=8, num_slots=6)
    out, st = run(w)
    state = w.state.double().numpy().copy()
    for t in range(w.T):
        sl = slice(t, t + 1)
        o1, state = oracle.kda_decode_ref(w.q[:, sl], w.k[:, sl], w.v[:, sl], w.g[:, sl],
                                          w.beta[:, sl], state, w.slot_idx, w.scale)
        assert np.array_equal(o1[:, 0], out[:, t])
    assert np.array_equal(state, st)


def test_units_are_independent_and_indexed_by_n_h_t():
    """The batched call equals one N=1, HV=1 call per (n, h) on explicitly sliced inputs."""
    w = rand_case(N=3, T=2, HV=3, K=4, V=6, num_slots=4)
    out, st = run(w)
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            sl = (slice(n, n + 1), slice(None), slice(h, h + 1))
            o1, s1 = oracle.kda_decode_ref(w.q[sl], w.k[sl], w.v[sl], w.g[sl], w.beta[n:n + 1, :, h:h + 1],
                                           w.state[slot:slot + 1, h:h + 1],
                                           torch.zeros(1, dtype=torch.int32), w.scale)
            assert np.array_equal(o1[0, :, 0], out[n, :, h])
            assert np.array_equal(s1[0, 0], st[slot, h])


def test_slot_mapping_untouched_and_inactive_rows():
    w = workloads.make(N=4, T=2, HV=2, K=4, V=4, num_slots=9, seed=3, inactive=1)
    out, st = run(w)
    s0 = w.state.double().numpy()
    active = {int(s) for s in w.slot_idx if s >= 0}
    for s in range(w.num_slots):
        if s not in active:
            assert np.array_equal(st[s], s0[s])
        else:
            assert not np.array_equal(st[s], s0[s])
    assert np.all(out[w.N - 1] == 0.0)
    # Permuting the rows together with their slots permutes the outputs.
    perm = torch.tensor([2, 0, 3, 1])
    out_p, st_p = oracle.kda_decode_ref(w.q[perm], w.k[perm], w.v[perm], w.g[perm], w.beta[perm],
                                        w.state, w.slot_idx[perm], w.scale)
    assert np.array_equal(out_p, out[perm.numpy()])
    assert np.array_equal(st_p, st)


def test_slot_out_of_range_is_rejected():
    w = rand_case(N=1, num_slots=1)
    w.slot_idx[0] = 1
    with pytest.raises(ValueError):
        run(w)


def test_threads_do_not_change_results():
    w = rand_case(N=5, T=2, HV=3, K=8, V=8, num_slots=7)
    o1, s1 = run(w)
    o2, s2 = run(w, threads=4)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


# ---------------------------------------------------------------------------
# hand-worked K = V = 4 case
# ---------------------------------------------------------------------------
def _golden():
    with open(os.path.join(GOLDEN, "kda_k4v4_hand.json")) as f:
        return json.load(f)


def _golden_inputs(c):
    T, K, V = c["T"], c["K"], c["V"]
    g = np.array(c["g"], np.float32)
    g[np.array(c["g_is_minus_ln2"])] = np.float32(-math.log(2.0))
    state = np.full((c["num_slots"], 1, K, V), c["other_slots_fill"], np.float32)
    state[c["slot_idx"][0], 0] = np.array(c["S0_slot2"], np.float32)
    q = bf16_exact(np.array(c["q"], np.float32).reshape(1, T, 1, K))
    k = bf16_exact(np.array(c["k"], np.float32).reshape(1, T, 1, K))
    v = bf16_exact(np.array(c["v"], np.float32).reshape(1, T, 1, V))
    return (q, k, v, torch.as_tensor(g.reshape(1, T, 1, K)),
            torch.as_tensor(np.array(c["beta"], np.float32).reshape(1, T, 1)),
            torch.as_tensor(state), torch.tensor(c["slot_idx"], dtype=torch.int32))


def test_hand_worked_k4v4():
    c = _golden()
    q, k, v, g, beta, state, slot = _golden_inputs(c)
    tol = c["tolerance_abs"]
    # one T=2 call
    out, st = oracle.kda_decode_ref(q, k, v, g, beta, state, slot, c["scale"])
    np.testing.assert_allclose(out[0, :, 0], np.array(c["o"]), rtol=0, atol=tol)
    np.testing.assert_allclose(st[2, 0], np.array(c["S2"]), rtol=0, atol=tol)
    assert np.all(st[:2] == c["other_slots_fill"])
    # the first token alone gives S1
    out1, st1 = oracle.kda_decode_ref(q[:, :1], k[:, :1], v[:, :1], g[:, :1], beta[:, :1], state, slot,
                                      c["scale"])
    np.testing.assert_allclose(st1[2, 0], np.array(c["S1"]), rtol=0, atol=tol)


def test_hand_worked_k4v4_gated():
    c = _golden()
    gc = c["gated"]
    q, k, v, g, beta, state, slot = _golden_inputs(c)
    z = bf16_exact(np.array(gc["z"], np.float32).reshape(1, c["T"], 1, c["V"]))
    wgt = bf16_exact(np.array(gc["norm_weight"], np.float32))
    out, st = oracle.kda_decode_ref(q, k, v, g, beta, state, slot, c["scale"],
                                    gate=z, norm_weight=wgt, eps=gc["eps"])
    exp_y = np.array(gc["y_numerators"]) / np.sqrt(np.array(gc["y_sqrt_denominators"], float))[:, None]
    np.testing.assert_allclose(out[0, :, 0], exp_y, rtol=0, atol=c["tolerance_abs"])
    np.testing.assert_allclose(st[2, 0], np.array(c["S2"]), rtol=0, atol=c["tolerance_abs"])


# ---------------------------------------------------------------------------
# gated RMS norm closed forms
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("eps", [1e-6, 0.5])
def test_gated_rank1_closed_form(eps):
    """S=0, one step: o = c v with c = scale beta (q.k), so
    y = c v / sqrt(c^2 mean(v^2) + eps) * w * sigmoid(z)."""
    w = workloads.make(N=2, T=1, HV=2, K=8, V=8, num_slots=3, gated=True, seed=5)
    w.state.zero_()
    out, _ = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale,
                                   gate=w.gate, norm_weight=w.norm_weight, eps=eps)
    q, k, v, z = bf16_vals(w.q), bf16_vals(w.k), bf16_vals(w.v), bf16_vals(w.gate)
    wt = bf16_vals(w.norm_weight)
    b = w.beta.double().numpy()
    for n in range(w.N):
        for h in range(w.HV):
            c = w.scale * b[n, 0, h] * np.dot(q[n, 0, h], k[n, 0, h])
            vv = v[n, 0, h]
            ref = c * vv / np.sqrt(c * c * np.mean(vv * vv) + eps) * wt * expit(z[n, 0, h])
            np.testing.assert_allclose(out[n, 0, h], ref, rtol=1e-12, atol=1e-15)


def test_gated_unit_gate_gives_unit_rms():
    """w = 1 and sigmoid(z) = 1 (z = 80 in bf16): mean(y^2) = ms / (ms + eps)."""
    w = workloads.make(N=2, T=3, HV=2, K=8, V=8, num_slots=3, gated=True, seed=6)
    z = torch.full_like(w.gate, 80.0)
    ones = torch.ones_like(w.norm_weight)
    eps = 1e-3
    y, st_y = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale,
                                    gate=z, norm_weight=ones, eps=eps)
    o, st_o = run(w)
    assert np.array_equal(st_y, st_o), "the norm must not touch the state"
    ms = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12)
    # and y is o scaled by a positive per-(n,t,h) factor
    ratio = y / o
    np.testing.assert_allclose(ratio, ratio[..., :1] * np.ones_like(ratio), rtol=1e-12)
    assert np.all(ratio > 0)


# ---------------------------------------------------------------------------
# bf16 state: the oracle's own rounding, and the state closed forms through it
# ---------------------------------------------------------------------------
def _bits_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def test_round_bf16_round_trip_and_ties():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 16, size=200_000, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    vals = _bits_to_f64(bits[finite])
    np.testing.assert_array_equal(oracle.round_bf16(vals), vals)  # exact values are kept
    # midpoints between neighbours round to the even neighbour, nudges go to the nearer one
    b = bits[finite & ((bits & 0x7FFF) < 0x7F7F) & ((bits & 0x7FFF) > 0)]
    lo, hi = _bits_to_f64(b), _bits_to_f64(b + 1)
    mid = (lo + hi) / 2
    even = np.where((b & 1) == 0, lo, hi)
    np.testing.assert_array_equal(oracle.round_bf16(mid), even)
    step = np.abs(hi - lo)
    np.testing.assert_array_equal(oracle.round_bf16(mid - step / 8 * np.sign(hi - lo)), lo)
    np.testing.assert_array_equal(oracle.round_bf16(mid + step / 8 * np.sign(hi - lo)), hi)


def test_round_bf16_matches_library_conversion():
    """torch's float64 -> bfloat16 conversion is an independent implementation
    of the same rounding, subnormals and overflow included.  It goes through
    float32, which double-rounds inputs whose float32 image is exactly a bf16
    midpoint; those (about 1 in 50,000) are left to the midpoint test above."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal(300_000) * np.exp2(rng.uniform(-140, 130, 300_000))
    x = np.concatenate([x, [0.0, -0.0, 3.3895313892515355e38, 3.3896e38, -3.5e38, 1e-45, 9.2e-41]])
    with np.errstate(over="ignore"):  # beyond the binary32 range the image is inf, never a midpoint
        f32_bits = x.astype(np.float32).view(np.uint32)
    single_rounding = (f32_bits & 0xFFFF) != 0x8000
    assert single_rounding.mean() > 0.999
    x = x[single_rounding]
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x), ref)


def test_bf16_state_closed_forms():
    """bf16 pool: beta=0, g=0 leaves it bit-identical; from S=0 one step stores
    round(beta k v^T)."""
    w = workloads.make(N=2, T=1, HV=2, K=8, V=8, num_slots=3, seed=9, state_dtype="bf16")
    w.beta.zero_()
    w.g.zero_()
    _, st = run(w)
    np.testing.assert_array_equal(st, w.state.double().numpy())
    w = workloads.make(N=2, T=1, HV=2, K=8, V=8, num_slots=3, seed=10, state_dtype="bf16")
    w.state.zero_()
    _, st = run(w)
    k, v = bf16_vals(w.k), bf16_vals(w.v)
    b = w.beta.double().numpy()
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            exact = b[n, 0, h] * np.outer(k[n, 0, h], v[n, 0, h])
            ref = torch.from_numpy(exact).to(torch.bfloat16).double().numpy()
            np.testing.assert_array_equal(st[slot, h], ref)


# ---------------------------------------------------------------------------
# raw gate / raw beta activation.  PARITY UNPINNED: the sources name the raw
# inputs (FlashInfer #4562's kernel launch passes raw_gate, A_log, dt_bias and
# raw_beta) but print no activation, so the formula the oracle uses is a
# reading.  What can be pinned without repeating that formula are properties
# any softplus-style decay gate and logistic beta must have; each slip the
# mutation tests plant in the activation breaks one of them.
# ---------------------------------------------------------------------------
def _activate_1head(raw, A_log=0.3, dt_bias=0.0, raw_beta=None):
    """Activate a 1-D sweep of raw gate values (one head, K = len(raw))."""
    raw = np.asarray(raw, dtype=np.float64)
    K = raw.size
    rb = np.zeros(1) if raw_beta is None else np.asarray(raw_beta, dtype=np.float64)
    g, beta = oracle.activate(bf16_exact(raw.reshape(1, 1, 1, K)), torch.tensor([A_log], dtype=torch.float32),
                              torch.full((1, K), dt_bias, dtype=torch.float32), bf16_exact(rb.reshape(1, 1, 1)))
    return g.reshape(K), float(beta.reshape(-1)[0])


def _bf16_grid(lo, hi, n):
    return np.unique(bf16(np.linspace(lo, hi, n)).float().numpy().astype(np.float64))


def test_activation_gate_is_a_nonpositive_nonincreasing_log_decay():
    """g <= 0 (a decay exp(g) never amplifies the state) and g does not
    increase as the raw gate grows (a larger raw gate forgets more)."""
    x = _bf16_grid(-60.0, 60.0, 4001)
    for A_log in (-2.0, 0.0, 1.5):
        g, _ = _activate_1head(x, A_log=A_log)
        assert np.all(np.isfinite(g)) and np.all(g <= 0.0)
        assert np.all(np.diff(g) <= 0.0)
        assert g[-1] < g[0]  # strictly forgets more at the top of the range


def test_activation_gate_limits():
    """raw gate -> -inf: g -> 0 (no decay); raw gate -> +inf: g is linear with
    slope -exp(A_log) (the rate per unit of raw gate is the head's A)."""
    for A_log in (-1.0, 0.0, 2.0):
        a = math.exp(float(np.float32(A_log)))
        g, _ = _activate_1head([-80.0, -60.0, 40.0, 64.0], A_log=A_log)
        assert abs(g[0]) < 1e-30 and abs(g[1]) < 1e-20
        slope = (g[3] - g[2]) / (64.0 - 40.0)
        assert slope == pytest.approx(-a, rel=1e-12)
        assert g[3] == pytest.approx(-a * 64.0, rel=1e-12)


def test_activation_dt_bias_shifts_the_raw_gate():
    """dt_bias adds to the raw gate before the nonlinearity: raw + b with bias 0
    equals raw with bias b (values chosen so raw + b is exact in bf16)."""
    raw = np.array([-3.0, -1.0, -0.5, 0.0, 0.25, 1.0, 2.0, 6.0])
    for b in (-1.5, 0.5, 2.0):
        shifted, _ = _activate_1head(raw + b, A_log=0.7, dt_bias=0.0)
        biased, _ = _activate_1head(raw, A_log=0.7, dt_bias=b)
        np.testing.assert_array_equal(biased, shifted)


def test_activation_beta_is_a_logistic_gate():
    """beta in (0, 1), increasing in the raw beta, beta(0) = 1/2 and
    beta(-x) = 1 - beta(x)."""
    xs = _bf16_grid(-12.0, 12.0, 97)
    betas = np.array([_activate_1head([0.0], raw_beta=[x])[1] for x in xs])
    assert np.all(betas > 0.0) and np.all(betas < 1.0)
    assert np.all(np.diff(betas) > 0.0)
    assert _activate_1head([0.0], raw_beta=[0.0])[1] == 0.5
    for x in xs:
        bp = _activate_1head([0.0], raw_beta=[x])[1]
        bm = _activate_1head([0.0], raw_beta=[-x])[1]
        assert bp + bm == pytest.approx(1.0, abs=1e-15)


def test_activation_feeds_the_recurrence():
    """The decode from raw inputs equals the decode from the activated g, beta."""
    w = workloads.make(N=2, T=2, HV=2, K=8, V=8, num_slots=3, seed=12)
    rng = np.random.default_rng(12)
    raw_gate = bf16(rng.standard_normal((2, 2, 2, 8)))
    raw_beta = bf16(rng.standard_normal((2, 2, 2)))
    A_log = torch.as_tensor(rng.standard_normal(2) - 1, dtype=torch.float32)
    dt_bias = torch.as_tensor(rng.standard_normal((2, 8)), dtype=torch.float32)
    g, beta = oracle.activate(raw_gate, A_log, dt_bias, raw_beta)
    o1, s1 = oracle.kda_decode_ref(w.q, w.k, w.v, g, beta, w.state, w.slot_idx, w.scale)
    # beta = 0 and g = 0 reached through the activation: raw_beta = -inf-ish, A_log -> -inf
    g0, b0 = oracle.activate(raw_gate, torch.full((2,), -200.0), dt_bias, bf16(np.full((2, 2, 2), -200.0)))
    assert np.all(np.abs(g0) < 1e-80) and np.all(b0 < 1e-80)
    o0, s0 = oracle.kda_decode_ref(w.q, w.k, w.v, g0, b0, w.state, w.slot_idx, w.scale)
    np.testing.assert_allclose(s0, w.state.double().numpy(), rtol=1e-12, atol=0)
    assert np.all(np.isfinite(o1)) and np.all(np.isfinite(s1))
