"""The multi-token kernel's regrouping of the recurrence, checked in fp64 on the CPU.

The kernel takes tokens four at a time against the chunk-start state S0:
with d_t = exp(g_t), A_t = d_0 ... d_t, B(s->t) = d_{s+1} ... d_t,
    R_t = S0^T (A_t k_t),  Q_t = S0^T (A_t q_t),
    M[t][s] = sum_i k_s,i B(s->t)_i k_t,i (s < t),  P[t][s] = sum_i k_s,i B(s->t)_i q_t,i (s <= t),
    u_t = beta_t (v_t - R_t - sum_{s<t} M[t][s] u_s),
    o_t = scale (Q_t + sum_{s<=t} P[t][s] u_s),
    S_end = A_last S0 + sum_t (B(t->last) k_t) u_t^T.
This test evaluates exactly these formulas in numpy fp64 and compares them
with the oracle's token-by-token recurrence: equal to rounding, for ragged
last chunks and several chunks in a row.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrent_decode_b200 import workloads

CHUNK = 4


def chunked_reference(q, k, v, g, beta, S, scale):
    """One (n, h): q, k [T, K], v [T, V], g [T, K], beta [T], S [K, V] (fp64)."""
    T = q.shape[0]
    S = S.copy()
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, CHUNK):
        tc = min(CHUNK, T - c0)
        d = np.exp(g[c0:c0 + tc])                      # [tc, K]
        A = np.cumprod(d, axis=0)                      # A_t = d_0 ... d_t
        kk, qq = k[c0:c0 + tc], q[c0:c0 + tc]
        R = (A * kk) @ S                               # [tc, V]
        Q = (A * qq) @ S
        u = np.zeros((tc, v.shape[1]))
        for t in range(tc):
            x = v[c0 + t] - R[t]
            for s in range(t):
                B = np.prod(d[s + 1:t + 1], axis=0)    # B(s->t)
                x = x - np.sum(kk[s] * B * kk[t]) * u[s]
            u[t] = beta[c0 + t] * x
            o = Q[t].copy()
            for s in range(t + 1):
                B = np.prod(d[s + 1:t + 1], axis=0)
                o = o + np.sum(kk[s] * B * qq[t]) * u[s]
            out[c0 + t] = scale * o
        S_new = A[tc - 1][:, None] * S
        for t in range(tc):
            Bl = np.prod(d[t + 1:tc], axis=0)          # B(t->last)
            S_new = S_new + np.outer(Bl * kk[t], u[t])
        S = S_new
    return out, S


@pytest.mark.parametrize("T", [1, 3, 4, 5, 9, 12])
def test_chunked_regrouping_equals_the_recurrence(T):
    w = workloads.make(N=2, T=T, HV=2, K=16, V=8, num_slots=3, seed=90 + T, decay="uniform")
    ref_out, ref_state = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale)
    q = w.q.double().numpy()
    k = w.k.double().numpy()
    v = w.v.double().numpy()
    g = w.g.double().numpy()
    beta = w.beta.double().numpy()
    S0 = w.state.double().numpy()
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            out, S = chunked_reference(q[n, :, h], k[n, :, h], v[n, :, h], g[n, :, h], beta[n, :, h],
                                       S0[slot, h], w.scale)
            np.testing.assert_allclose(out, ref_out[n, :, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(S, ref_state[slot, h], rtol=1e-12, atol=1e-13)


def test_regrouping_check_sees_a_wrong_coupling():
    """The comparison above fails if a coupling term is dropped (here M)."""
    w = workloads.make(N=1, T=4, HV=1, K=16, V=8, num_slots=1, seed=99, decay="uniform")
    ref_out, _ = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale)
    q, k, v = (x.double().numpy()[0, :, 0] for x in (w.q, w.k, w.v))
    g, beta = w.g.double().numpy()[0, :, 0], w.beta.double().numpy()[0, :, 0]
    S0 = w.state.double().numpy()[0, 0]
    # same formulas without the M[t][s] u_s terms
    d = np.exp(g)
    A = np.cumprod(d, axis=0)
    R = (A * k) @ S0
    u = beta[:, None] * (v - R)
    o0 = w.scale * ((A[0] * q[0]) @ S0 + np.sum(k[0] * q[0]) * u[0])
    assert np.allclose(o0, ref_out[0, 0, 0])            # token 0 has no coupling
    wrong_o3 = w.scale * ((A[3] * q[3]) @ S0 + sum(np.sum(k[s] * np.prod(d[s + 1:4], axis=0) * q[3]) * u[s]
                                                   for s in range(4)))
    assert not np.allclose(wrong_o3, ref_out[0, 3, 0], rtol=1e-6)


def test_one_pass_readout_identity():
    """The one-token kernel reads out o = scale (S'^T q + (q . k) u) from the
    decayed state S' and the correction u, without a second pass over the
    updated state; in fp64 this equals the oracle's scale S^T q."""
    w = workloads.make(N=3, T=1, HV=2, K=32, V=16, num_slots=4, seed=77)
    ref_out, ref_state = oracle.kda_decode_ref(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx, w.scale)
    for n in range(w.N):
        slot = int(w.slot_idx[n])
        for h in range(w.HV):
            q, k, v = (x.double().numpy()[n, 0, h] for x in (w.q, w.k, w.v))
            g, beta = w.g.double().numpy()[n, 0, h], float(w.beta[n, 0, h])
            Sd = np.exp(g)[:, None] * w.state.double().numpy()[slot, h]     # S'
            u = beta * (v - Sd.T @ k)
            o = w.scale * (Sd.T @ q + float(q @ k) * u)
            np.testing.assert_allclose(o, ref_out[n, 0, h], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(Sd + np.outer(k, u), ref_state[slot, h], rtol=1e-12, atol=1e-14)
