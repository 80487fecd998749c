"""Pins for the fp64 oracle, each against something other than the oracle.

Sources ("page" = the web page the passage sits on):
  * KDA recurrence and gate: "NLP--技术报告解读-Kimi-K3" (joezjh.github.io),
    Model Architecture > Kimi Delta Attention (KDA): state-update equation,
    Lower-bounded decay equation (g_min = -5, alpha > e^-5).
  * Forgetting bound printed as "at most 99.33% per step": "Kimi K3 技术报告 ·
    大白话版" (CSDN), 2.1.1 KDA, improvement one.
  * KCP decomposition S = S~ + M S_prev: the joezjh.github.io page,
    Infrastructure > KDA Context Parallelism (KCP) equation.

Each pin is chosen so that a plausible slip in the oracle (decay after the
write, a missing beta, a transposed state, o read before the update, a sign
error in the delta term, a wrong gate sign or scale) fails at least one.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import expit

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_inputs(rng, B, T, H, dk, dv, g_scale=1.0):
    q = _unit_rows(rng.standard_normal((B, T, H, dk)))
    k = _unit_rows(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    g = -g_scale * rng.uniform(0.0, 5.0, size=(B, T, H, dk))
    beta = rng.uniform(0.05, 0.95, size=(B, T, H))
    return q, k, v, g, beta


# ----------------------------------------------------------------- gate pins

def test_gate_matches_library_sigmoid(oracle_mod):
    """g = g_min * Sigmoid(e^{A_h} z) against scipy's expit (library routine)."""
    rng = _rng(1)
    z = rng.standard_normal((5, 3, 7))
    A_log = np.log(rng.uniform(1.0, 16.0, size=3))
    g = oracle_mod.gate(z, A_log, -5.0)
    ref = -5.0 * expit(np.exp(A_log)[None, :, None] * z)
    np.testing.assert_allclose(g, ref, rtol=1e-14, atol=0)


def test_gate_special_values(oracle_mod):
    """Sigmoid(0) = 1/2; saturation at g_min and at 0; A_log rescales z."""
    z = np.array([[[0.0, 60.0, -60.0, 1.0]]])
    g = oracle_mod.gate(z, np.array([0.0]), -5.0)[0, 0]
    assert g[0] == -2.5
    assert abs(g[1] - (-5.0)) < 1e-20
    assert g[2] < 0 and g[2] > -1e-24
    g2 = oracle_mod.gate(np.array([[[2.0]]]), np.array([0.0]), -5.0)
    g1 = oracle_mod.gate(np.array([[[1.0]]]), np.array([math.log(2.0)]), -5.0)
    assert abs(g1[0, 0, 0] - g2[0, 0, 0]) < 1e-15


def test_gate_lower_bound_and_printed_forgetting(oracle_mod):
    """alpha = e^g >= e^-5 on the workloads' distribution, i.e. at most
    1 - e^-5 = 99.33% of a channel is forgotten per step, the figure the
    CSDN page prints (golden fixture)."""
    with open(os.path.join(GOLDEN, "forgetting_bound.txt")) as f:
        rows = dict(line.split("=", 1) for line in f.read().split("\n")
                    if line and not line.startswith("#"))
    g_min = float(rows["g_min"])
    printed_pct = float(rows["max_forgotten_percent"])
    rng = _rng(2)
    z = rng.standard_normal((64, 8, 32))
    A_log = np.log(rng.uniform(1.0, 16.0, size=8))
    g = oracle_mod.gate(z, A_log, g_min)
    assert np.all(g >= g_min) and np.all(g < 0)
    alpha = np.exp(g)
    assert np.all(alpha >= math.exp(g_min))
    worst_pct = 100.0 * (1.0 - math.exp(g_min))
    assert round(worst_pct, 2) == printed_pct
    assert np.all(100.0 * (1.0 - alpha) <= worst_pct + 1e-12)


# ------------------------------------------------------------ recurrence pins

def test_one_step_from_zero(oracle_mod):
    """S_0 = 0: S_1 = beta k v^T and o_1 = beta (k.q) v, whatever alpha is."""
    rng = _rng(3)
    q, k, v, g, beta = _rand_inputs(rng, 1, 1, 2, 6, 5)
    o, S = oracle_mod.forward(q, k, v, g, beta)
    for h in range(2):
        kk, vv, qq, bb = k[0, 0, h], v[0, 0, h], q[0, 0, h], beta[0, 0, h]
        np.testing.assert_allclose(S[0, h], bb * np.outer(kk, vv), rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(o[0, 0, h], bb * (kk @ qq) * vv, rtol=1e-13, atol=1e-15)


def test_delta_identity(oracle_mod):
    """alpha = 1, beta = 1, |k| = 1: S_t^T k_t = v_t for every t, from any
    starting state (erase what the memory predicts, then write)."""
    rng = _rng(4)
    T, H, dk, dv = 9, 2, 7, 4
    k = _unit_rows(rng.standard_normal((1, T, H, dk)))
    v = rng.standard_normal((1, T, H, dv))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, _ = oracle_mod.forward(k, k, v, np.zeros_like(k), np.ones((1, T, H)),
                              init_state=S0)
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)


def test_beta_zero_invariants(oracle_mod):
    """beta = 0: S_t = Diag(prod alpha) S_0 and o_t = S_t^T q_t; with alpha = 1
    too, the state is unchanged bit for bit."""
    rng = _rng(5)
    B, T, H, dk, dv = 2, 6, 2, 5, 3
    q, k, v, g, _ = _rand_inputs(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    zeros = np.zeros((B, T, H))
    o, S = oracle_mod.forward(q, k, v, g, zeros, init_state=S0)
    decay = np.exp(np.cumsum(g, axis=1))  # [B, T, H, dk]
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(S[b, h], decay[b, -1, h][:, None] * S0[b, h],
                                       rtol=1e-13, atol=1e-300)
            for t in range(T):
                St = decay[b, t, h][:, None] * S0[b, h]
                np.testing.assert_allclose(o[b, t, h], St.T @ q[b, t, h], rtol=1e-12,
                                           atol=1e-14)
    o1, S1 = oracle_mod.forward(q, k, v, np.zeros_like(g), zeros, init_state=S0)
    assert np.array_equal(S1, S0)


def _brute_force(q, k, v, g, beta, S0, scale):
    """Dense-matrix product form, written from the pages' equation:
    S_t = P_t S_{t-1} + beta_t k_t v_t^T with P_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
    and the expanded sum S_T = P_T..P_1 S_0 + sum_s P_T..P_{s+1} beta_s k_s v_s^T."""
    T, dk = k.shape
    P = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t]))
         for t in range(T)]
    outs = []
    for t in range(T):
        # expanded form of S_t, not a recurrence
        prod = np.eye(dk)
        for u in range(t, -1, -1):
            prod = prod @ P[u]
        St = prod @ S0
        for s in range(t + 1):
            tail = np.eye(dk)
            for u in range(t, s, -1):
                tail = tail @ P[u]
            St = St + tail @ (beta[s] * np.outer(k[s], v[s]))
        outs.append(scale * St.T @ q[t])
    return np.array(outs), St


@pytest.mark.parametrize("dk,dv,T", [(1, 1, 5), (3, 2, 7), (8, 8, 12), (6, 4, 1)])
def test_brute_force_product_form(oracle_mod, dk, dv, T):
    rng = _rng(10 + dk * 13 + T)
    q, k, v, g, beta = _rand_inputs(rng, 1, T, 1, dk, dv)
    k = k * rng.uniform(0.5, 1.5, size=(1, T, 1, 1))  # not unit-norm on purpose
    S0 = rng.standard_normal((1, 1, dk, dv))
    scale = 0.7
    o, S = oracle_mod.forward(q, k, v, g, beta, init_state=S0, scale=scale)
    ref_o, ref_S = _brute_force(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0],
                                beta[0, :, 0], S0[0, 0], scale)
    np.testing.assert_allclose(o[0, :, 0], ref_o, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], ref_S, rtol=1e-11, atol=1e-13)


def test_kcp_linearity_and_split(oracle_mod):
    """oracle(S_0) = oracle(0) + M S_0 with M the segment transition (the
    recurrence run on zero values from the identity), and running T1 then T2
    with the state handed over equals running T1+T2."""
    rng = _rng(6)
    T, H, dk, dv = 11, 2, 5, 4
    q, k, v, g, beta = _rand_inputs(rng, 1, T, H, dk, dv, g_scale=0.3)
    S0 = rng.standard_normal((1, H, dk, dv))
    o_full, S_full = oracle_mod.forward(q, k, v, g, beta, init_state=S0)
    _, S_zero = oracle_mod.forward(q, k, v, g, beta)
    eye = np.broadcast_to(np.eye(dk), (1, H, dk, dk)).copy()
    _, M = oracle_mod.forward(q, k, np.zeros((1, T, H, dk)), g, beta, init_state=eye)
    for h in range(H):
        np.testing.assert_allclose(S_full[0, h], S_zero[0, h] + M[0, h] @ S0[0, h],
                                   rtol=1e-12, atol=1e-13)
    t1 = 4
    sl = lambda a, s: a[:, s]
    o1, S1 = oracle_mod.forward(*(sl(a, slice(0, t1)) for a in (q, k, v, g, beta)),
                                init_state=S0)
    o2, S2 = oracle_mod.forward(*(sl(a, slice(t1, T)) for a in (q, k, v, g, beta)),
                                init_state=S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o_full, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S2, S_full, rtol=1e-13, atol=1e-14)


def test_orthonormal_key_recall(oracle_mod):
    """Orthonormal keys with alpha = 1, beta = 1: after t writes, S_t^T k_i = v_i
    for every i <= t (a textbook property of the delta rule)."""
    rng = _rng(7)
    dk, dv = 8, 3
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q.T[:6]  # 6 orthonormal rows
    T = keys.shape[0]
    v = rng.standard_normal((1, T, 1, dv))
    k = keys.reshape(1, T, 1, dk)
    _, S = oracle_mod.forward(k, k, v, np.zeros_like(k), np.ones((1, T, 1)))
    for i in range(T):
        np.testing.assert_allclose(S[0, 0].T @ keys[i], v[0, i, 0], rtol=1e-12, atol=1e-12)


def test_scalar_case_closed_form(oracle_mod):
    """dk = dv = 1: s_t = (1 - beta k^2) alpha s_{t-1} + beta k v, whose solution
    is s_T = (prod c) s_0 + sum_s (prod_{u>s} c_u) beta_s k_s v_s."""
    rng = _rng(8)
    T = 10
    k = rng.uniform(-1.2, 1.2, size=(1, T, 1, 1))
    q = rng.standard_normal((1, T, 1, 1))
    v = rng.standard_normal((1, T, 1, 1))
    g = -rng.uniform(0, 3, size=(1, T, 1, 1))
    beta = rng.uniform(0, 1, size=(1, T, 1))
    s0 = rng.standard_normal((1, 1, 1, 1))
    o, S = oracle_mod.forward(q, k, v, g, beta, init_state=s0)
    c = (1 - beta[0, :, 0] * k[0, :, 0, 0] ** 2) * np.exp(g[0, :, 0, 0])
    w = beta[0, :, 0] * k[0, :, 0, 0] * v[0, :, 0, 0]
    for t in range(T):
        st = np.prod(c[: t + 1]) * s0[0, 0, 0, 0] + sum(
            np.prod(c[s + 1: t + 1]) * w[s] for s in range(t + 1))
        assert abs(o[0, t, 0, 0] - st * q[0, t, 0, 0]) < 1e-12 * (1 + abs(st))
    assert abs(S[0, 0, 0, 0] - st) < 1e-12 * (1 + abs(st))


def test_output_scale_and_varlen_packing(oracle_mod):
    """o is linear in scale; a packed varlen batch equals separate runs, and a
    zero-length sequence returns its initial state unchanged."""
    rng = _rng(9)
    lens = [5, 0, 3, 7]
    T = sum(lens)
    H, dk, dv = 2, 4, 3
    q, k, v, g, beta = _rand_inputs(rng, 1, T, H, dk, dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    o, S = oracle_mod.forward(q, k, v, g, beta, init_state=S0, cu_seqlens=cu, scale=2.0)
    o1, _ = oracle_mod.forward(q, k, v, g, beta, init_state=S0, cu_seqlens=cu, scale=1.0)
    np.testing.assert_allclose(o, 2.0 * o1, rtol=1e-15, atol=0)
    for n, L in enumerate(lens):
        a, b = cu[n], cu[n + 1]
        if L == 0:
            assert np.array_equal(S[n], S0[n])
            continue
        on, Sn = oracle_mod.forward(*(x[:, a:b] for x in (q, k, v, g, beta)),
                                    init_state=S0[n:n + 1], scale=2.0)
        np.testing.assert_allclose(o[:, a:b], on, rtol=1e-15, atol=0)
        np.testing.assert_allclose(S[n], Sn[0], rtol=1e-15, atol=0)


def test_unit_subset_matches_full(oracle_mod):
    rng = _rng(11)
    q, k, v, g, beta = _rand_inputs(rng, 3, 6, 4, 5, 3)
    o, S = oracle_mod.forward(q, k, v, g, beta)
    units = [(2, 1), (0, 3)]
    os_, Ss = oracle_mod.forward(q, k, v, g, beta, units=units)
    for n, h in units:
        assert np.array_equal(os_[n, :, h], o[n, :, h])
        assert np.array_equal(Ss[n, h], S[n, h])
    assert np.isnan(os_[1, :, 0]).all()
