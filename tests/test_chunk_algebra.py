"""fp64 check of the chunkwise algebra the CUDA kernels implement.

This is a test aid, not the oracle: a numpy restatement of the chunk form
(WY/UT representation) that the kernels use, compared with the sequential
fp64 oracle to ~1e-12.  It validates the derivation before any GPU runs:

Within a chunk of C tokens starting from state S (dk x dv), with
Gamma_r = sum_{s<=r} g_s (per channel) and gamma_r = exp(Gamma_r):
  L[r,s]   = sum_i k_ri k_si exp(Gamma_ri - Gamma_si)            (s <= r)
  A_kk     = Diag(beta) strict_lower(L)        A_qk = lower_incl(Q-version of L)
  T        = (I + A_kk)^-1 Diag(beta)
  W        = T (k * gamma)                      U~ = T V
  U        = U~ - W S                            (the delta-rule errors)
  O        = scale ((q * gamma) S + A_qk U)
  S_next   = Diag(gamma_C) S + (k * exp(Gamma_C - Gamma))^T U
The tensor-core kernel evaluates L with one rebasing point per 32-token
chunk (row 15): left operands x_r exp(Gamma_r - Gamma_15), right operand
k_s exp(Gamma_15 - Gamma_s); with g >= -5 every factor stays inside
[e^-80, e^80], so each Gram matrix is one GEMM.  The segment split used for
long sequences composes per-segment transitions (KCP form
S = S~ + M S_prev, "NLP--技术报告解读-Kimi-K3", Infrastructure > KCP).
"""
import numpy as np
import pytest


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def chunk_forward(q, k, v, g, beta, S0, C, scale=1.0, rebase="direct",
                  dtype=np.float64):
    """One (sequence, head): q,k,g [L,dk], v [L,dv], beta [L], S0 [dk,dv]."""
    L, dk = k.shape
    dv = v.shape[1]
    S = S0.astype(dtype).copy()
    O = np.zeros((L, dv), dtype)
    for t0 in range(0, L, C):
        n = min(C, L - t0)
        pad = lambda a, w: np.concatenate([a[t0:t0 + n], np.zeros((C - n,) + a.shape[1:])]).astype(dtype)
        qc, kc, vc, gc = pad(q, 0), pad(k, 0), pad(v, 0), pad(g, 0)
        bc = pad(beta, 0)
        G = np.cumsum(gc, axis=0)
        gam = np.exp(G)
        if rebase == "direct":
            D = np.exp(G[:, None, :] - G[None, :, :])  # [r, s, i]
            D = np.where(np.arange(C)[:, None, None] >= np.arange(C)[None, :, None], D, 0)
            Lk = np.einsum("ri,si,rsi->rs", kc, kc, D)
            Lq = np.einsum("ri,si,rsi->rs", qc, kc, D)
        else:  # one rebasing point at row m (the tensor-core form, C <= 32)
            m = C // 2 - 1
            E = np.exp(G - G[m])
            Lk = (kc * E) @ (kc / E).T
            Lq = (qc * E) @ (kc / E).T
        tri_s = np.tril(np.ones((C, C)), -1)
        tri_i = np.tril(np.ones((C, C)), 0)
        Akk = bc[:, None] * np.where(tri_s > 0, Lk, 0)
        Aqk = np.where(tri_i > 0, Lq, 0)
        T = np.linalg.inv(np.eye(C) + Akk) * bc[None, :]
        W = T @ (kc * gam)
        Ut = T @ vc
        U = Ut - W @ S
        Oc = scale * ((qc * gam) @ S + Aqk @ U)
        Kc = kc * np.exp(G[-1] - G)
        S = gam[-1][:, None] * S + Kc.T @ U
        O[t0:t0 + n] = Oc[:n]
    return O, S


@pytest.mark.parametrize("C,rebase", [(16, "direct"), (32, "direct"), (64, "direct"),
                                      (16, "mid"), (32, "mid")])
@pytest.mark.parametrize("L", [1, 31, 32, 77])
def test_chunk_form_matches_sequential(oracle_mod, C, rebase, L):
    rng = np.random.default_rng(100 + L + C)
    dk, dv = 16, 8
    q = _unit_rows(rng.standard_normal((L, dk)))
    k = _unit_rows(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    g = -5.0 / (1.0 + np.exp(-rng.uniform(1, 16) * rng.standard_normal((L, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    O, S = chunk_forward(q, k, v, g, beta, S0, C, scale=0.9, rebase=rebase)
    ro, rS = oracle_mod.forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                g[None, :, None], beta[None, :, None],
                                init_state=S0[None, None], scale=0.9)
    np.testing.assert_allclose(O, ro[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, rS[0, 0], rtol=1e-10, atol=1e-12)


def test_rebased_factors_stay_finite_in_fp32():
    """Worst case g = -5 on every channel: with the row-15 rebasing point of a
    32-token chunk all operand factors are finite, nonzero fp32 numbers, and
    the Gram entries the kernel keeps (s <= r) are finite."""
    C, dk = 32, 8
    G = np.cumsum(np.full((C, dk), -5.0, np.float32), axis=0, dtype=np.float32)
    E = np.exp((G - G[15]).astype(np.float32))
    inv = np.exp((G[15] - G).astype(np.float32))
    assert np.isfinite(E).all() and np.isfinite(inv).all()
    assert (E > 0).all() and (inv > 0).all()
    with np.errstate(over="ignore"):  # the masked upper triangle may overflow
        prod = (E[:, None, :] * inv[None, :, :]).astype(np.float32)
    keep = np.tril(np.ones((C, C), bool))
    assert np.isfinite(prod[keep]).all()
    assert (prod[keep] <= 1.0 + 1e-6).all()


def test_segment_split_composes(oracle_mod):
    """Split one sequence into G segments; per segment the chunk form gives
    S~ (from zero, true values) and M (from the identity, zero values); the
    exact combine S_in[g+1] = S~_g + M_g S_in[g] and a second pass from the
    true incoming states reproduce the unsplit run."""
    rng = np.random.default_rng(7)
    L, dk, dv, C = 150, 8, 6, 16
    q = _unit_rows(rng.standard_normal((L, dk)))
    k = _unit_rows(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    g = -0.2 * rng.uniform(0, 1, (L, dk))  # slow decay so M matters
    beta = rng.uniform(0.1, 0.9, L)
    S0 = rng.standard_normal((dk, dv))
    bounds = [0, 48, 96, 150]
    S_in = [S0]
    for a, b in zip(bounds[:-2], bounds[1:-1]):
        _, St = chunk_forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], np.zeros((dk, dv)), C)
        _, M = chunk_forward(q[a:b], k[a:b], np.zeros((b - a, dk)), g[a:b], beta[a:b], np.eye(dk), C)
        S_in.append(St + M @ S_in[-1])
    O = []
    for j, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        Oj, S = chunk_forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], S_in[j], C)
        O.append(Oj)
    ro, rS = oracle_mod.forward(q[None, :, None], k[None, :, None], v[None, :, None],
                                g[None, :, None], beta[None, :, None], init_state=S0[None, None])
    np.testing.assert_allclose(np.concatenate(O), ro[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, rS[0, 0], rtol=1e-10, atol=1e-12)
