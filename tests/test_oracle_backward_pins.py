"""Pins for the oracle's backward (gradients through the KDA recurrence of
"NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Model Architecture > Kimi Delta
Attention (KDA)).  The pages give the forward only, so the backward is pinned
to the forward: central finite differences of the (separately pinned) fp64
forward oracle, element by element, plus closed forms."""
import numpy as np
import pytest


def _problem(rng, B=1, T=6, H=2, dk=3, dv=4):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) * 0.6
    v = rng.standard_normal((B, T, H, dv))
    g = -rng.uniform(0.05, 2.0, (B, T, H, dk))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5
    W = rng.standard_normal((B, T, H, dv))   # dL/do
    V = rng.standard_normal((B, H, dk, dv))  # dL/dS_T
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0), W, V


def _loss(oracle_mod, x, W, V, scale):
    o, S = oracle_mod.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], init_state=x["S0"],
                              scale=scale)
    return float(np.sum(o * W) + np.sum(S * V))


@pytest.mark.parametrize("seed,scale", [(0, 1.0), (1, 0.7)])
def test_backward_matches_finite_differences(oracle_mod, seed, scale):
    rng = np.random.default_rng(seed)
    x, W, V = _problem(rng)
    grads = oracle_mod.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], W,
                                init_state=x["S0"], d_final=V, scale=scale)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", S0="dS0")
    eps = 1e-6
    for name, gname in names.items():
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(*x[name].shape):
            keep = x[name][idx]
            x[name][idx] = keep + eps
            up = _loss(oracle_mod, x, W, V, scale)
            x[name][idx] = keep - eps
            dn = _loss(oracle_mod, x, W, V, scale)
            x[name][idx] = keep
            fd[idx] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(grads[gname], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_one_token_closed_form(oracle_mod):
    """T = 1 from a zero state: S_1 = beta k v^T, o = scale beta (k.q) v, so
    dq = scale beta (v.do) k, dv = scale beta (k.q) do, dbeta = scale (k.q)(v.do)."""
    rng = np.random.default_rng(3)
    dk, dv, scale = 5, 3, 0.9
    q, k = rng.standard_normal((1, 1, 1, dk)), rng.standard_normal((1, 1, 1, dk))
    v, do = rng.standard_normal((1, 1, 1, dv)), rng.standard_normal((1, 1, 1, dv))
    g = -rng.uniform(0.1, 1.0, (1, 1, 1, dk))
    beta = np.array([[[0.4]]])
    r = oracle_mod.backward(q, k, v, g, beta, do, scale=scale)
    kq, vdo = float(k.ravel() @ q.ravel()), float(v.ravel() @ do.ravel())
    np.testing.assert_allclose(r["dq"].ravel(), scale * 0.4 * vdo * k.ravel(), rtol=1e-12)
    np.testing.assert_allclose(r["dv"].ravel(), scale * 0.4 * kq * do.ravel(), rtol=1e-12)
    np.testing.assert_allclose(r["dbeta"].ravel(), [scale * kq * vdo], rtol=1e-12)
    # from a zero state the decay acts on nothing
    np.testing.assert_array_equal(r["dg"], 0.0)


def test_backward_beta_zero_writes_nothing(oracle_mod):
    """beta = 0: the state only decays, so v has no influence: dv == 0 exactly."""
    rng = np.random.default_rng(4)
    x, W, V = _problem(rng)
    x["beta"][:] = 0.0
    r = oracle_mod.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], W,
                            init_state=x["S0"], d_final=V)
    np.testing.assert_array_equal(r["dv"], 0.0)
    assert np.abs(r["dbeta"]).max() > 0  # but the loss still depends on beta


def test_gate_backward_matches_finite_differences(oracle_mod):
    """dz and dA_log of L = sum(g * W) against central differences of the
    (separately pinned) gate oracle, element by element."""
    rng = np.random.default_rng(5)
    z = rng.standard_normal((3, 2, 4, 5))
    A_log = rng.uniform(-1.0, 2.0, 4)
    W = rng.standard_normal(z.shape)
    dz, dA = oracle_mod.gate_backward(z, A_log, W, g_min=-5.0)
    loss = lambda zz, aa: float(np.sum(oracle_mod.gate(zz, aa, -5.0) * W))
    eps = 1e-6
    fz = np.zeros_like(z)
    for idx in np.ndindex(*z.shape):
        zp, zm = z.copy(), z.copy()
        zp[idx] += eps
        zm[idx] -= eps
        fz[idx] = (loss(zp, A_log) - loss(zm, A_log)) / (2 * eps)
    np.testing.assert_allclose(dz, fz, rtol=1e-6, atol=1e-8)
    fa = np.zeros_like(A_log)
    for h in range(A_log.shape[0]):
        ap, am = A_log.copy(), A_log.copy()
        ap[h] += eps
        am[h] -= eps
        fa[h] = (loss(z, ap) - loss(z, am)) / (2 * eps)
    np.testing.assert_allclose(dA, fa, rtol=1e-6, atol=1e-8)


def test_gate_backward_closed_form_at_zero(oracle_mod):
    """At z = 0: sigmoid = 1/2, so dz = dg g_min e^{A} / 4 and dA_log = 0."""
    A_log = np.array([0.3, -0.7])
    z = np.zeros((2, 2, 3))
    dg = np.arange(12, dtype=np.float64).reshape(z.shape) - 5.0
    dz, dA = oracle_mod.gate_backward(z, A_log, dg, g_min=-5.0)
    np.testing.assert_allclose(dz, dg * -5.0 * np.exp(A_log)[None, :, None] / 4.0, rtol=1e-15)
    np.testing.assert_array_equal(dA, np.zeros(2))
