"""fp64 check of the chunkwise backward algebra the CUDA backward implements.

A test aid, not the oracle: a numpy restatement of the three passes of the
chunked backward, compared with the oracle's sequential backward (itself
pinned by finite differences).  Per (sequence, head), chunks of C tokens,
Gamma the in-chunk cumulative log-decay, E[r,s,i] = exp(Gamma_ri - Gamma_si)
for s <= r (never overflows for g <= 0):

  forward pass (chunk order), from the chunk-start state S:
    L = strict_lower(sum_i k_ri k_si E_rsi),  A_qk = lower(sum_i q_ri k_si E_rsi)
    X = (I + Diag(beta) L)^-1,  T = X Diag(beta)
    Qg = q e^Gamma,  Ka = k e^Gamma,  Kc = k e^{Gamma_C - Gamma}
    U = T (V - Ka S),  S_next = Diag(e^{Gamma_C}) S + Kc^T U
  state-gradient pass (reverse chunk order), dS = dL/dS_next of the chunk:
    dU = A_qk^T dO' + Kc dS          (dO' = scale dO)
    dS <- Diag(e^{Gamma_C}) dS + Qg^T dO' - Ka^T T^T dU
  per-chunk gradients (independent chunks), from S and dS = dL/dS_next:
    P = Ka S, R = V - P, U = T R, dU as above, W = T^T dU  ->  dv = W
    dQg = dO' S^T,  dKa = -W S^T,  dKc = U dS^T
    dA_qk = lower(dO' U^T),  dT = dU R^T
    dbeta_s += sum_r dT_rs X_rs;  dX = dT Diag(beta);  dM = -X^T dX X^T
    dbeta_r += sum_{s<r} dM_rs L_rs;  dL = Diag(beta) strict_lower(dM)
    through E: dq, dk and dGamma from dL and dA_qk;  through the decays:
    dq += dQg e^Gamma, dk += dKa e^Gamma + dKc e^{Gamma_C - Gamma},
    dGamma += dQg Qg + dKa Ka - dKc Kc,  dGamma_C += sum_r dKc Kc + e^{Gamma_C} rowsum(dS . S)
    dg = reverse cumulative sum of dGamma within the chunk.
Tail chunks are padded with g = 0, beta = 0, k = q = v = dO = 0, which leaves
every real token's gradients unchanged.
"""
import numpy as np
import pytest


def _pad(a, t0, n, C):
    out = np.zeros((C,) + a.shape[1:])
    out[:n] = a[t0:t0 + n]
    return out


def _keyside(qc, kc, gc, bc):
    C = kc.shape[0]
    G = np.cumsum(gc, axis=0)
    low_i = np.arange(C)[:, None] >= np.arange(C)[None, :]
    E = np.where(low_i[:, :, None], np.exp(np.minimum(G[:, None, :] - G[None, :, :], 0.0)), 0.0)
    Lf = np.einsum("ri,si,rsi->rs", kc, kc, E)
    L = np.tril(Lf, -1)
    Aqk = np.tril(np.einsum("ri,si,rsi->rs", qc, kc, E))
    X = np.linalg.inv(np.eye(C) + bc[:, None] * L)
    return dict(G=G, E=E, L=L, Aqk=Aqk, X=X, T=X * bc[None, :], gC=G[-1],
                Qg=qc * np.exp(G), Ka=kc * np.exp(G), Kc=kc * np.exp(G[-1][None, :] - G))


def chunked_backward(q, k, v, g, beta, dout, S0, dF, C, scale=1.0):
    """One (sequence, head): q, k, g [L, dk]; v, dout [L, dv]; beta [L];
    S0, dF [dk, dv].  Returns dq, dk, dv, dg, dbeta, dS0."""
    Ltok, dk = k.shape
    dv = v.shape[1]
    nc = (Ltok + C - 1) // C
    chunks = []
    for c in range(nc):
        t0 = c * C
        n = min(C, Ltok - t0)
        ch = {name: _pad(a, t0, n, C) for name, a in
              (("q", q), ("k", k), ("v", v), ("g", g), ("b", beta), ("do", dout))}
        ch.update(_keyside(ch["q"], ch["k"], ch["g"], ch["b"]))
        ch["t0"], ch["n"] = t0, n
        chunks.append(ch)
    # forward pass: chunk-start states
    S = S0.copy()
    for ch in chunks:
        ch["S"] = S.copy()
        U = ch["T"] @ (ch["v"] - ch["Ka"] @ S)
        S = np.exp(ch["gC"])[:, None] * S + ch["Kc"].T @ U
    # state-gradient pass: dL/dS_next of every chunk
    dS = dF.copy()
    for ch in reversed(chunks):
        ch["dSn"] = dS.copy()
        dO = scale * ch["do"]
        dU = ch["Aqk"].T @ dO + ch["Kc"] @ dS
        dS = np.exp(ch["gC"])[:, None] * dS + ch["Qg"].T @ dO - ch["Ka"].T @ (ch["T"].T @ dU)
    dS0 = dS
    # per-chunk gradients
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros_like(beta))
    for ch in chunks:
        S, dSn, X, T, E = ch["S"], ch["dSn"], ch["X"], ch["T"], ch["E"]
        qc, kc, bc = ch["q"], ch["k"], ch["b"]
        dO = scale * ch["do"]
        R = ch["v"] - ch["Ka"] @ S
        U = T @ R
        dU = ch["Aqk"].T @ dO + ch["Kc"] @ dSn
        W = T.T @ dU
        dQg = dO @ S.T
        dKa = -W @ S.T
        dKc = U @ dSn.T
        dAqk = np.tril(dO @ U.T)
        dT = dU @ R.T
        dbeta = np.sum(dT * X, axis=0)
        dX = dT * bc[None, :]
        dM = -X.T @ dX @ X.T
        dbeta += np.sum(np.tril(dM, -1) * ch["L"], axis=1)
        dL = bc[:, None] * np.tril(dM, -1)
        # through E: L_rs = sum_i k_ri k_si E_rsi, A_qk,rs = sum_i q_ri k_si E_rsi
        Fr = dL[:, :, None] * kc[:, None, :] + dAqk[:, :, None] * qc[:, None, :]  # [r,s,i] d/dk_si
        dq = np.einsum("rs,si,rsi->ri", dAqk, kc, E)
        dk_ = np.einsum("rs,si,rsi->ri", dL, kc, E) + np.einsum("rsi,rsi->si", Fr, E)
        Z = Fr * kc[None, :, :] * E  # d/dGamma_ri (+), d/dGamma_si (-)
        dG = Z.sum(axis=1) - Z.sum(axis=0)
        G = ch["G"]
        dq += dQg * np.exp(G)
        dk_ += dKa * np.exp(G) + dKc * np.exp(ch["gC"][None, :] - G)
        dG += dQg * ch["Qg"] + dKa * ch["Ka"] - dKc * ch["Kc"]
        dG[-1] += np.sum(dKc * ch["Kc"], axis=0) + np.exp(ch["gC"]) * np.sum(dSn * S, axis=1)
        dg = np.cumsum(dG[::-1], axis=0)[::-1]
        t0, n = ch["t0"], ch["n"]
        out["dq"][t0:t0 + n] = dq[:n]
        out["dk"][t0:t0 + n] = dk_[:n]
        out["dv"][t0:t0 + n] = W[:n]
        out["dg"][t0:t0 + n] = dg[:n]
        out["dbeta"][t0:t0 + n] = dbeta[:n]
    out["dS0"] = dS0
    return out


def _problem(rng, L, dk, dv):
    q = rng.standard_normal((L, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, dv))
    g = -5.0 / (1.0 + np.exp(-rng.standard_normal((L, dk)) * 3))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    dout = rng.standard_normal((L, dv))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    dF = 0.3 * rng.standard_normal((dk, dv))
    return q, k, v, g, beta, dout, S0, dF


@pytest.mark.parametrize("L,C,dk,dv,scale", [(70, 16, 8, 6, 1.0), (64, 32, 16, 8, 0.7),
                                             (45, 32, 12, 12, 1.0), (100, 8, 6, 10, 0.5),
                                             (1, 32, 4, 4, 1.0)])
def test_chunked_backward_matches_oracle(oracle_mod, L, C, dk, dv, scale):
    rng = np.random.default_rng(L * 7 + C)
    q, k, v, g, beta, dout, S0, dF = _problem(rng, L, dk, dv)
    got = chunked_backward(q, k, v, g, beta, dout, S0, dF, C, scale)
    e = lambda a: a[None, :, None]
    ref = oracle_mod.backward(e(q), e(k), e(v), e(g), beta[None, :, None], e(dout),
                              init_state=S0[None, None], d_final=dF[None, None], scale=scale)
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        np.testing.assert_allclose(got[name], ref[name][0, :, 0], rtol=1e-9, atol=1e-10,
                                   err_msg=name)
    np.testing.assert_allclose(got["dS0"], ref["dS0"][0, 0], rtol=1e-9, atol=1e-10)
