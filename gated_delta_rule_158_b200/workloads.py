"""Seeded synthetic inputs for the KDA path.

This module holds input generation only -- random draws, the row
normalisation and casts of the input recipe -- and none of the KDA
arithmetic: the gate g = g_min*sigmoid(e^A z) and the recurrence are computed
by libkda on the GPU and by the fp64 oracle on the CPU, each on its own, from
the raw draws produced here (z, A_log, beta, q, k, v, initial states).

Recipe (shared by tests and bench):
  * q, k ~ N(0, 1) in fp32, each [token, head] row L2-normalised, then cast
    (round to nearest even) to the run's input dtype;
  * v ~ N(0, 1) in fp32, cast to the input dtype;
  * z ~ N(0, 1) fp32 with q's shape; A_log[h] = log U[1, 16];
  * beta = sigmoid(N(0, 1)) fp32, one per [token, head];
  * initial states (where the workload has them) ~ N(0, 0.02^2) fp32;
  * varlen lengths L = floor(exp(U[ln 128, ln 32768])) clamped to
    [128, 32768].
Draw order: q, k, v, z, A_log, beta, initial state.  Large tensors are drawn
in slabs of SLAB_TOKENS tokens so the fp32 temporaries stay small; the
result depends only on the seed and the shapes.
"""
import math

import torch

SLAB_TOKENS = 1 << 15


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, gen, device, dtype, normalise=False, slab_dim=0):
    """N(0,1) draws in fp32, optionally L2-normalised along the last dim,
    cast to dtype; generated slab by slab along dimension ``slab_dim``."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n = shape[slab_dim]
    for s0 in range(0, n, SLAB_TOKENS):
        s1 = min(n, s0 + SLAB_TOKENS)
        sub = list(shape)
        sub[slab_dim] = s1 - s0
        x = torch.randn(sub, generator=gen, device=device, dtype=torch.float32)
        if normalise:
            x = x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)
        out.narrow(slab_dim, s0, s1 - s0).copy_(x)
    return out


def varlen_lengths(num_seqs: int, seed: int, lo: int = 128, hi: int = 32768):
    """Log-uniform sequence lengths in [lo, hi] (CPU generator, so the
    lengths do not depend on the device)."""
    g = _gen(seed, "cpu")
    u = torch.rand(num_seqs, generator=g, dtype=torch.float64)
    L = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return [int(x) for x in L.clamp(lo, hi).tolist()]


def cu_seqlens_from_lengths(lengths):
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return cu


def make_prefill_inputs(B, T, H, dk, dv, dtype=torch.bfloat16, seed=0,
                        device="cpu", init_state=False, num_states=None):
    """Dense [B, T, H, *] (or varlen with B == 1) prefill inputs.

    Returns a dict with q, k, v (dtype), z (fp32, [B,T,H,dk]), A_log (fp32,
    [H]), beta (fp32, [B,T,H]) and init_state (fp32 [N,H,dk,dv] or None,
    N = num_states or B)."""
    gen = _gen(seed, device)
    q = _normal((B, T, H, dk), gen, device, dtype, normalise=True, slab_dim=1)
    k = _normal((B, T, H, dk), gen, device, dtype, normalise=True, slab_dim=1)
    v = _normal((B, T, H, dv), gen, device, dtype, slab_dim=1)
    z = _normal((B, T, H, dk), gen, device, torch.float32, slab_dim=1)
    u = torch.rand(H, generator=gen, device=device, dtype=torch.float32)
    A_log = torch.log(1.0 + 15.0 * u)
    beta = torch.sigmoid(
        torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float32))
    S0 = None
    if init_state:
        N = num_states if num_states is not None else B
        S0 = 0.02 * torch.randn((N, H, dk, dv), generator=gen, device=device,
                                dtype=torch.float32)
    return dict(q=q, k=k, v=v, z=z, A_log=A_log, beta=beta, init_state=S0)


def make_backward_cotangents(B, T, H, dv, dk=None, dtype=torch.bfloat16, seed=0,
                             device="cpu"):
    """Seeded upstream gradients for the backward: dout [B, T, H, dv]
    (dtype, unit-variance Gaussian) and, when dk is given, d_final
    [B, H, dk, dv] fp32 (Gaussian, std 0.1); otherwise d_final is None."""
    gen = _gen(seed, device)
    dout = _normal((B, T, H, dv), gen, device, dtype, slab_dim=1)
    d_final = None
    if dk is not None:
        d_final = 0.1 * torch.randn((B, H, dk, dv), generator=gen, device=device,
                                    dtype=torch.float32)
    return dict(dout=dout, d_final=d_final)


def make_decode_state(N, H, dk, dv, seed, device):
    gen = _gen(seed, device)
    return 0.02 * torch.randn((N, H, dk, dv), generator=gen, device=device,
                              dtype=torch.float32)


def make_decode_gate_params(H, seed, device):
    gen = _gen(seed, device)
    u = torch.rand(H, generator=gen, device=device, dtype=torch.float32)
    return torch.log(1.0 + 15.0 * u)


def make_decode_step_inputs(N, H, dk, dv, dtype, seed, device):
    """Fresh single-token inputs for one decode step: q, k (normalised), v,
    z, beta with a leading [N, H] shape."""
    gen = _gen(seed, device)
    q = _normal((N, H, dk), gen, device, dtype, normalise=True)
    k = _normal((N, H, dk), gen, device, dtype, normalise=True)
    v = _normal((N, H, dv), gen, device, dtype)
    z = _normal((N, H, dk), gen, device, torch.float32)
    beta = torch.sigmoid(
        torch.randn((N, H), generator=gen, device=device, dtype=torch.float32))
    return dict(q=q, k=k, v=v, z=z, beta=beta)
