"""Shared helpers for the parity tests: run the CUDA path through the C ABI,
run the fp64 oracle on the same inputs, and compare.

The two sides meet only here, on the same seeded inputs from
gated_delta_rule_158_b200.workloads; each side computes the gate and the
recurrence on its own.
"""
import numpy as np
import torch

import gated_delta_rule_158_b200 as kda

# Tolerances (relative L2 over the whole tensor):
TOL_F32 = 1e-5        # fp32-input runs, outputs and states
TOL_BF16_O = 2e-2     # bf16-input runs, outputs
TOL_BF16_S = 1e-2     # bf16-input runs, fp32 final states
TOL_GATE = 1e-6       # gate, elementwise relative


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0:
        return float(num)
    return float(num / den)


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy() if t is not None else None


def gpu_gate(z, A_log):
    g = torch.empty_like(z)
    kda.kda_gate_fwd(z, A_log, g)
    return g


def gpu_prefill(inp, cu=None, chunk=0, scale=1.0, with_init=True, want_final=True):
    """gate + chunk_fwd on the GPU through the C ABI; returns (o, final, g, ws)."""
    q, k, v, z, A_log, beta = (inp[n] for n in ("q", "k", "v", "z", "A_log", "beta"))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = gpu_gate(z, A_log)
    N = B if cu is None else cu.numel() - 1
    init = inp["init_state"] if with_init else None
    final = torch.full((N, H, dk, dv), float("nan"), device=q.device) if want_final else None
    out = torch.full((B, T, H, dv), float("nan"), device=q.device, dtype=q.dtype)
    nbytes = kda.kda_chunk_fwd_workspace_size(
        B, T, H, dk, dv, 0 if cu is None else N, chunk,
        kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)
    kda.kda_chunk_fwd(q, k, v, g, beta, out, ws, init_state=init, cu_seqlens=cu,
                      final_state=final, scale=scale, chunk_size=chunk)
    return out, final, g, ws


def oracle_prefill(oracle, inp, cu=None, scale=1.0, with_init=True, units=None):
    """The oracle on the same inputs: its own gate, then the recurrence."""
    g = oracle.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    init = to64(inp["init_state"]) if with_init and inp["init_state"] is not None else None
    cu_np = None if cu is None else cu.cpu().numpy().astype(np.int64)
    return oracle.forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), g,
                          to64(inp["beta"]), init_state=init, cu_seqlens=cu_np, scale=scale,
                          units=units)


def unit_slices(o, final, units, cu=None):
    """Gather o rows and final states of (seq, head) units into lists."""
    outs, states = [], []
    for n, h in units:
        if cu is None:
            outs.append(o[n, :, h])
        else:
            a, b = int(cu[n]), int(cu[n + 1])
            outs.append(o[0, a:b, h])
        states.append(final[n, h])
    return outs, states
