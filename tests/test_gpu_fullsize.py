"""Parity at the benchmark workloads' full sizes, in the launch
configuration bench.py times, on sampled (sequence, head) units that the
fp64 oracle recomputes one by one (whole sequences: the recurrence has no
shortcut), plus properties checked over every output.

Workloads: dense prefill B=8 H=32 T=4096; varlen 64 log-uniform sequences,
H=16, nonzero initial states; decode 256 x 32 heads for 1024 steps; long
prefill B=1 H=32 T=1048576 (segment split).  All dk = dv = 128, bf16
q/k/v, fp32 g/beta/state.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import (TOL_BF16_O, TOL_BF16_S, gpu_gate, gpu_prefill, rel_l2, to64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _oracle_units(oracle_mod, inp, units, cu=None):
    """Oracle on the listed (seq, head) units only; returns per-unit (o, S)."""
    A = to64(inp["A_log"])
    res = []
    for n, h in units:
        if cu is None:
            sl = lambda t: t[n:n + 1, :, h:h + 1]
        else:
            a, b = int(cu[n]), int(cu[n + 1])
            sl = lambda t: t[:, a:b, h:h + 1]
        z = to64(sl(inp["z"]))
        g = oracle_mod.gate(z, A[h:h + 1], -5.0)
        init = None
        if inp["init_state"] is not None:
            init = to64(inp["init_state"][n:n + 1, h:h + 1])
        o, S = oracle_mod.forward(to64(sl(inp["q"])), to64(sl(inp["k"])), to64(sl(inp["v"])),
                                  g, to64(sl(inp["beta"])), init_state=init)
        res.append((o[0, :, 0], S[0, 0]))
    return res


def _check_units(o, S, ref, units, cu=None):
    for (n, h), (o_ref, S_ref) in zip(units, ref):
        if cu is None:
            o_u = to64(o[n, :, h])
        else:
            o_u = to64(o[0, int(cu[n]):int(cu[n + 1]), h])
        assert rel_l2(o_u, o_ref) <= TOL_BF16_O, (n, h, rel_l2(o_u, o_ref))
        assert rel_l2(to64(S[n, h]), S_ref) <= TOL_BF16_S, (n, h)


def test_dense_prefill_full_size(oracle_mod):
    inp = W.make_prefill_inputs(8, 4096, 32, 128, 128, torch.bfloat16, seed=1, device=DEV)
    o, S, _, ws = gpu_prefill(inp, with_init=False)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    units = [(0, 0), (3, 17), (7, 31), (5, 9)]
    _check_units(o, S, _oracle_units(oracle_mod, inp, units), units)


def test_varlen_prefill_full_size(oracle_mod):
    lens = W.varlen_lengths(64, 3)
    cu_list = W.cu_seqlens_from_lengths(lens)
    inp = W.make_prefill_inputs(1, cu_list[-1], 16, 128, 128, torch.bfloat16, seed=3,
                                device=DEV, init_state=True, num_states=64)
    cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    o, S, _, ws = gpu_prefill(inp, cu=cu)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    longest = int(np.argmax(lens))
    shortest = int(np.argmin(lens))
    units = [(longest, 3), (shortest, 0), (17, 15), (40, 8)]
    _check_units(o, S, _oracle_units(oracle_mod, inp, units, cu=cu_list), units, cu=cu_list)


def test_decode_full_size(oracle_mod):
    N, H, d, steps = 256, 32, 128, 1024
    S0 = W.make_decode_state(N, H, d, d, 4, DEV)
    A_log = W.make_decode_gate_params(H, 4 + 1000, DEV)
    state = S0.clone()
    units = [(0, 0), (100, 5), (255, 31)]
    sel_n = torch.tensor([u[0] for u in units], device=DEV)
    sel_h = torch.tensor([u[1] for u in units], device=DEV)
    keep = {k: [] for k in ("q", "k", "v", "z", "beta", "o")}
    g = torch.empty((N, H, d), device=DEV)
    o = torch.empty((N, H, d), dtype=torch.bfloat16, device=DEV)
    for s in range(steps):
        x = W.make_decode_step_inputs(N, H, d, d, torch.bfloat16, 4 + s, DEV)
        kda.kda_gate_fwd(x["z"], A_log, g)
        kda.kda_decode_step(x["q"], x["k"], x["v"], g, x["beta"], state, o)
        for k in ("q", "k", "v", "z", "beta"):
            keep[k].append(x[k][sel_n, sel_h].clone())
        keep["o"].append(o[sel_n, sel_h].clone())
    torch.cuda.synchronize()
    assert torch.isfinite(state).all()
    st = {k: torch.stack(v, dim=1) for k, v in keep.items()}  # [units, steps, ...]
    for u, (n, h) in enumerate(units):
        z = to64(st["z"][u])[None, :, None]
        gref = oracle_mod.gate(z, to64(A_log)[h:h + 1], -5.0)
        o_ref, S_ref = oracle_mod.forward(
            to64(st["q"][u])[None, :, None], to64(st["k"][u])[None, :, None],
            to64(st["v"][u])[None, :, None], gref, to64(st["beta"][u])[None, :, None],
            init_state=to64(S0[n, h])[None, None])
        assert rel_l2(to64(st["o"][u]), o_ref[0, :, 0]) <= TOL_BF16_O
        assert rel_l2(to64(state[n, h]), S_ref[0, 0]) <= TOL_BF16_S


def test_long_prefill_full_size(oracle_mod):
    """T = 1,048,576 with B*H = 32: the segment-split launch sequence."""
    T, H = 1 << 20, 32
    inp = W.make_prefill_inputs(1, T, H, 128, 128, torch.bfloat16, seed=2, device=DEV)
    o, S, _, ws = gpu_prefill(inp, with_init=False)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    assert torch.isfinite(S).all()
    assert torch.isfinite(o[0, ::4096].float()).all()
    units = [(0, 11)]
    _check_units(o, S, _oracle_units(oracle_mod, inp, units), units)
