"""Parity at the benchmark workloads' full sizes, in the launch
configuration bench.py times, on sampled (sequence, head) units that the
fp64 oracle recomputes one by one (whole sequences: the recurrence has no
shortcut), plus properties checked over every output.

Workloads: dense prefill B=8 H=32 T=4096 (bf16, and fp32 inputs on the
fp32-accuracy path); varlen 64 log-uniform sequences,
H=16, nonzero initial states; decode 256 x 32 heads for 1024 steps; long
prefill B=1 H=32 T=1048576 (segment split); speculative verify / replay
256 x 32 heads with 4 draft tokens.  All dk = dv = 128, bf16 q/k/v, fp32
g/beta/state.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import (TOL_BF16_O, TOL_BF16_S, TOL_F32, gpu_gate, gpu_prefill, rel_l2,
                          to64)

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


def _unit_gate(oracle_mod, inp, h, z64):
    return oracle_mod.gate(z64, to64(inp["A_log"])[h:h + 1], -5.0)


def _oracle_packed(oracle_mod, inp, units, cu):
    """The oracle on many (sequence, head) units of a packed batch in one call:
    each unit's rows of its head become one sequence of a packed batch with a
    single head, run by the oracle's thread pool.  Returns per-unit (o, S)."""
    rows = [(int(cu[n]), int(cu[n + 1])) for n, _ in units]
    cat = lambda name: np.concatenate([to64(inp[name][0, a:b, h]) for (a, b), (_, h) in
                                       zip(rows, units)], axis=0)
    z = [to64(inp["z"][0, a:b, h:h + 1])[None] for (a, b), (_, h) in zip(rows, units)]
    g = np.concatenate([_unit_gate(oracle_mod, inp, h, zz)[0, :, 0] for zz, (_, h) in
                        zip(z, units)], axis=0)
    sub_cu = np.concatenate([[0], np.cumsum([b - a for a, b in rows])]).astype(np.int64)
    init = None
    if inp["init_state"] is not None:
        init = np.stack([to64(inp["init_state"][n, h]) for n, h in units])[:, None]
    o, S = oracle_mod.forward(cat("q")[None, :, None], cat("k")[None, :, None],
                              cat("v")[None, :, None], g[None, :, None],
                              cat("beta")[None, :, None], init_state=init, cu_seqlens=sub_cu)
    return [(o[0, sub_cu[u]:sub_cu[u + 1], 0], S[u, 0]) for u in range(len(units))]


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


def test_prefill_fp32_full_size(oracle_mod):
    """The fp32-accuracy path (key-side pass, then the tcgen05 scan) at the
    prefill_fp32 workload's size, B=8 H=32 T=4096 with fp32 inputs and
    initial states: sampled units against the oracle at the fp32 bar."""
    inp = W.make_prefill_inputs(8, 4096, 32, 128, 128, torch.float32, seed=1, device=DEV,
                                init_state=True)
    o, S, _, ws = gpu_prefill(inp)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    units = [(0, 0), (2, 13), (7, 31)]
    for (n, h), (o_ref, S_ref) in zip(units, _oracle_units(oracle_mod, inp, units)):
        assert rel_l2(to64(o[n, :, h]), o_ref) <= TOL_F32, (n, h, rel_l2(to64(o[n, :, h]), o_ref))
        assert rel_l2(to64(S[n, h]), S_ref) <= TOL_F32, (n, h)


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
    # 16 sequences: the longest and the shortest, the rest spread over the batch,
    # each with its own head (every head appears)
    others = [n for n in range(0, 64, 4) if n not in (longest, shortest)][:14]
    seqs = [longest, shortest] + others
    units = [(n, (3 * i) % 16) for i, n in enumerate(seqs)]
    assert len(units) == 16
    _check_units(o, S, _oracle_packed(oracle_mod, inp, units, cu_list), units, cu=cu_list)


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


def _unsplit_reference(inp, g, piece=4064):
    """The long sequence without the segment split: consecutive calls of fewer
    than 4096 tokens each (below the split's threshold), each starting from the
    previous call's final state (the fp32 state is handed over exactly)."""
    q = inp["q"]
    B, T, H, d = q.shape
    out = torch.empty_like(q)
    state = None
    for a in range(0, T, piece):
        b = min(T, a + piece)
        sl = lambda t: t[:, a:b].contiguous()
        o_p = torch.empty((1, b - a, H, d), dtype=q.dtype, device=DEV)
        fin = torch.empty((1, H, d, d), device=DEV)
        ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(1, b - a, H, d, d), dtype=torch.uint8,
                         device=DEV)
        kda.kda_chunk_fwd(sl(q), sl(inp["k"]), sl(inp["v"]), sl(g), sl(inp["beta"]), o_p, ws,
                          init_state=state, final_state=fin)
        out[:, a:b] = o_p
        state = fin
    return out, state


def test_long_prefill_full_size(oracle_mod):
    """T = 1,048,576 with B*H = 32: the segment-split launch sequence.  Every
    unit (outputs and final state) against the same recurrence run without the
    split, and 8 units spread over the heads against the oracle over the whole
    sequence (run in pieces, its fp64 state carried from piece to piece, which
    is exactly one sequential run)."""
    T, H = 1 << 20, 32
    inp = W.make_prefill_inputs(1, T, H, 128, 128, torch.bfloat16, seed=2, device=DEV)
    o, S, g, ws = gpu_prefill(inp, with_init=False)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    assert torch.isfinite(S).all() and torch.isfinite(o.float()).all()

    o_ref, S_ref = _unsplit_reference(inp, g)
    torch.cuda.synchronize()
    for h in range(H):
        d_o = (o[0, :, h].double() - o_ref[0, :, h].double()).norm() / o_ref[0, :, h].double().norm()
        d_s = (S[0, h] - S_ref[0, h]).double().norm() / S_ref[0, h].double().norm()
        assert float(d_o) <= TOL_BF16_O, (h, float(d_o))
        assert float(d_s) <= TOL_BF16_S, (h, float(d_s))
    del o_ref, S_ref

    heads = [0, 5, 9, 14, 18, 23, 27, 31]
    piece = 1 << 16
    num = np.zeros(len(heads))
    den = np.zeros(len(heads))
    state = None
    for a in range(0, T, piece):
        b = a + piece
        stack = lambda name: np.stack([to64(inp[name][0, a:b, h]) for h in heads])[:, :, None]
        gg = np.stack([_unit_gate(oracle_mod, inp, h, to64(inp["z"][0:1, a:b, h:h + 1]))[0, :, 0]
                       for h in heads])[:, :, None]
        o_u, state = oracle_mod.forward(stack("q"), stack("k"), stack("v"), gg, stack("beta"),
                                        init_state=state)
        got = np.stack([to64(o[0, a:b, h]) for h in heads])
        num += ((got - o_u[:, :, 0]) ** 2).sum(axis=(1, 2))
        den += (o_u[:, :, 0] ** 2).sum(axis=(1, 2))
    for u, h in enumerate(heads):
        assert np.sqrt(num[u] / den[u]) <= TOL_BF16_O, (h, np.sqrt(num[u] / den[u]))
        assert rel_l2(to64(S[0, h]), state[u, 0]) <= TOL_BF16_S, h


def test_spec_decode_full_size(oracle_mod):
    """Speculative verify / replay at the benchmark's size (N256 H32 d128,
    K = 4 draft tokens, bf16): verify leaves the committed state bit for bit;
    replay with accepted lengths 0 ... K across the batch leaves the
    zero-accept sequences untouched; sampled units' outputs and replayed
    states against the oracle."""
    N, H, d, K = 256, 32, 128, 4
    inp = W.make_prefill_inputs(N, K, H, d, d, torch.bfloat16, seed=7, device=DEV)
    S0 = W.make_decode_state(N, H, d, d, 8, DEV)
    state = S0.clone()
    out = torch.full((N, K, H, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], state, out,
                          A_log=inp["A_log"])
    torch.cuda.synchronize()
    assert torch.equal(state, S0)
    assert torch.isfinite(out.float()).all()
    acc = torch.arange(N, device=DEV, dtype=torch.int32) % (K + 1)
    kda.kda_decode_replay(inp["k"], inp["v"], inp["z"], inp["beta"], state, acc,
                          A_log=inp["A_log"])
    torch.cuda.synchronize()
    zero = (acc == 0).nonzero().flatten()
    assert torch.equal(state[zero], S0[zero])
    units = [(0, 0), (1, 7), (2, 31), (3, 12), (4, 20), (129, 5), (254, 30), (255, 31)]
    A = to64(inp["A_log"])
    for n, h in units:
        sl = lambda t: to64(t[n:n + 1, :, h:h + 1])
        g = oracle_mod.gate(sl(inp["z"]), A[h:h + 1], -5.0)
        o_ref, _ = oracle_mod.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), g, sl(inp["beta"]),
                                      init_state=to64(S0[n:n + 1, h:h + 1]))
        assert rel_l2(to64(out[n, :, h]), o_ref[0, :, 0]) <= TOL_BF16_O, (n, h)
        m = int(acc[n])
        if m == 0:
            continue
        cut = lambda t: np.ascontiguousarray(t[:, :m])
        _, S_ref = oracle_mod.forward(cut(sl(inp["q"])), cut(sl(inp["k"])), cut(sl(inp["v"])),
                                      cut(g), cut(sl(inp["beta"])),
                                      init_state=to64(S0[n:n + 1, h:h + 1]))
        assert rel_l2(to64(state[n, h]), S_ref[0, 0]) <= TOL_BF16_S, (n, h)
