"""GPU parity of the training backward (kda_recurrent_bwd, through the C ABI)
against the fp64 oracle backward.

The kernel reads q, k, v, dout in their element type and computes in fp32
from there on, so bf16 inputs change nothing in the arithmetic: the oracle
takes the same bf16 values, widened exactly.  Every gradient is held to the
fp32 bound (relative L2 <= 1e-5).  An fp32 re-run of the same token-by-token
chain rule on the CPU lands near 2e-7 on these shapes, so the bound leaves a
factor of ~50 for the different summation order and expf.  Every output is
filled with NaN first, so an element the kernel fails to write fails.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import TOL_F32, gpu_gate, rel_l2, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dg", "dbeta")


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def gpu_backward(inp, cot, g, scale, with_init, with_dfinal, want_dinit=True):
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(B, T, H, dk), dk=nan(B, T, H, dk), dv=nan(B, T, H, dv),
                 dg=nan(B, T, H, dk), dbeta=nan(B, T, H))
    if want_dinit:
        grads["d_init"] = nan(B, H, dk, dv)
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(B, T, H, dk, dv), dtype=torch.uint8,
                     device=DEV)
    kda.kda_recurrent_bwd(q, inp["k"], v, g, inp["beta"], cot["dout"], grads, ws,
                          init_state=inp["init_state"] if with_init else None,
                          d_final=cot["d_final"] if with_dfinal else None, scale=scale)
    torch.cuda.synchronize()
    return {n: to64(t) for n, t in grads.items()}


def oracle_backward(oracle, inp, cot, scale, with_init, with_dfinal):
    """The oracle's own gate, then its backward, on the same inputs."""
    g = oracle.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    return oracle.backward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), g,
                           to64(inp["beta"]), to64(cot["dout"]),
                           init_state=to64(inp["init_state"]) if with_init else None,
                           d_final=to64(cot["d_final"]) if with_dfinal else None, scale=scale)


def unit_inputs(inp, cot, b, h):
    """The inputs of one (b, h) unit as a B = 1, H = 1 problem (units are
    independent)."""
    tok = lambda t: t[b:b + 1, :, h:h + 1].contiguous()
    st = lambda t: t[b:b + 1, h:h + 1].contiguous()
    u = {n: tok(inp[n]) for n in ("q", "k", "v", "z", "beta")}
    u["A_log"] = inp["A_log"][h:h + 1].contiguous()
    u["init_state"] = st(inp["init_state"])
    return u, dict(dout=tok(cot["dout"]), d_final=st(cot["d_final"]))


CASES = [
    # B, T, H, dk, dv, dtype, init, d_final, scale
    (2, 150, 3, 128, 128, torch.float32, True, True, 0.7),   # 3 blocks of 64, ragged 22
    (1, 64, 2, 128, 128, torch.bfloat16, False, False, 1.0),  # exactly one block
    (2, 97, 2, 64, 32, torch.bfloat16, True, True, 0.5),
    (1, 200, 2, 32, 128, torch.float32, False, True, 1.0),
    (1, 130, 2, 128, 64, torch.bfloat16, True, False, 0.125),
    (1, 70, 2, 128, 32, torch.float32, True, True, 1.0),    # dk 128, two 16-column dv blocks
    (3, 1, 2, 32, 32, torch.float32, True, True, 1.0),       # one token
    (1, 129, 1, 64, 64, torch.float32, True, True, 1.0),     # one token past two blocks
]


@pytest.mark.parametrize("B,T,H,dk,dv,dtype,init,dfin,scale", CASES)
def test_backward_parity(oracle_mod, B, T, H, dk, dv, dtype, init, dfin, scale):
    inp = W.make_prefill_inputs(B, T, H, dk, dv, dtype, seed=T + dk, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, dv, dk=dk, dtype=dtype, seed=T + 1, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    got = gpu_backward(inp, cot, g, scale, init, dfin)
    ref = oracle_backward(oracle_mod, inp, cot, scale, init, dfin)
    for n in NAMES:
        assert np.isfinite(got[n]).all(), n
        assert rel_l2(got[n], ref[n]) <= TOL_F32, (n, rel_l2(got[n], ref[n]))
    assert rel_l2(got["d_init"], ref["dS0"]) <= TOL_F32


def test_backward_empty_sequence_passes_d_final_through():
    B, H, dk, dv = 2, 3, 64, 128
    inp = W.make_prefill_inputs(B, 0, H, dk, dv, torch.bfloat16, seed=3, device=DEV)
    cot = W.make_backward_cotangents(B, 0, H, dv, dk=dk, seed=4, device=DEV)
    g = torch.empty((B, 0, H, dk), device=DEV)
    got = gpu_backward(inp, cot, g, 1.0, False, True)
    assert np.array_equal(got["d_init"], to64(cot["d_final"]))
    got = gpu_backward(inp, cot, g, 1.0, False, False)
    assert (got["d_init"] == 0).all()


def test_backward_without_d_init_leaves_other_grads_unchanged(oracle_mod):
    B, T, H, dk, dv = 1, 70, 2, 64, 64
    inp = W.make_prefill_inputs(B, T, H, dk, dv, torch.float32, seed=21, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, dv, dk=dk, dtype=torch.float32, seed=22,
                                     device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    a = gpu_backward(inp, cot, g, 1.0, True, True, want_dinit=False)
    b = gpu_backward(inp, cot, g, 1.0, True, True, want_dinit=True)
    for n in NAMES:
        assert np.array_equal(a[n], b[n]), n


def test_backward_fullsize_sampled(oracle_mod):
    """The prefill workload's shape (B 8, H 32, T 4096, d 128, bf16 inputs):
    every gradient finite (so written: the buffers start as NaN), and three
    (b, h) units against the oracle element by element."""
    B, T, H, d = 8, 4096, 32, 128
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=1, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, d, dk=d, seed=2, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(B, T, H, d), dk=nan(B, T, H, d), dv=nan(B, T, H, d),
                 dg=nan(B, T, H, d), dbeta=nan(B, T, H), d_init=nan(B, H, d, d))
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(B, T, H, d, d), dtype=torch.uint8,
                     device=DEV)
    kda.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], cot["dout"], grads, ws,
                          init_state=inp["init_state"], d_final=cot["d_final"])
    torch.cuda.synchronize()
    for n, t in grads.items():
        assert bool(torch.isfinite(t).all()), n
    for b, h in [(0, 0), (B - 1, H - 1), (3, 17)]:
        ui, uc = unit_inputs(inp, cot, b, h)
        ref = oracle_backward(oracle_mod, ui, uc, 1.0, True, True)
        for n in NAMES:
            got = to64(grads[n][b, :, h])
            assert rel_l2(got, ref[n][0, :, 0]) <= TOL_F32, (b, h, n)
        assert rel_l2(to64(grads["d_init"][b, h]), ref["dS0"][0, 0]) <= TOL_F32


def test_backward_strong_decay_takes_exact_exponents(oracle_mod):
    """A gate floor of -40 lets a 16-token half chunk decay by far more than
    e^80, which sends the key-side Gram to its exponent-difference form; the
    gradients still meet the fp32 bar."""
    B, T, H, dk, dv = 1, 150, 2, 64, 64
    inp = W.make_prefill_inputs(B, T, H, dk, dv, torch.float32, seed=31, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, dv, dk=dk, dtype=torch.float32, seed=32,
                                     device=DEV)
    g = torch.empty_like(inp["z"])
    kda.kda_gate_fwd(inp["z"], inp["A_log"], g, g_min=-40.0)
    assert float(g.min()) < -10.0
    got = gpu_backward(inp, cot, g, 1.0, True, True)
    g_ref = oracle_mod.gate(to64(inp["z"]), to64(inp["A_log"]), -40.0)
    ref = oracle_mod.backward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), g_ref,
                              to64(inp["beta"]), to64(cot["dout"]),
                              init_state=to64(inp["init_state"]),
                              d_final=to64(cot["d_final"]))
    for n in NAMES:
        assert rel_l2(got[n], ref[n]) <= TOL_F32, (n, rel_l2(got[n], ref[n]))
    assert rel_l2(got["d_init"], ref["dS0"]) <= TOL_F32


def gpu_gate_bwd(z, A_log, dg, g_min=-5.0, in_place=False):
    H = z.shape[-2]
    dz = dg.clone() if in_place else torch.full_like(z, float("nan"))
    src = dz if in_place else dg
    dA = torch.full((H,), float("nan"), device=DEV)
    ws = torch.empty(kda.kda_gate_bwd_workspace_size(H), dtype=torch.uint8, device=DEV)
    kda.kda_gate_bwd(z, A_log, src, dz, dA, ws, g_min=g_min)
    torch.cuda.synchronize()
    return dz, dA


@pytest.mark.parametrize("shape,g_min,in_place", [((2, 77, 5, 64), -5.0, False),
                                                  ((1, 1, 3, 32), -5.0, False),
                                                  ((3, 40, 2, 128), -40.0, True),
                                                  ((8, 4096, 32, 128), -5.0, False)])
def test_gate_backward_parity(oracle_mod, shape, g_min, in_place):
    """dz elementwise and dA_log per head against the fp64 gate backward: the
    fp32 bar (relative L2 1e-5)."""
    inp = W.make_prefill_inputs(shape[0], shape[1], shape[2], shape[3], 32, torch.float32,
                                seed=shape[1], device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(77)
    dg = torch.randn(inp["z"].shape, generator=gen, device=DEV)
    dz, dA = gpu_gate_bwd(inp["z"], inp["A_log"], dg, g_min, in_place)
    rz, rA = oracle_mod.gate_backward(to64(inp["z"]), to64(inp["A_log"]), to64(dg), g_min)
    assert rel_l2(to64(dz), rz) <= TOL_F32
    # dA_log is a sum of rows * dk signed terms: bound its error by the fp32 bar
    # times the sum of the terms' magnitudes (the scale summation error has)
    x = np.exp(to64(inp["A_log"]))[None, None, :, None] * to64(inp["z"])
    sg = 1.0 / (1.0 + np.exp(-x))
    terms = np.abs(to64(dg) * g_min * sg * (1.0 - sg) * x)
    scale = terms.sum(axis=(0, 1, 3))
    assert (np.abs(to64(dA) - rA) <= TOL_F32 * scale).all()
    dz2, dA2 = gpu_gate_bwd(inp["z"], inp["A_log"], dg, g_min, in_place)
    assert torch.equal(dz, dz2) and torch.equal(dA, dA2)  # fixed summation order


def test_gated_training_backward_chain(oracle_mod):
    """The gated model's input gradients: kda_recurrent_bwd gives dg, the gate
    backward turns it into dz and dA_log; the oracle does the same chain in
    fp64 on its own gate.  All at the fp32 bar."""
    B, T, H, dk, dv = 2, 90, 3, 64, 64
    inp = W.make_prefill_inputs(B, T, H, dk, dv, torch.bfloat16, seed=41, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, dv, dk=dk, seed=42, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    got = gpu_backward(inp, cot, g, 1.0, True, True)
    dz, dA = gpu_gate_bwd(inp["z"], inp["A_log"],
                          torch.from_numpy(got["dg"]).float().to(DEV))
    ref = oracle_backward(oracle_mod, inp, cot, 1.0, True, True)
    rz, rA = oracle_mod.gate_backward(to64(inp["z"]), to64(inp["A_log"]), ref["dg"], -5.0)
    assert rel_l2(to64(dz), rz) <= TOL_F32
    assert rel_l2(to64(dA), rA) <= TOL_F32


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 64),
                                     (torch.bfloat16, 128)])
def test_backward_varlen_parity(oracle_mod, dtype, d):
    """A packed batch (cu_seqlens) with empty, one-token, ragged and
    whole-chunk sequences: each sequence's gradients and dS0 against the
    oracle run on that sequence alone; an empty sequence passes d_final
    through to d_init.  d = 128 takes the tensor-core products (tcgen05 in
    the token-gradient pass)."""
    lengths = [0, 1, 31, 32, 33, 100, 64, 7, 0, 45]
    N, H, dk, dv = len(lengths), 2, d, d
    cu_list = W.cu_seqlens_from_lengths(lengths)
    T = cu_list[-1]
    cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    inp = W.make_prefill_inputs(1, T, H, dk, dv, dtype, seed=51, device=DEV, init_state=True,
                                num_states=N)
    cot = W.make_backward_cotangents(1, T, H, dv, dk=None, dtype=dtype, seed=52, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(53)
    cot["d_final"] = 0.1 * torch.randn((N, H, dk, dv), generator=gen, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(1, T, H, dk), dk=nan(1, T, H, dk), dv=nan(1, T, H, dv),
                 dg=nan(1, T, H, dk), dbeta=nan(1, T, H), d_init=nan(N, H, dk, dv))
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(1, T, H, dk, dv, N), dtype=torch.uint8,
                     device=DEV)
    kda.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], cot["dout"], grads, ws,
                          init_state=inp["init_state"], d_final=cot["d_final"], cu_seqlens=cu)
    st, _ = kda.kda_get_device_status(ws)
    assert st == kda.KDA_OK
    got = {n_: to64(t) for n_, t in grads.items()}
    g_ref = oracle_mod.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    for n in range(N):
        a, b = cu_list[n], cu_list[n + 1]
        if a == b:
            assert np.array_equal(got["d_init"][n], to64(cot["d_final"][n]))
            continue
        sl = lambda x: np.ascontiguousarray(x[:, a:b])
        ref = oracle_mod.backward(sl(to64(inp["q"])), sl(to64(inp["k"])), sl(to64(inp["v"])),
                                  sl(g_ref), sl(to64(inp["beta"])), sl(to64(cot["dout"])),
                                  init_state=to64(inp["init_state"][n:n + 1]),
                                  d_final=to64(cot["d_final"][n:n + 1]))
        for name in NAMES:
            assert rel_l2(got[name][:, a:b], ref[name]) <= TOL_F32, (n, name)
        assert rel_l2(got["d_init"][n], ref["dS0"][0]) <= TOL_F32, n


def test_backward_varlen_bad_offsets_are_reported():
    """Offsets that decrease: the plan kernel records KDA_ERR_BAD_SEQLENS and
    no gradient is written (the outputs keep their NaN fill)."""
    T, H, d = 64, 2, 32
    cu = torch.tensor([0, 40, 20, 64], dtype=torch.int32, device=DEV)
    inp = W.make_prefill_inputs(1, T, H, d, d, torch.float32, seed=61, device=DEV)
    cot = W.make_backward_cotangents(1, T, H, d, dk=None, dtype=torch.float32, seed=62,
                                     device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(1, T, H, d), dk=nan(1, T, H, d), dv=nan(1, T, H, d), dg=nan(1, T, H, d),
                 dbeta=nan(1, T, H), d_init=nan(3, H, d, d))
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(1, T, H, d, d, 3), dtype=torch.uint8,
                     device=DEV)
    kda.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], cot["dout"], grads, ws,
                          cu_seqlens=cu)
    st, _ = kda.kda_get_device_status(ws)
    assert st == kda.KDA_ERR_BAD_SEQLENS
    for name, t in grads.items():
        assert bool(torch.isnan(t).all()), name


# ------------------------------------------------- long sequences (windowed)

@pytest.mark.parametrize("d,H", [(64, 2), (128, 1)])
def test_backward_windowed_matches_oracle(oracle_mod, d, H):
    """T = 20000 > 8192: the bounded-workspace schedule (windows of 8192
    tokens, the last ragged, start states checkpointed, the state gradient
    handed from window to window) against the oracle, with an initial state, a
    final-state gradient and a scale; every gradient element at the fp32 bar.
    d = 128 takes the tensor-core products."""
    B, T = 1, 20000
    assert kda.kda_recurrent_bwd_workspace_size(B, T, H, d, d) < \
        kda.kda_recurrent_bwd_workspace_size(B, 8192, H, d, d) * 1.1
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=301, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, d, dk=d, dtype=torch.bfloat16, seed=302, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    got = gpu_backward(inp, cot, g, 0.9, True, True)
    ref = oracle_backward(oracle_mod, inp, cot, 0.9, True, True)
    for n in NAMES:
        assert np.isfinite(got[n]).all(), n
        assert rel_l2(got[n], ref[n]) <= TOL_F32, (n, rel_l2(got[n], ref[n]))
    assert rel_l2(got["d_init"], ref["dS0"]) <= TOL_F32


def test_backward_long_sequence_bounded_workspace(oracle_mod):
    """B1 H32 T = 262,144: the workspace stays bounded (one window's chunks
    plus a state per window, not two states per 32 tokens), and sampled units
    match the oracle over the whole sequence at the fp32 bar."""
    B, T, H, d = 1, 1 << 18, 32, 32
    per_chunk = 2 * d * d + 3 * 32 * 32 + 4 * 32 * d  # floats per chunk of the full schedule
    full = B * H * (T // 32) * per_chunk * 4
    ws_bytes = kda.kda_recurrent_bwd_workspace_size(B, T, H, d, d)
    assert ws_bytes < full / 20, (ws_bytes, full)
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=311, device=DEV,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, d, dk=d, dtype=torch.bfloat16, seed=312, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(B, T, H, d), dk=nan(B, T, H, d), dv=nan(B, T, H, d),
                 dg=nan(B, T, H, d), dbeta=nan(B, T, H), d_init=nan(B, H, d, d))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    kda.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], cot["dout"], grads, ws,
                          init_state=inp["init_state"], d_final=cot["d_final"])
    torch.cuda.synchronize()
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    for n, t in grads.items():
        assert torch.isfinite(t).all(), n
    for h in (0, 21):
        ui, uc = unit_inputs(inp, cot, 0, h)
        ref = oracle_backward(oracle_mod, ui, uc, 1.0, True, True)
        for n in NAMES:
            got = to64(grads[n][0:1, :, h:h + 1])
            assert rel_l2(got, ref[n]) <= TOL_F32, (h, n, rel_l2(got, ref[n]))
        assert rel_l2(to64(grads["d_init"][0:1, h:h + 1]), ref["dS0"]) <= TOL_F32
