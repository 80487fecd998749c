"""GPU parity: libkda (through its C ABI) against the fp64 oracle.

Small cases compare every element; they span several chunks and a ragged
tail.  Tolerances (relative L2, written in kda_testutil): 1e-5 for fp32
inputs; 2e-2 on outputs and 1e-2 on final states for bf16 inputs with fp32
state.  Every output buffer is filled with NaN first, so an element the
kernels fail to write fails the comparison.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import (TOL_BF16_O, TOL_BF16_S, TOL_F32, TOL_GATE, gpu_gate, gpu_prefill,
                          oracle_prefill, rel_l2, to64, unit_slices)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


# ------------------------------------------------------------------- gate

def test_gate_parity(oracle_mod):
    """Elementwise bound derived from fp32 arithmetic: x = e^A z carries a
    relative rounding error <= 2 eps (the rounding of e^A and of the product),
    which the sigmoid turns into |dg/g| <= (1 - sigmoid(x)) |x| 2 eps; exp and
    the division add <= 3 eps.  With eps = 2^-24 and a factor 2 of margin:
    |g - g_ref| <= |g_ref| (4 |x| + 8) 2^-24."""
    inp = W.make_prefill_inputs(2, 77, 5, 64, 64, torch.float32, seed=11, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    ref = oracle_mod.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    x = np.exp(to64(inp["A_log"]))[None, None, :, None] * to64(inp["z"])
    got = to64(g)
    bound = np.abs(ref) * (4.0 * np.abs(x) + 8.0) * 2.0 ** -24
    assert (np.abs(got - ref) <= bound).all(), float(np.max(np.abs(got - ref) / bound))
    assert np.max(np.abs(got - ref) / np.abs(ref)) <= TOL_GATE * 20
    assert (got >= -5.0).all() and (got < 0).all()


# ----------------------------------------------------------------- decode

def _decode_run(oracle_mod, N, H, dk, dv, dtype, steps, seed0):
    S0 = W.make_decode_state(N, H, dk, dv, seed0, DEV)
    A_log = W.make_decode_gate_params(H, seed0 + 1000, DEV)
    state = S0.clone()
    outs, steps_in = [], []
    for s in range(steps):
        x = W.make_decode_step_inputs(N, H, dk, dv, dtype, seed0 + s, DEV)
        g = gpu_gate(x["z"], A_log)
        o = torch.full((N, H, dv), float("nan"), device=DEV, dtype=dtype)
        kda.kda_decode_step(x["q"], x["k"], x["v"], g, x["beta"], state, o)
        outs.append(o)
        steps_in.append(x)
    torch.cuda.synchronize()
    # oracle: the decode steps form a length-`steps` sequence per (n, h)
    st = lambda name: torch.stack([x[name] for x in steps_in], dim=1)  # [N, steps, H, ...]
    g_ref = oracle_mod.gate(to64(st("z")), to64(A_log), -5.0)
    o_ref, S_ref = oracle_mod.forward(to64(st("q")), to64(st("k")), to64(st("v")), g_ref,
                                      to64(st("beta")), init_state=to64(S0))
    o_gpu = to64(torch.stack(outs, dim=1))
    return o_gpu, to64(state), o_ref, S_ref


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128), (32, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_parity(oracle_mod, dk, dv, dtype):
    o, S, o_ref, S_ref = _decode_run(oracle_mod, 3, 5, dk, dv, dtype, steps=6, seed0=40)
    tol_o, tol_s = (TOL_F32, TOL_F32) if dtype == torch.float32 else (TOL_BF16_O, TOL_BF16_S)
    assert rel_l2(o, o_ref) <= tol_o
    assert rel_l2(S, S_ref) <= tol_s


# --------------------------------------------------------------- prefill

def test_prefill_tiny_fp32_config(oracle_mod):
    """B=1, H=2, T=64, dk=dv=32, chunk 16, fp32 throughout, seed 0, zero state."""
    inp = W.make_prefill_inputs(1, 64, 2, 32, 32, torch.float32, seed=0, device=DEV)
    o, S, _, _ = gpu_prefill(inp, chunk=16, with_init=False)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, with_init=False)
    assert rel_l2(to64(o), o_ref) <= TOL_F32
    assert rel_l2(to64(S), S_ref) <= TOL_F32


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(32, 64), (64, 32), (128, 128)])
def test_prefill_fp32_shapes(oracle_mod, chunk, dk, dv):
    inp = W.make_prefill_inputs(2, 150, 3, dk, dv, torch.float32, seed=5, device=DEV,
                                init_state=True)
    o, S, _, _ = gpu_prefill(inp, chunk=chunk, scale=0.75)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, scale=0.75)
    assert rel_l2(to64(o), o_ref) <= TOL_F32
    assert rel_l2(to64(S), S_ref) <= TOL_F32


@pytest.mark.parametrize("chunk", [0, 16, 64])
@pytest.mark.parametrize("T", [1, 31, 300])
def test_prefill_bf16_dense(oracle_mod, chunk, T):
    """bf16 dk = dv = 128: chunk 0 is the tensor-core path; 16/64 the fp32 one."""
    inp = W.make_prefill_inputs(2, T, 3, 128, 128, torch.bfloat16, seed=6 + T, device=DEV,
                                init_state=True)
    o, S, _, _ = gpu_prefill(inp, chunk=chunk)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S


@pytest.mark.parametrize("chunk", [0, 32])
def test_prefill_bf16_varlen(oracle_mod, chunk):
    lens = [1, 33, 0, 100, 64, 5, 257]
    cu_list = W.cu_seqlens_from_lengths(lens)
    T = cu_list[-1]
    inp = W.make_prefill_inputs(1, T, 2, 128, 128, torch.bfloat16, seed=21, device=DEV,
                                init_state=True, num_states=len(lens))
    cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    o, S, _, ws = gpu_prefill(inp, cu=cu, chunk=chunk)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, cu=cu)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S
    # zero-length sequence: final state equals its initial state
    assert torch.equal(S[2], inp["init_state"][2])


def test_chunk_size_invariance():
    inp = W.make_prefill_inputs(1, 200, 2, 64, 64, torch.float32, seed=3, device=DEV,
                                init_state=True)
    res = [gpu_prefill(inp, chunk=c)[:2] for c in (16, 32, 64)]
    for o, S in res[1:]:
        assert rel_l2(to64(o), to64(res[0][0])) <= 1e-5
        assert rel_l2(to64(S), to64(res[0][1])) <= 1e-5


@pytest.mark.parametrize("dk,dv", [(32, 128), (128, 64), (64, 128), (128, 32)])
@pytest.mark.parametrize("T", [45, 301])
def test_prefill_bf16_other_head_sizes(oracle_mod, dk, dv, T):
    """bf16 inputs with dk or dv below 128 take the fp32-accuracy chunk path:
    ragged lengths, initial states and scale against the oracle (o at the
    bf16 bar, the fp32 state at the fp32 bar)."""
    inp = W.make_prefill_inputs(2, T, 3, dk, dv, torch.bfloat16, seed=160 + T, device=DEV,
                                init_state=True)
    o, S, _, _ = gpu_prefill(inp, scale=0.8)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, scale=0.8)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_F32


@pytest.mark.parametrize("dtype,dk,dv", [(torch.float32, 128, 128), (torch.float32, 64, 32),
                                         (torch.bfloat16, 64, 64)])
def test_prefill_f32_path_packed_gated(oracle_mod, dtype, dk, dv):
    """The fp32-accurate chunk path (key-side pass, then the scan with the
    outputs) on a packed batch with empty, one-token, ragged and whole-chunk
    sequences, the gate fused into both of its kernels, initial states and
    scale, against the oracle: the fp32 state at the fp32 bar for both input
    types (bf16 inputs are widened exactly and every product keeps fp32
    accuracy), o at the bar of its type (bf16 o is rounded on store); an
    empty sequence keeps its initial state."""
    lengths = [0, 1, 31, 32, 33, 100, 5, 64]
    cu_list = W.cu_seqlens_from_lengths(lengths)
    N, H = len(lengths), 3
    inp = W.make_prefill_inputs(1, cu_list[-1], H, dk, dv, dtype, seed=150, device=DEV,
                                init_state=True, num_states=N)
    cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    o, S = _gated_prefill(inp, cu=cu, scale=0.6)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, cu=cu, scale=0.6)
    assert rel_l2(to64(o), o_ref) <= (TOL_F32 if dtype == torch.float32 else TOL_BF16_O)
    assert rel_l2(to64(S), S_ref) <= TOL_F32
    assert torch.equal(S[0], inp["init_state"][0])


def test_state_handoff_equals_full_run():
    """Running T1 then T2 with final_state -> init_state equals one run over T."""
    inp = W.make_prefill_inputs(1, 160, 2, 128, 128, torch.bfloat16, seed=9, device=DEV,
                                init_state=True)
    o_full, S_full, _, _ = gpu_prefill(inp)
    for t1 in (64, 77):
        # clone: a time slice of a B == 1 batch is already contiguous but
        # starts at an offset that need not be 16-byte aligned
        a = {k: (v[:, :t1].clone() if k in ("q", "k", "v", "z", "beta") else v)
             for k, v in inp.items()}
        b = {k: (v[:, t1:].clone() if k in ("q", "k", "v", "z", "beta") else v)
             for k, v in inp.items()}
        o1, S1, _, _ = gpu_prefill(a)
        b["init_state"] = S1
        o2, S2, _, _ = gpu_prefill(b)
        assert rel_l2(to64(torch.cat([o1, o2], 1)), to64(o_full)) <= 1e-2
        assert rel_l2(to64(S2), to64(S_full)) <= 1e-2


def test_guard_bands_untouched():
    """Outputs are written only inside their extents (canary slack around them)."""
    B, T, H, d = 1, 70, 2, 128
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=4, device=DEV,
                                init_state=True)
    g = gpu_gate(inp["z"], inp["A_log"])
    pad = 4096
    o_buf = torch.full((pad + B * T * H * d + pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    s_buf = torch.full((pad + B * H * d * d + pad,), 7.0, dtype=torch.float32, device=DEV)
    out = o_buf[pad:pad + B * T * H * d].view(B, T, H, d)
    fin = s_buf[pad:pad + B * H * d * d].view(B, H, d, d)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(B, T, H, d, d), dtype=torch.uint8,
                     device=DEV)
    kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], out, ws,
                      init_state=inp["init_state"], final_state=fin)
    torch.cuda.synchronize()
    for buf in (o_buf, s_buf):
        assert (buf[:pad] == 7.0).all() and (buf[-pad:] == 7.0).all()
    assert torch.isfinite(out).all() and torch.isfinite(fin).all()


def test_bad_seqlens_reported_on_device():
    T, H, d = 96, 2, 128
    inp = W.make_prefill_inputs(1, T, H, d, d, torch.bfloat16, seed=8, device=DEV)
    cu = torch.tensor([0, 50, 40, 96], dtype=torch.int32, device=DEV)  # not monotone
    out, _, _, ws = gpu_prefill(inp, cu=cu, with_init=False)
    st, _ = kda.kda_get_device_status(ws)
    assert st == kda.KDA_ERR_BAD_SEQLENS
    assert torch.isnan(out.float()).all()  # no unit ran


def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    kda.kda_selftest_bounded_wait(ws, 2_000_000)  # 2 ms on a flag nothing sets
    st, _ = kda.kda_get_device_status(ws)
    assert st == kda.KDA_ERR_TIMEOUT
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0  # the context is still usable


def test_chunk_kernel_timeout_path_returns_and_context_survives():
    """The tensor-core chunk kernel's own abort path: with its internal wait
    limit lowered to 0, a hand-off between its warp roles runs out; the kernel
    records KDA_ERR_TIMEOUT, drains what it issued, frees its tensor memory and
    returns.  With the limit restored the same call on the same workspace
    succeeds and matches a fresh run bit for bit."""
    B, T, H, d = 2, 4096, 4, 128
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=12, device=DEV,
                                init_state=True)
    o_ref, S_ref, g, _ = gpu_prefill(inp)
    out = torch.full_like(o_ref, float("nan"))
    fin = torch.full_like(S_ref, float("nan"))
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(B, T, H, d, d), dtype=torch.uint8,
                     device=DEV)
    try:
        kda.kda_set_wait_limit_ns(0)
        kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], out, ws,
                          init_state=inp["init_state"], final_state=fin)
        st, where = kda.kda_get_device_status(ws)
    finally:
        kda.kda_set_wait_limit_ns(2_000_000_000)
    assert st == kda.KDA_ERR_TIMEOUT, kda.kda_status_string(st)
    assert where > 0  # the wait that ran out names itself
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0  # the context is still usable
    kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], out, ws,
                      init_state=inp["init_state"], final_state=fin)
    st, _ = kda.kda_get_device_status(ws)
    assert st == kda.KDA_OK
    assert torch.equal(out, o_ref) and torch.equal(fin, S_ref)


# ------------------------------------------------- tensor-core path specifics

def _slow_decay(inp, shift=4.0):
    """Same draws with z shifted down: g close to 0, so memory spans many
    chunks and segment transitions M stay far from zero."""
    out = dict(inp)
    out["z"] = (inp["z"] - shift).contiguous()
    return out


@pytest.mark.parametrize("slow", [False, True])
def test_prefill_tc_segment_split(oracle_mod, slow):
    """B*H = 2 units over T = 5000 tokens: the tensor-core path splits each
    sequence into segments, computes their transitions, combines them and
    reruns the segments from the true incoming states."""
    inp = W.make_prefill_inputs(1, 5000, 2, 128, 128, torch.bfloat16, seed=31, device=DEV,
                                init_state=True)
    if slow:
        inp = _slow_decay(inp)
    o, S, _, ws = gpu_prefill(inp)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    o_ref, S_ref = oracle_prefill(oracle_mod, inp)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S


@pytest.mark.parametrize("T", [32, 33, 700])
def test_prefill_tc_slow_decay(oracle_mod, T):
    inp = _slow_decay(W.make_prefill_inputs(3, T, 2, 128, 128, torch.bfloat16, seed=40 + T,
                                            device=DEV, init_state=True))
    o, S, _, _ = gpu_prefill(inp, scale=0.5)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, scale=0.5)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S


def test_tc_matches_fp32_kernel():
    """Chunk-size / kernel consistency: tensor-core C = 32 against the fp32
    CUDA-core kernel at C = 64 on the same bf16 inputs."""
    inp = W.make_prefill_inputs(2, 257, 4, 128, 128, torch.bfloat16, seed=12, device=DEV,
                                init_state=True)
    o_tc, S_tc, _, _ = gpu_prefill(inp, chunk=0)
    o_64, S_64, _, _ = gpu_prefill(inp, chunk=64)
    assert rel_l2(to64(o_tc), to64(o_64)) <= TOL_BF16_O
    assert rel_l2(to64(S_tc), to64(S_64)) <= TOL_BF16_S


def test_tc_rerun_is_deterministic_and_input_sensitive():
    """Same inputs twice give bit-identical outputs; changing one value of v
    changes the output (no caching of results between calls)."""
    inp = W.make_prefill_inputs(1, 96, 2, 128, 128, torch.bfloat16, seed=13, device=DEV)
    o1, S1, _, _ = gpu_prefill(inp)
    o2, S2, _, _ = gpu_prefill(inp)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    inp["v"][0, 50, 1, 7] += 1.0
    o3, _, _, _ = gpu_prefill(inp)
    assert not torch.equal(o1[0, 50:, 1], o3[0, 50:, 1])
    assert torch.equal(o1[0, :50], o3[0, :50])


# ------------------------------------------------------------ fused gate

def _gated_prefill(inp, cu=None, chunk=0, scale=1.0):
    q, k, v, z, A_log, beta = (inp[n] for n in ("q", "k", "v", "z", "A_log", "beta"))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu is None else cu.numel() - 1
    out = torch.full((B, T, H, dv), float("nan"), device=q.device, dtype=q.dtype)
    fin = torch.full((N, H, dk, dv), float("nan"), device=q.device)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(
        B, T, H, dk, dv, 0 if cu is None else N, chunk,
        kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32), dtype=torch.uint8,
        device=q.device)
    kda.kda_chunk_fwd_gated(q, k, v, z, A_log, beta, out, ws, init_state=inp["init_state"],
                            cu_seqlens=cu, final_state=fin, scale=scale, chunk_size=chunk)
    assert kda.kda_get_device_status(ws)[0] == kda.KDA_OK
    return out, fin


def test_gated_prefill_fp32_tiny(oracle_mod):
    inp = W.make_prefill_inputs(1, 64, 2, 32, 32, torch.float32, seed=0, device=DEV)
    o, S = _gated_prefill(inp, chunk=16)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, with_init=False)
    assert rel_l2(to64(o), o_ref) <= TOL_F32
    assert rel_l2(to64(S), S_ref) <= TOL_F32


@pytest.mark.parametrize("B,T,H", [(2, 300, 3), (1, 5000, 2)])
def test_gated_prefill_bf16(oracle_mod, B, T, H):
    """Tensor-core path with the gate fused (the second case takes the
    segment-split route)."""
    inp = W.make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, seed=50 + T, device=DEV,
                                init_state=True)
    o, S = _gated_prefill(inp)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S
    o2, S2, _, _ = gpu_prefill(inp)  # unfused: gate kernel + chunk kernel
    assert rel_l2(to64(o), to64(o2)) <= 1e-2
    assert rel_l2(to64(S), to64(S2)) <= 1e-3


def test_gated_prefill_varlen(oracle_mod):
    lens = [5, 0, 130, 64, 33]
    cu_list = W.cu_seqlens_from_lengths(lens)
    inp = W.make_prefill_inputs(1, cu_list[-1], 2, 128, 128, torch.bfloat16, seed=61,
                                device=DEV, init_state=True, num_states=len(lens))
    cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    o, S = _gated_prefill(inp, cu=cu)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, cu=cu)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(S), S_ref) <= TOL_BF16_S


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gated_decode(oracle_mod, dtype):
    N, H, d, steps = 3, 4, 128, 5
    S0 = W.make_decode_state(N, H, d, d, 70, DEV)
    A_log = W.make_decode_gate_params(H, 71, DEV)
    state = S0.clone()
    xs, outs = [], []
    for s in range(steps):
        x = W.make_decode_step_inputs(N, H, d, d, dtype, 72 + s, DEV)
        o = torch.full((N, H, d), float("nan"), device=DEV, dtype=dtype)
        kda.kda_decode_step_gated(x["q"], x["k"], x["v"], x["z"], A_log, x["beta"], state, o)
        xs.append(x)
        outs.append(o)
    torch.cuda.synchronize()
    st = lambda n: torch.stack([x[n] for x in xs], dim=1)
    g_ref = oracle_mod.gate(to64(st("z")), to64(A_log), -5.0)
    o_ref, S_ref = oracle_mod.forward(to64(st("q")), to64(st("k")), to64(st("v")), g_ref,
                                      to64(st("beta")), init_state=to64(S0))
    tol_o, tol_s = (TOL_F32, TOL_F32) if dtype == torch.float32 else (TOL_BF16_O, TOL_BF16_S)
    assert rel_l2(to64(torch.stack(outs, 1)), o_ref) <= tol_o
    assert rel_l2(to64(state), S_ref) <= tol_s


# ------------------------------------------ speculative decoding: verify / replay

def _draft_inputs(N, K, H, dk, dv, dtype, seed):
    """K draft tokens per sequence ([N, K, H, *] layouts) and a committed state."""
    inp = W.make_prefill_inputs(N, K, H, dk, dv, dtype, seed=seed, device=DEV)
    S0 = W.make_decode_state(N, H, dk, dv, seed + 500, DEV)
    return inp, S0


@pytest.mark.parametrize("K", [1, 4, 16])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 32, torch.float32),
                                         (32, 128, torch.bfloat16)])
def test_decode_verify(oracle_mod, K, dk, dv, dtype):
    N, H = 3, 4
    inp, S0 = _draft_inputs(N, K, H, dk, dv, dtype, seed=90 + K)
    state = S0.clone()
    out = torch.full((N, K, H, dv), float("nan"), dtype=dtype, device=DEV)
    kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], state, out,
                          A_log=inp["A_log"], scale=0.8)
    torch.cuda.synchronize()
    assert torch.equal(state, S0)  # the committed state is only read
    g_ref = oracle_mod.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    o_ref, _ = oracle_mod.forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), g_ref,
                                  to64(inp["beta"]), init_state=to64(S0), scale=0.8)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16_O
    assert rel_l2(to64(out), o_ref) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_replay_accepted_prefix(oracle_mod, dtype):
    N, K, H, d = 5, 8, 3, 128
    inp, S0 = _draft_inputs(N, K, H, d, d, dtype, seed=120)
    accept = [0, 8, 3, 1, 5]
    acc = torch.tensor(accept, dtype=torch.int32, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    state = S0.clone()
    kda.kda_decode_replay(inp["k"], inp["v"], g, inp["beta"], state, acc)
    torch.cuda.synchronize()
    g_ref = oracle_mod.gate(to64(inp["z"]), to64(inp["A_log"]), -5.0)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16_S
    for n, m in enumerate(accept):
        if m == 0:
            assert torch.equal(state[n], S0[n])
            continue
        sl = lambda t: t[n:n + 1, :m]
        _, S_ref = oracle_mod.forward(to64(sl(inp["q"])), to64(sl(inp["k"])), to64(sl(inp["v"])),
                                      g_ref[n:n + 1, :m], to64(sl(inp["beta"])),
                                      init_state=to64(S0[n:n + 1]))
        assert rel_l2(to64(state[n]), S_ref[0]) <= tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_verify_replay_strong_decay(oracle_mod, dtype):
    """Raw log-decays down to -12 per token over 12 draft tokens (cumulative
    decays far below fp32's normal range) beside heads with mild decays in
    the same launch: outputs and replayed states against the oracle."""
    N, K, H, d = 3, 12, 4, 64
    inp, S0 = _draft_inputs(N, K, H, d, d, dtype, seed=140)
    gen = torch.Generator(device=DEV).manual_seed(141)
    g = -6.0 - 6.0 * torch.rand((N, K, H, d), generator=gen, device=DEV)
    g[:, :, 2:] *= 0.02  # heads 2, 3: cumulative decay stays well inside the range
    out = torch.full((N, K, H, d), float("nan"), dtype=dtype, device=DEV)
    kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], g, inp["beta"], S0, out, scale=0.9)
    state = S0.clone()
    acc = torch.tensor([K, 5, 1], dtype=torch.int32, device=DEV)
    kda.kda_decode_replay(inp["k"], inp["v"], g, inp["beta"], state, acc)
    torch.cuda.synchronize()
    o_ref, _ = oracle_mod.forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), to64(g),
                                  to64(inp["beta"]), init_state=to64(S0), scale=0.9)
    tol_o = TOL_F32 if dtype == torch.float32 else TOL_BF16_O
    tol_s = TOL_F32 if dtype == torch.float32 else TOL_BF16_S
    for h in range(H):
        assert rel_l2(to64(out[:, :, h]), o_ref[:, :, h]) <= tol_o, h
    for n, m in enumerate(acc.tolist()):
        sl = lambda t: t[n:n + 1, :m]
        _, S_ref = oracle_mod.forward(to64(sl(inp["q"])), to64(sl(inp["k"])), to64(sl(inp["v"])),
                                      to64(sl(g)), to64(sl(inp["beta"])),
                                      init_state=to64(S0[n:n + 1]))
        for h in range(H):
            assert rel_l2(to64(state[n, h]), S_ref[0, h]) <= tol_s, (n, h)


def test_verify_then_replay_equals_step_by_step():
    """verify(K) outputs and replay(K) state equal K single decode steps."""
    N, K, H, d = 4, 6, 2, 128
    inp, S0 = _draft_inputs(N, K, H, d, d, torch.bfloat16, seed=130)
    g = gpu_gate(inp["z"], inp["A_log"])
    out = torch.empty((N, K, H, d), dtype=torch.bfloat16, device=DEV)
    kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], g, inp["beta"], S0, out)
    state = S0.clone()
    kda.kda_decode_replay(inp["k"], inp["v"], g, inp["beta"], state,
                          torch.full((N,), K, dtype=torch.int32, device=DEV))
    ref_state = S0.clone()
    ref_out = []
    for t in range(K):
        o = torch.empty((N, H, d), dtype=torch.bfloat16, device=DEV)
        kda.kda_decode_step(inp["q"][:, t].contiguous(), inp["k"][:, t].contiguous(),
                            inp["v"][:, t].contiguous(), g[:, t].contiguous(),
                            inp["beta"][:, t].contiguous(), ref_state, o)
        ref_out.append(o)
    torch.cuda.synchronize()
    assert rel_l2(to64(out), to64(torch.stack(ref_out, 1))) <= 1e-2
    assert rel_l2(to64(state), to64(ref_state)) <= 1e-5
