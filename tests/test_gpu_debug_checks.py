"""The KDA_DEBUG_CHECKS build (libkda_debug.so) on the GPU.

Its device-side bounds checks record KDA_ERR_BOUNDS in the workspace status
word instead of trapping; the selftest makes one check fail (without any
memory access) and the context must stay usable.  On valid inputs the checks
never fire: every path (dense, packed, segment split, the fp32-accuracy
scans at d 64 and 128, backward at d 64 and 128 including its windowed
schedule) must report KDA_OK and give results bit-identical to the release
library's.
"""
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import gpu_gate

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _with(debug, fn):
    prev = kda.select_library(debug)
    try:
        return fn()
    finally:
        kda.select_library(prev.endswith("libkda_debug.so"))


def test_debug_selftest_records_bounds_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)

    def run():
        assert kda.kda_debug_checks_enabled()
        kda.kda_selftest_bounds_check(ws)
        torch.cuda.synchronize()
        return kda.kda_get_device_status(ws)

    st, detail = _with(True, run)
    assert st == kda.KDA_ERR_BOUNDS and detail == 0x5E1F
    x = torch.arange(1024, device=DEV, dtype=torch.float32)
    assert float(x.sum()) == 1023 * 1024 / 2  # the context still works
    assert not kda.kda_debug_checks_enabled()  # the release library is selected again


def _prefill(inp, cu=None, num_states=None):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    N = B if cu is None else cu.numel() - 1
    out = torch.full((B, T, H, dv), float("nan"), device=DEV, dtype=q.dtype)
    fin = torch.full((N, H, dk, dv), float("nan"), device=DEV)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(
        B, T, H, dk, dv, 0 if cu is None else N, 0,
        kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32), dtype=torch.uint8,
        device=DEV)
    kda.kda_chunk_fwd_gated(q, inp["k"], inp["v"], inp["z"], inp["A_log"], inp["beta"], out, ws,
                            init_state=inp["init_state"], cu_seqlens=cu, final_state=fin)
    torch.cuda.synchronize()
    return out, fin, kda.kda_get_device_status(ws)


@pytest.mark.parametrize("case", ["dense", "varlen", "split", "fp32", "fp32_128"])
def test_debug_build_prefill_matches_release(case):
    cu = None
    if case == "dense":
        inp = W.make_prefill_inputs(2, 300, 4, 128, 128, torch.bfloat16, seed=61, device=DEV,
                                    init_state=True)
    elif case == "varlen":
        lengths = [0, 1, 31, 33, 700, 64, 5]
        cu_list = W.cu_seqlens_from_lengths(lengths)
        inp = W.make_prefill_inputs(1, cu_list[-1], 4, 128, 128, torch.bfloat16, seed=62,
                                    device=DEV, init_state=True, num_states=len(lengths))
        cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    elif case == "split":  # B*H*2 < SMs and T >= 4096: the segment split
        inp = W.make_prefill_inputs(1, 9000, 2, 128, 128, torch.bfloat16, seed=63, device=DEV,
                                    init_state=True)
    elif case == "fp32":  # fp32 inputs, d 64: the warp-MMA scan
        inp = W.make_prefill_inputs(2, 130, 3, 64, 64, torch.float32, seed=64, device=DEV,
                                    init_state=True)
    else:  # fp32 inputs, d 128: the tcgen05 scan
        inp = W.make_prefill_inputs(2, 130, 3, 128, 128, torch.float32, seed=65, device=DEV,
                                    init_state=True)
    o_r, f_r, st_r = _with(False, lambda: _prefill(inp, cu))
    o_d, f_d, st_d = _with(True, lambda: _prefill(inp, cu))
    assert st_r[0] == kda.KDA_OK and st_d[0] == kda.KDA_OK, (st_r, st_d)
    assert torch.equal(o_d, o_r) and torch.equal(f_d, f_r)


def _backward(inp, cot, g, cu=None, N=None):
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if N is None else N
    nan = lambda *s: torch.full(s, float("nan"), device=DEV)
    grads = dict(dq=nan(B, T, H, dk), dk=nan(B, T, H, dk), dv=nan(B, T, H, dv),
                 dg=nan(B, T, H, dk), dbeta=nan(B, T, H), d_init=nan(N, H, dk, dv))
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(B, T, H, dk, dv,
                                                          0 if cu is None else N),
                     dtype=torch.uint8, device=DEV)
    kda.kda_recurrent_bwd(q, inp["k"], v, g, inp["beta"], cot["dout"], grads, ws,
                          init_state=inp["init_state"], d_final=cot["d_final"], cu_seqlens=cu)
    torch.cuda.synchronize()
    return grads, kda.kda_get_device_status(ws)


@pytest.mark.parametrize("case", ["dense", "dense128", "varlen", "windowed"])
def test_debug_build_backward_matches_release(case):
    cu, N = None, None
    if case == "dense":
        B, T, H, d = 2, 150, 3, 64
    elif case == "dense128":  # the tcgen05 scans and token-gradient products
        B, T, H, d = 2, 150, 3, 128
    elif case == "windowed":  # longer than one 8192-token window
        B, T, H, d = 1, 9000, 1, 32
    else:
        lengths = [0, 1, 31, 32, 100, 7]
        cu_list = W.cu_seqlens_from_lengths(lengths)
        B, T, H, d, N = 1, cu_list[-1], 2, 64, len(lengths)
        cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=71, device=DEV,
                                init_state=True, num_states=N or B)
    cot = W.make_backward_cotangents(B, T, H, d, dk=None, dtype=torch.bfloat16, seed=72,
                                     device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(73)
    cot["d_final"] = 0.1 * torch.randn((N or B, H, d, d), generator=gen, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    gr, st_r = _with(False, lambda: _backward(inp, cot, g, cu, N))
    gd, st_d = _with(True, lambda: _backward(inp, cot, g, cu, N))
    assert st_r[0] == kda.KDA_OK and st_d[0] == kda.KDA_OK, (st_r, st_d)
    for name in gr:
        assert torch.equal(gd[name], gr[name]), name
