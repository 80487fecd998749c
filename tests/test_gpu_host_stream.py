"""GPU parity of the host-buffer prefill (kda_chunk_fwd_gated_host): inputs in
page-locked host memory, streamed through the device in time slices with the
state carried across slices.  Checked against the fp64 oracle (the parity
bars: rel-L2 1e-5 for fp32 inputs, 2e-2 on o and 1e-2 on the final state for
bf16 inputs) and against the device-buffer entry on the same inputs.
Outputs start as NaN, so an element never copied back fails."""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import TOL_BF16_O, TOL_BF16_S, TOL_F32, oracle_prefill, rel_l2, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def host_run(inp, with_init, want_final=True, overlap=True):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    pin = lambda t: None if t is None else t.cpu().pin_memory()
    h = {n: pin(t) for n, t in inp.items()}
    out = torch.full((B, T, H, dv), float("nan"), dtype=q.dtype).pin_memory()
    fin = torch.full((B, H, dk, dv), float("nan")).pin_memory() if want_final else None
    dt = kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32
    ws = torch.empty(kda.kda_chunk_fwd_gated_host_workspace_size(B, T, H, dk, dv, dt),
                     dtype=torch.uint8, device=DEV)
    cs = torch.cuda.Stream()
    xs = torch.cuda.Stream() if overlap else None
    kda.kda_chunk_fwd_gated_host(h["q"], h["k"], h["v"], h["z"], h["A_log"], h["beta"], out, ws,
                                 init_state=h["init_state"] if with_init else None,
                                 final_state=fin, stream=cs, copy_stream=xs)
    cs.synchronize()
    st, _ = kda.kda_get_device_status(ws, stream=cs)
    assert st == kda.KDA_OK
    return out, fin


def device_run(inp, with_init):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=DEV)
    fin = torch.empty((B, H, dk, dv), device=DEV)
    dt = kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(B, T, H, dk, dv, 0, 0, dt),
                     dtype=torch.uint8, device=DEV)
    kda.kda_chunk_fwd_gated(q, inp["k"], inp["v"], inp["z"], inp["A_log"], inp["beta"], out, ws,
                            init_state=inp["init_state"] if with_init else None,
                            final_state=fin)
    torch.cuda.synchronize()
    return out, fin


@pytest.mark.parametrize("B,T,H,d,dtype,init,overlap", [
    (2, 3000, 3, 128, torch.bfloat16, True, True),   # 6 slices of 512, last 440
    (1, 2500, 4, 128, torch.bfloat16, False, True),  # one sequence: per-sequence copies
    (3, 700, 2, 64, torch.float32, True, True),      # a single slice
    (2, 1100, 2, 32, torch.float32, False, False),   # 3 slices, no copy stream
])
def test_host_stream_parity(oracle_mod, B, T, H, d, dtype, init, overlap):
    inp = W.make_prefill_inputs(B, T, H, d, d, dtype, seed=T + d, device=DEV, init_state=True)
    out, fin = host_run(inp, init, overlap=overlap)
    o_ref, S_ref = oracle_prefill(oracle_mod, inp, with_init=init)
    tol_o, tol_s = (TOL_F32, TOL_F32) if dtype == torch.float32 else (TOL_BF16_O, TOL_BF16_S)
    assert np.isfinite(to64(out)).all() and np.isfinite(to64(fin)).all()
    assert rel_l2(to64(out), o_ref) <= tol_o
    assert rel_l2(to64(fin), S_ref) <= tol_s
    # the same kernels on device buffers, one launch over the whole length
    o_dev, f_dev = device_run(inp, init)
    assert rel_l2(to64(out), to64(o_dev)) <= tol_o
    assert rel_l2(to64(fin), to64(f_dev)) <= tol_s


def test_host_stream_without_final_state(oracle_mod):
    inp = W.make_prefill_inputs(2, 1500, 2, 64, 64, torch.float32, seed=8, device=DEV)
    out, fin = host_run(inp, False, want_final=False)
    assert fin is None
    o_ref, _ = oracle_prefill(oracle_mod, inp, with_init=False)
    assert rel_l2(to64(out), o_ref) <= TOL_F32
