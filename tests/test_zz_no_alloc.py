"""kda_chunk_fwd_noalloc: the chunkwise forward for callers that cannot
allocate device memory (it uses a scratch array built into libkda instead of
a caller workspace).

Both entry points run the same deterministic kernels, so the outputs must be
bit-identical to kda_chunk_fwd's (given a workspace) on the same inputs, call
after call: the built-in scratch keeps the previous call's contents, so two
calls in a row are checked, and stale scratch (a varlen order or segment
states left by an earlier call) would show as a difference.  Cases cover the
three users of the scratch: the status word (every call, read back through
kda_noalloc_get_device_status), the varlen processing order, and the segment
states of the long-sequence split.  This file sorts last so that a failure
here does not stop the rest of a `-x` run.
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


def _with_workspace(inp, g, cu):
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    N = B if cu is None else cu.numel() - 1
    out = torch.empty((B, T, H, v.shape[-1]), dtype=q.dtype, device=DEV)
    fin = torch.empty((N, H, dk, v.shape[-1]), device=DEV)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(B, T, H, dk, v.shape[-1],
                                                      0 if cu is None else N),
                     dtype=torch.uint8, device=DEV)
    kda.kda_chunk_fwd(inp["q"], inp["k"], v, g, inp["beta"], out, ws,
                      init_state=inp["init_state"], cu_seqlens=cu, final_state=fin)
    return out, fin


def _noalloc(inp, g, cu):
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    N = B if cu is None else cu.numel() - 1
    out = torch.full((B, T, H, v.shape[-1]), float("nan"), dtype=q.dtype, device=DEV)
    fin = torch.full((N, H, dk, v.shape[-1]), float("nan"), device=DEV)
    kda.kda_chunk_fwd_noalloc(inp["q"], inp["k"], v, g, inp["beta"], out,
                              init_state=inp["init_state"], cu_seqlens=cu, final_state=fin)
    return out, fin


@pytest.mark.parametrize("case", ["dense", "varlen", "split"])
def test_noalloc_matches_workspace_entry_two_calls(case):
    cu = None
    if case == "dense":
        inp = W.make_prefill_inputs(2, 300, 3, 128, 128, torch.bfloat16, seed=81, device=DEV,
                                    init_state=True)
    elif case == "varlen":
        lens = [7, 0, 200, 64, 33]
        cu_list = W.cu_seqlens_from_lengths(lens)
        inp = W.make_prefill_inputs(1, cu_list[-1], 2, 128, 128, torch.bfloat16, seed=82,
                                    device=DEV, init_state=True, num_states=len(lens))
        cu = torch.tensor(cu_list, dtype=torch.int32, device=DEV)
    else:  # 2 (sequence, head) units over 5000 tokens: segment split in the scratch
        inp = W.make_prefill_inputs(1, 5000, 2, 128, 128, torch.bfloat16, seed=83, device=DEV,
                                    init_state=True)
    g = gpu_gate(inp["z"], inp["A_log"])
    o_ref, S_ref = _with_workspace(inp, g, cu)
    for _ in range(2):
        o, S = _noalloc(inp, g, cu)
        st, _ = kda.kda_noalloc_get_device_status()
        assert st == kda.KDA_OK, kda.kda_status_string(st)
        assert torch.equal(o, o_ref)
        assert torch.equal(S, S_ref)


def test_noalloc_reports_malformed_offsets_then_recovers():
    """Offsets that are not monotone: the plan kernel records
    KDA_ERR_BAD_SEQLENS in the built-in scratch and no unit runs; the status
    reader returns it, and the next (valid) call starts from a clean status."""
    T, H, d = 96, 2, 128
    inp = W.make_prefill_inputs(1, T, H, d, d, torch.bfloat16, seed=84, device=DEV)
    g = gpu_gate(inp["z"], inp["A_log"])
    bad = torch.tensor([0, 50, 40, 96], dtype=torch.int32, device=DEV)
    o, _ = _noalloc(inp, g, bad)
    st, _ = kda.kda_noalloc_get_device_status()
    assert st == kda.KDA_ERR_BAD_SEQLENS
    assert torch.isnan(o.float()).all()  # nothing was written
    good = torch.tensor([0, 40, 96], dtype=torch.int32, device=DEV)
    o_ref, S_ref = _with_workspace(inp, g, good)
    o, S = _noalloc(inp, g, good)
    st, _ = kda.kda_noalloc_get_device_status()
    assert st == kda.KDA_OK
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_noalloc_rejects_oversized_problem():
    """A million-token sequence over 32 heads needs ~12 MB of segment states,
    more than the built-in scratch: rejected before anything is enqueued."""
    need = kda.kda_chunk_fwd_workspace_size(1, 1 << 20, 32, 128, 128)
    assert need > (8 << 20)
    L = kda.lib()
    fake = 0x7F0000000000
    st = L.kda_chunk_fwd_noalloc(fake, fake + 0x1000, fake + 0x2000, fake + 0x3000,
                                 fake + 0x4000, kda.KDA_BF16, None, None, 0, 1, 1 << 20, 32,
                                 128, 128, 1.0, 0, fake + 0x5000, None, None)
    assert st == kda.KDA_ERR_WORKSPACE
