"""Cross-device context parallelism kernels on one GPU: a sequence cut into
three segments ("ranks" emulated in one process; the exchange is a stack)
must give the outputs and final state of one pass over the whole sequence.
The identity is the KCP one of "NLP--技术报告解读-Kimi-K3" (joezjh.github.io),
Infrastructure > KDA kernels: S_end = S~ + M S_in."""
import numpy as np
import pytest
import torch

import gated_delta_rule_158_b200 as kda
from gated_delta_rule_158_b200 import kcp
from gated_delta_rule_158_b200 import workloads as W

from kda_testutil import TOL_BF16_O, TOL_BF16_S, rel_l2, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _segments(inp, bounds):
    segs = []
    for s, e in bounds:
        seg = {n: inp[n][:, s:e].contiguous() for n in ("q", "k", "v", "z", "beta")}
        seg["A_log"] = inp["A_log"]
        segs.append(seg)
    return segs


def _single_pass(inp):
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    out = torch.empty_like(v)
    fin = torch.empty((B, H, dk, v.shape[-1]), device=DEV)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(B, T, H, dk, v.shape[-1]),
                     dtype=torch.uint8, device=DEV)
    kda.kda_chunk_fwd_gated(q, inp["k"], v, inp["z"], inp["A_log"], inp["beta"], out, ws,
                            init_state=inp["init_state"], final_state=fin)
    return out, fin


@pytest.mark.parametrize("T,R", [(3000, 3), (4096, 2)])
def test_kcp_segments_match_single_pass(oracle_mod, T, R):
    inp = W.make_prefill_inputs(1, T, 4, 128, 128, torch.bfloat16, seed=90 + R, device=DEV,
                                init_state=True)
    be = kcp.LibkdaBackend()
    bounds = kcp.segment_bounds(T, R)
    segs = _segments(inp, bounds)
    pairs = [be.transition(sg) for sg in segs[:-1]]
    pairs.append(torch.zeros_like(pairs[0]))
    gathered = torch.stack(pairs)
    outs, ends = [], []
    for r, sg in enumerate(segs):
        s_in = be.prefix(gathered, r, inp["init_state"])
        o, S = be.forward(sg, s_in)
        outs.append(o)
        ends.append((s_in, S))
    torch.cuda.synchronize()
    o_kcp = torch.cat(outs, dim=1)
    o_one, S_one = _single_pass(inp)
    assert rel_l2(to64(o_kcp), to64(o_one)) <= TOL_BF16_O
    assert rel_l2(to64(ends[-1][1]), to64(S_one)) <= TOL_BF16_S
    # each segment's end state from its own pair: S_end = S~ + M S_in
    for r in range(R - 1):
        St, M = to64(gathered[r, :, :, 0]), to64(gathered[r, :, :, 1])
        s_in, S_end = to64(ends[r][0]), to64(ends[r][1])
        assert rel_l2(St + M @ s_in, S_end) <= TOL_BF16_S, r
    # against the fp64 oracle over the whole sequence
    A = to64(inp["A_log"])
    g = oracle_mod.gate(to64(inp["z"]), A, -5.0)
    o_ref, S_ref = oracle_mod.forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), g,
                                      to64(inp["beta"]), init_state=to64(inp["init_state"]))
    assert rel_l2(to64(o_kcp), o_ref) <= TOL_BF16_O
    assert rel_l2(to64(ends[-1][1]), S_ref) <= TOL_BF16_S


def test_state_prefix_is_the_fold():
    """kda_chunk_state_prefix against the fold written out in fp64."""
    g = torch.Generator(device=DEV).manual_seed(7)
    count, B, H = 4, 2, 3
    pairs = torch.randn((count, B, H, 2, 128, 128), generator=g, device=DEV) * 0.05
    init = torch.randn((B, H, 128, 128), generator=g, device=DEV)
    for index in range(count):
        out = torch.empty((B, H, 128, 128), device=DEV)
        kda.kda_chunk_state_prefix(pairs, index, out, init_state=init)
        torch.cuda.synchronize()
        S = to64(init)
        P = to64(pairs)
        for r in range(index):
            S = P[r, :, :, 0] + P[r, :, :, 1] @ S
        assert rel_l2(to64(out), S) <= 1e-5, index
    out = torch.empty((B, H, 128, 128), device=DEV)
    kda.kda_chunk_state_prefix(pairs, 0, out)  # no initial state: zeros
    torch.cuda.synchronize()
    assert float(out.abs().max()) == 0.0
