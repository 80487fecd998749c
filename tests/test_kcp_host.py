"""Host logic of cross-device context parallelism (gated_delta_rule_158_b200.kcp),
on CPU: two gloo ranks, each holding one segment of a sequence, with the
compute steps done by the fp64 oracle, must reproduce one sequential oracle
run over the whole sequence (outputs of every segment, final state on the
last rank).  The identity checked is the KCP one of "NLP--技术报告解读-Kimi-K3"
(joezjh.github.io), Infrastructure > KDA kernels: S_end = S~ + M S_in."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_158_b200 import kcp


def test_segment_bounds_cover_in_order():
    for T, parts in [(1000, 2), (4096, 3), (31, 4), (0, 2), (64, 1), (33, 2)]:
        b = kcp.segment_bounds(T, parts)
        assert len(b) == parts and b[0][0] == 0 and b[-1][1] == T
        for (s0, e0), (s1, _) in zip(b, b[1:]):
            assert e0 == s1 and (e0 % 32 == 0 or e0 == T)
        assert all(e >= s for s, e in b)
    with pytest.raises(ValueError):
        kcp.segment_bounds(10, 0)


class OracleBackend:
    """kcp's three compute steps done by the fp64 oracle on CPU tensors."""

    pair_dtype = torch.float64

    def __init__(self, oracle):
        self.o = oracle

    def _g(self, seg):
        return self.o.gate(seg["z"].numpy(), seg["A_log"].numpy(), -5.0)

    def transition(self, seg):
        q, k, v, beta = (seg[n].numpy() for n in ("q", "k", "v", "beta"))
        B, T, H, dk = q.shape
        g = self._g(seg)
        _, St = self.o.forward(q, k, v, g, beta)
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, M = self.o.forward(q, k, np.zeros((B, T, H, dk)), g, beta, init_state=eye)
        return torch.from_numpy(np.stack([St, M], axis=2))

    def prefix(self, gathered, index, init_state):
        g = gathered.numpy()
        S = np.zeros(g.shape[1:3] + g.shape[-2:]) if init_state is None else init_state.numpy()
        for r in range(index):
            S = g[r, :, :, 0] + g[r, :, :, 1] @ S
        return torch.from_numpy(S)

    def forward(self, seg, state_in):
        q, k, v, beta = (seg[n].numpy() for n in ("q", "k", "v", "beta"))
        o, S = self.o.forward(q, k, v, self._g(seg), beta, init_state=state_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(S)


def _inputs(T=77, H=2, d=8, seed=5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, H, d))
    k = rng.standard_normal((1, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((1, T, H, d)),
                z=rng.standard_normal((1, T, H, d)), A_log=np.log(rng.uniform(1, 16, H)),
                beta=1 / (1 + np.exp(-rng.standard_normal((1, T, H)))),
                init=0.1 * rng.standard_normal((1, H, d, d)))


def _rank_main(rank, world, T, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        x = _inputs(T=T)
        s, e = kcp.segment_bounds(T, world)[rank]
        seg = {n: torch.from_numpy(np.ascontiguousarray(x[n][:, s:e])) for n in ("q", "k", "v", "z", "beta")}
        seg["A_log"] = torch.from_numpy(x["A_log"])
        o, S = kcp.kcp_prefill(seg, init_state=torch.from_numpy(x["init"]),
                               backend=OracleBackend(oracle))
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"S{rank}.npy"), S.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        return sck.getsockname()[1]


@pytest.mark.parametrize("world,T", [(2, 77), (3, 77), (4, 70)])
def test_kcp_ranks_match_one_sequential_run(tmp_path, oracle_mod, world, T):
    """T = 70 over 4 ranks leaves the last rank an empty segment."""
    mp.spawn(_rank_main, args=(world, T, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x = _inputs(T=T)
    g = oracle_mod.gate(x["z"], x["A_log"], -5.0)
    o_ref, S_ref = oracle_mod.forward(x["q"], x["k"], x["v"], g, x["beta"], init_state=x["init"])
    bounds = kcp.segment_bounds(x["q"].shape[1], world)
    for r, (s, e) in enumerate(bounds):
        o = np.load(tmp_path / f"o{r}.npy")
        np.testing.assert_allclose(o, o_ref[:, s:e], rtol=1e-9, atol=1e-11)
    S_last = np.load(tmp_path / f"S{world - 1}.npy")
    np.testing.assert_allclose(S_last, S_ref, rtol=1e-9, atol=1e-11)
