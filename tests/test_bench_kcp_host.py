"""bench.py's context-parallel mode (--workload long --kcp) on CPU: two gloo
ranks build their segments with bench.kcp_segment_inputs and run
bench.KcpStep, with the fp64 oracle doing the compute steps.  The outputs of
both segments and the last rank's end state must equal one sequential oracle
run over the concatenated segments: the identity S_end = S~ + M S_in of
"NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Infrastructure > KDA kernels
(KCP)."""
import importlib.util
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WL = dict(name="long (tiny)", B=1, T=150, H=2, dk=8, dv=8, seed=2)


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class OracleBackend:
    """The three KCP compute steps by the fp64 oracle, on CPU tensors."""

    pair_dtype = torch.float64

    def __init__(self, oracle):
        self.o = oracle

    @staticmethod
    def _np(seg, n):
        return seg[n].double().numpy()

    def _g(self, seg):
        return self.o.gate(self._np(seg, "z"), self._np(seg, "A_log"), -5.0)

    def transition(self, seg):
        q, k, v, beta = (self._np(seg, n) for n in ("q", "k", "v", "beta"))
        B, T, H, dk = q.shape
        g = self._g(seg)
        _, St = self.o.forward(q, k, v, g, beta)
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, M = self.o.forward(q, k, np.zeros_like(v), g, beta, init_state=eye)
        return torch.from_numpy(np.stack([St, M], axis=2))

    def prefix(self, gathered, index, init_state):
        g = gathered.numpy()
        S = np.zeros(g.shape[1:3] + g.shape[-2:]) if init_state is None else init_state.numpy()
        for r in range(index):
            S = g[r, :, :, 0] + g[r, :, :, 1] @ S
        return torch.from_numpy(S)

    def forward(self, seg, state_in):
        q, k, v, beta = (self._np(seg, n) for n in ("q", "k", "v", "beta"))
        o, S = self.o.forward(q, k, v, self._g(seg), beta, init_state=state_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(S)


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        bench = _bench()
        seg, _ = bench.kcp_segment_inputs(WL, rank, world, "cpu", dtype=torch.float32)
        step = bench.KcpStep(seg, backend=OracleBackend(oracle))
        step()
        np.save(os.path.join(out_dir, f"o{rank}.npy"), step.o.numpy())
        np.save(os.path.join(out_dir, f"S{rank}.npy"), step.S.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        return sck.getsockname()[1]


def test_bench_kcp_step_two_ranks_match_sequential(tmp_path, oracle_mod):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    bench = _bench()
    segs = [bench.kcp_segment_inputs(WL, r, world, "cpu", dtype=torch.float32)[0]
            for r in range(world)]
    assert all(torch.equal(segs[0]["A_log"], s["A_log"]) for s in segs)  # one sequence
    full = {n: torch.cat([s[n] for s in segs], 1).double().numpy()
            for n in ("q", "k", "v", "z", "beta")}
    assert full["q"].shape[1] == WL["T"]
    g = oracle_mod.gate(full["z"], segs[0]["A_log"].double().numpy(), -5.0)
    o_ref, S_ref = oracle_mod.forward(full["q"], full["k"], full["v"], g, full["beta"])
    start = 0
    for r in range(world):
        o = np.load(tmp_path / f"o{r}.npy")
        np.testing.assert_allclose(o, o_ref[:, start:start + o.shape[1]], rtol=1e-9,
                                   atol=1e-11)
        start += o.shape[1]
    np.testing.assert_allclose(np.load(tmp_path / f"S{world - 1}.npy"), S_ref, rtol=1e-9,
                               atol=1e-11)
