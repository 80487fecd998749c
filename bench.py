"""Benchmark of the KDA hot path on B200 through libkda's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libkda|reference]
                    [--workload prefill|long|varlen|decode] [--no-cpu-baseline]

A step is one pass of the path over one batch of synthetic inputs already
resident in HBM: the gate (g = -5 sigmoid(e^A z)) then the chunkwise forward
for the prefill workloads; gate + decode step for the decode workload.  The
default workload is the dense prefill B=8, H=32, T=4096, dk=dv=128 (bf16
q/k/v, fp32 g/beta/state); its line also carries the decode workload
(256 sequences x 32 heads, 1024 consecutive steps) as a secondary figure.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and torch.cuda.synchronize(), with CUDA events on the launching stream; the
per-kernel durations that feed the roofline come from events around each
launch on the same stream.  Inputs are larger than L2 (126 MB), so no flush
is needed.  Under torchrun every rank runs its own batch (weak scaling, no
collective on the data path); the step time is the max over ranks.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (the slow baseline), printing the same JSON keys.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gated_delta_rule_158_b200 as kda  # noqa: E402
from gated_delta_rule_158_b200 import kcp  # noqa: E402
from gated_delta_rule_158_b200 import workloads as W  # noqa: E402

METRIC = "KDA prefill Mtokens/s & decode steps/s on 1 B200; % of TC / HBM roofline"

WORKLOADS = {
    "prefill": dict(name="prefill B8 H32 T4096 d128", B=8, T=4096, H=32, dk=128, dv=128,
                    seed=1, init=False, varlen=False),
    "long": dict(name="long prefill B1 H32 T1048576 d128", B=1, T=1048576, H=32, dk=128,
                 dv=128, seed=2, init=False, varlen=False),
    "varlen": dict(name="varlen 64 seqs log-uniform[128,32768] H16 d128", B=1, T=None, H=16,
                   dk=128, dv=128, seed=3, init=True, varlen=True, num_seqs=64),
    "decode": dict(name="decode N256 H32 d128 x1024 steps", N=256, H=32, dk=128, dv=128,
                   steps=1024, seed=4),
    "backward": dict(name="backward B8 H32 T4096 d128", B=8, T=4096, H=32, dk=128, dv=128,
                     seed=3, varlen=False),
    "spec_decode": dict(name="speculative verify/replay N256 H32 d128, K=4 draft tokens", N=256,
                        H=32, dk=128, dv=128, K=4, seed=7),
    # fp32 inputs take the CUDA-core chunk kernel (the tensor-core one is bf16)
    "prefill_fp32": dict(name="prefill fp32 B8 H32 T4096 d128", B=8, T=4096, H=32, dk=128,
                         dv=128, seed=1, init=False, varlen=False, dtype="f32"),
}

# bytes per (token, head) of the chunkwise forward, bf16 q/k/v/o, fp32 g/beta:
# q, k, v 3*256 + g 512 + beta 4 + o 256
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 256 + 512 + 4 + 256


def prefill_bytes_per_token_head(wl):
    """Algorithmic bytes per (token, head) at d = 128: q, k, v, o in the
    input type (2 or 4 bytes), z fp32, beta fp32."""
    if wl.get("dtype", "bf16") == "f32":
        return 4 * 512 + 512 + 4
    return PREFILL_BYTES_PER_TOKEN_HEAD


def wl_torch_dtype(wl):
    return torch.float32 if wl.get("dtype", "bf16") == "f32" else torch.bfloat16
# FLOPs per (token, head) of the chunk form counted once:
# C(3dk + 2dv) + C^2/3 + 6 dk dv.  The tensor-core kernel runs C = 32
# (118,869 at d = 128); the reference count of the measurement plan is taken
# at C = 64 (140,629).  Both are reported.
def prefill_flops_per_token_head(C=32, dk=128, dv=128):
    return C * (3 * dk + 2 * dv) + C * C / 3 + 6 * dk * dv


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one
# chunk_tc_kernel launch, from the ncu capture summarised in
# profiles/chunk_tc_kernel_prefill_B4_H32_T4096.md (128 (sequence, head) units
# of 4096 tokens): 673.5 MB read + 123.2 MB written.  Traffic grows with the
# units a launch processes, so a launch over U such units moves U times the
# per-unit figure.  The figure belongs to the kernel it was taken on: the
# text of kda_chunk_tc.cu up to the end of chunk_tc_kernel (its constants,
# structures and body) and the headers it includes.  Once those change it is
# reported as null until a new capture replaces it.
CHUNK_TRAFFIC = {
    "kernel_file": "gated_delta_rule_158_b200/csrc/kda_chunk_tc.cu",
    "kernel_end_marker": "\n// S_in[g+1] = S~_g + M_g S_in[g]",
    "headers": ["gated_delta_rule_158_b200/csrc/kda_sync.cuh",
                "gated_delta_rule_158_b200/csrc/kda_tc_ptx.cuh",
                "gated_delta_rule_158_b200/csrc/kda_internal.cuh"],
    "sha256": "efbf25df15e88cb84589ea19899855a0296fe8561a4a80db777c9b6b8b91a649",
    "bytes_per_unit_T4096": (673.389824e6 + 122.219776e6) / 128,
}


def chunk_kernel_source_hash():
    with open(os.path.join(ROOT, CHUNK_TRAFFIC["kernel_file"]), encoding="utf-8") as fh:
        text = fh.read()
    end = text.find(CHUNK_TRAFFIC["kernel_end_marker"])
    if end < 0:
        return None
    h = hashlib.sha256(text[:end].encode("utf-8"))
    for f in CHUNK_TRAFFIC["headers"]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def chunk_traffic(B, H, T):
    if T != 4096 or chunk_kernel_source_hash() != CHUNK_TRAFFIC["sha256"]:
        return None
    return round(B * H * CHUNK_TRAFFIC["bytes_per_unit_T4096"])


def kernels_per_step(wl, B, T):
    """libkda kernels one prefill step launches: one chunk kernel; the varlen
    plan kernel in front for varlen; three (transitions, combine, outputs)
    when the long-sequence split applies (B*H*2 < SMs and T >= 4096); two
    (key-side pass, scan) for fp32 inputs."""
    if wl.get("varlen"):
        return 2
    if wl.get("dtype", "bf16") == "f32":  # key-side pass, then the scan
        return 2
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if 2 * B * wl["H"] < sms and T >= 4096:
        return 3
    return 1


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], tc=d["bf16_tflops"], tc_sustained=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, src="fallback")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def extend_window(self, step, min_s=1.5):
        """The timed region can be shorter than nvidia-smi's start-up and its
        50 ms period: keep running the same (untimed) step until the sampling
        window spans min_s seconds, then stop and summarise."""
        t0 = time.time()
        n = 0
        while time.time() - t0 < min_s:
            step()
            n += 1
            if n % 8 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        out = self.stop()
        if out is not None:
            out["window"] = f"timed region + {n} further untimed steps ({min_s:.1f} s)"
        return out

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():  # the reference arm also runs on a host without a GPU
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- prefill
def make_prefill(wl, device):
    if wl["varlen"]:
        lens = W.varlen_lengths(wl["num_seqs"], wl["seed"])
        cu_list = W.cu_seqlens_from_lengths(lens)
        T = cu_list[-1]
        inp = W.make_prefill_inputs(1, T, wl["H"], wl["dk"], wl["dv"], torch.bfloat16,
                                    seed=wl["seed"], device=device, init_state=True,
                                    num_states=wl["num_seqs"])
        cu = torch.tensor(cu_list, dtype=torch.int32, device=device)
        return inp, cu, T, wl["num_seqs"]
    inp = W.make_prefill_inputs(wl["B"], wl["T"], wl["H"], wl["dk"], wl["dv"], wl_torch_dtype(wl),
                                seed=wl["seed"], device=device, init_state=wl["init"])
    return inp, None, wl["T"], wl["B"]


class PrefillStep:
    """One step: kda_chunk_fwd_gated (gate fused into the chunk kernel) on
    resident inputs, with events around the launch."""

    def __init__(self, inp, cu, N):
        self.inp, self.cu = inp, cu
        q = inp["q"]
        B, T, H, dk = q.shape
        dv = inp["v"].shape[-1]
        self.out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
        self.final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
        nbytes = kda.kda_chunk_fwd_workspace_size(
            B, T, H, dk, dv, 0 if cu is None else N, 0,
            kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device)

    def __call__(self, ev=None):
        i = self.inp
        if ev:
            ev[0].record()
        kda.kda_chunk_fwd_gated(i["q"], i["k"], i["v"], i["z"], i["A_log"], i["beta"], self.out,
                                self.ws, init_state=i["init_state"], cu_seqlens=self.cu,
                                final_state=self.final)
        if ev:
            ev[1].record()


def time_steps(step, K, Wm, world):
    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record()
    for k in range(K):
        step(evs[k])
    stop.record()
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(stop)
    chunk_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    barrier(world)
    return max_over_ranks(total_ms, world), chunk_ms


def e2e_prefill_host_entry(inp, K):
    """Dense batches: one kda_chunk_fwd_gated_host call per step on page-locked
    host buffers (the library streams the batch through the device in time
    slices, copies in both directions overlapping the kernels).  The timed
    region holds every step's host-to-device copies of q, k, v, z, beta (and
    A_log, init_state) and the device-to-host copies of o and the final state."""
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
    q = host["q"]
    B, T, H, dk = q.shape
    dv = host["v"].shape[-1]
    out_h = torch.empty((B, T, H, dv), dtype=q.dtype).pin_memory()
    fin_h = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    dt = kda.KDA_BF16 if q.dtype == torch.bfloat16 else kda.KDA_F32
    ws = torch.empty(kda.kda_chunk_fwd_gated_host_workspace_size(B, T, H, dk, dv, dt),
                     dtype=torch.uint8, device=inp["q"].device)
    cs, xs = torch.cuda.Stream(), torch.cuda.Stream()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_h.numel() * out_h.element_size() + fin_h.numel() * 4

    def one():
        kda.kda_chunk_fwd_gated_host(host["q"], host["k"], host["v"], host["z"], host["A_log"],
                                     host["beta"], out_h, ws, init_state=host["init_state"],
                                     final_state=fin_h, stream=cs, copy_stream=xs)

    one()
    cs.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(cs)
    for _ in range(K):
        one()
    b.record(cs)
    b.synchronize()
    st, _ = kda.kda_get_device_status(ws, stream=cs)
    if st != kda.KDA_OK:
        raise RuntimeError(f"device status {kda.kda_status_string(st)}")
    return a.elapsed_time(b) / K, h2d, d2h


def e2e_prefill(wl, inp, cu, N, K):
    """Same step through the public API with host buffers: H2D of the step's
    inputs from pinned memory, gate + chunk_fwd, D2H of o and final state."""
    if cu is None:
        return e2e_prefill_host_entry(inp, K)
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
    dev = {k: (torch.empty_like(v) if v is not None else None) for k, v in inp.items()}
    step = PrefillStep(dev, cu, N)
    out_h = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    fin_h = torch.empty(step.final.shape, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_h.numel() * out_h.element_size() + fin_h.numel() * 4

    def one():
        for k, v in host.items():
            if v is not None:
                dev[k].copy_(v, non_blocking=True)
        step()
        out_h.copy_(step.out, non_blocking=True)
        fin_h.copy_(step.final, non_blocking=True)

    one()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(K):
        one()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / K, h2d, d2h


# --------------------------------------------- context parallelism (KCP)
def kcp_segment_inputs(wl, rank, world, device, dtype=torch.bfloat16):
    """This rank's segment of the long workload's sequence (whole 32-token
    chunks in token order, kcp.segment_bounds).  Each rank draws only its own
    segment (seed derived from the rank), with the workload's shapes and
    distributions; the per-head gate parameter A_log is drawn from a seed
    shared by all ranks, as one sequence has one A_log."""
    s, e = kcp.segment_bounds(wl["T"], world)[rank]
    seg = W.make_prefill_inputs(1, e - s, wl["H"], wl["dk"], wl["dv"], dtype,
                                seed=wl["seed"] * 1000 + 1 + rank, device=device)
    shared = W.make_prefill_inputs(1, 1, wl["H"], wl["dk"], wl["dv"], dtype,
                                   seed=wl["seed"] * 1000, device=device)
    seg["A_log"] = shared["A_log"]
    return seg, (s, e)


class KcpStep:
    """One step of the long workload split across the ranks: kcp_prefill on
    this rank's segment (segment transition, one all-gather of the pairs,
    prefix fold, segment outputs)."""

    def __init__(self, seg, backend=None, group=None):
        self.seg, self.backend, self.group = seg, backend, group
        self.o = self.S = None

    def __call__(self, ev=None):
        if ev:
            ev[0].record()
        self.o, self.S = kcp.kcp_prefill(self.seg, init_state=None, group=self.group,
                                         backend=self.backend)
        if ev:
            ev[1].record()


def bench_kcp_line(args, wl, world, rank, peaks):
    dev = torch.device("cuda", torch.cuda.current_device())
    if world == 1:  # kcp_prefill needs a process group, even of one rank
        import datetime
        import torch.distributed as dist
        if not dist.is_initialized():
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29533")
            dist.init_process_group("nccl", rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=120),
                                    device_id=dev)
    seg, (s, e) = kcp_segment_inputs(wl, rank, world, dev)
    step = KcpStep(seg)
    clocks = None if args.no_clocks else ClockSampler(dev.index)
    total_ms, step_ms = time_steps(step, args.steps, args.warmup, world)
    clk = clocks.stop() if clocks else None
    step_ms = max_over_ranks(step_ms, world)
    ms = total_ms / args.steps
    T, H, dk, dv = wl["T"], wl["H"], wl["dk"], wl["dv"]
    alg = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + H * dk * dv * 4
    ach = alg / (step_ms * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": round(T / (ms * 1e-3) / 1e6, 3), "unit": "Mtokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (each rank draws its own segment)",
        "config": {"workload": wl["name"] + " (KCP)", "global_batch": 1, "seq_len": T,
                   "heads": H, "dk": dk, "dv": dv,
                   "parallelism": f"kcp{world} (one sequence split over the ranks; "
                                  "one all-gather of 2 x 64 KB per head per rank)",
                   "l2": "inputs larger than L2 (no flush needed)",
                   "step": "kcp.kcp_prefill: kda_chunk_segment_transition, all_gather, "
                           "kda_chunk_state_prefix, kda_chunk_fwd_gated"},
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"] * world,
                     "unit": "GB/s", "frac": round(ach / (peaks["hbm"] * world), 4),
                     "traffic": None, "kernel": "whole KCP step, all ranks",
                     "kernel_ms": round(step_ms, 4), "algorithmic_bytes": alg,
                     "peak_source": peaks["src"] + " (x ranks)"},
        "gpu_launches": args.steps * ((2 if world > 1 else 0) + 1 + 3),
        "clocks": clk,
    }


# ----------------------------------------------------------------- decode
def run_decode(wl, device, warmup=3):
    N, H, dk, dv, steps = wl["N"], wl["H"], wl["dk"], wl["dv"], wl["steps"]
    state = W.make_decode_state(N, H, dk, dv, wl["seed"], device)
    A_log = W.make_decode_gate_params(H, wl["seed"] + 1000, device)
    # all steps' inputs resident before timing (fresh inputs per step)
    xs = [W.make_decode_step_inputs(N, H, dk, dv, torch.bfloat16, wl["seed"] + s, device)
          for s in range(steps)]
    o = torch.empty((N, H, dv), dtype=torch.bfloat16, device=device)

    def step(x, ev=None):
        if ev:
            ev[0].record()
        kda.kda_decode_step_gated(x["q"], x["k"], x["v"], x["z"], A_log, x["beta"], state, o)
        if ev:
            ev[1].record()

    for s in range(warmup):
        step(xs[s])
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for s in range(steps):
        step(xs[s], evs[s])
    b.record()
    torch.cuda.synchronize()
    total_ms = a.elapsed_time(b)
    dec_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    bytes_per_launch = N * H * (2 * dk * dv * 4 + (2 * dk + dv) * 2 + dk * 4 + 4 + dv * 2)
    return total_ms, dec_ms, bytes_per_launch


def run_spec_decode(device, N=256, H=32, d=128, K=4, reps=50, seed=7):
    """Speculative decoding: verify K draft tokens per sequence (state read
    once, outputs for every token), then replay all K accepted tokens into the
    state.  Returns per-launch times and algorithmic bytes."""
    inp = W.make_prefill_inputs(N, K, H, d, d, torch.bfloat16, seed=seed, device=device)
    state = W.make_decode_state(N, H, d, d, seed + 1, device)
    out = torch.empty((N, K, H, d), dtype=torch.bfloat16, device=device)
    acc = torch.full((N,), K, dtype=torch.int32, device=device)

    def verify():
        kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], state, out,
                              A_log=inp["A_log"])

    def replay():
        kda.kda_decode_replay(inp["k"], inp["v"], inp["z"], inp["beta"], state, acc,
                              A_log=inp["A_log"])

    res = {}
    for name, fn in (("verify", verify), ("replay", replay)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        res[name] = a.elapsed_time(b) / reps
    per_head_in = K * (3 * d * 2 + d * 4 + 4)        # q, k, v bf16; z fp32; beta
    bytes_verify = N * H * (d * d * 4 + per_head_in + K * d * 2)   # state read, o written
    bytes_replay = N * H * (2 * d * d * 4 + per_head_in - K * d * 2)  # no q, state r+w
    return res, bytes_verify, bytes_replay, K


# --------------------------------------------------------------- backward
# Algorithmic bytes of the backward per token-head at d = 128 with bf16 q, k,
# v, dout: those four read (4 x 256 B), g fp32 read (512 B), beta (4 B), and
# dq, dk, dg, dv fp32 written (4 x 512 B), dbeta (4 B).
BWD_BYTES_PER_TOKEN_HEAD = 4 * 256 + 512 + 4 + 4 * 512 + 4


def oracle_backward_sample(T=4096, d=128, budget_s=8.0, seed=3):
    """The oracle's backward on whole (sequence, head) units of the backward
    workload's shape, one after another until the budget is spent; returns
    Mtokens/s counted like the GPU line (a position with all 32 heads is one
    token), the cores used and a description of the sample."""
    import oracle
    inp = W.make_prefill_inputs(1, T, 1, d, d, torch.bfloat16, seed=seed, init_state=True)
    cot = W.make_backward_cotangents(1, T, 1, d, dk=d, seed=seed + 1)
    f = lambda t: t.to(torch.float64).numpy()
    g = oracle.gate(f(inp["z"]), f(inp["A_log"]), -5.0)
    t0 = time.perf_counter()
    units = 0
    while True:
        oracle.backward(f(inp["q"]), f(inp["k"]), f(inp["v"]), g, f(inp["beta"]),
                        f(cot["dout"]), init_state=f(inp["init_state"]),
                        d_final=f(cot["d_final"]))
        units += 1
        secs = time.perf_counter() - t0
        if secs >= budget_s:
            break
    value = units * T / 32 / secs / 1e6
    return value, 1, f"{units} (sequence, head) units x {T} tokens, one thread", secs


def run_backward(device, B=8, H=32, T=4096, d=128, reps=3, seed=3):
    """kda_recurrent_bwd on the prefill workload's shape (bf16 inputs, with an
    initial state and a final-state gradient).  Returns the per-launch time
    and the algorithmic bytes of one launch (states read and written once)."""
    inp = W.make_prefill_inputs(B, T, H, d, d, torch.bfloat16, seed=seed, device=device,
                                init_state=True)
    cot = W.make_backward_cotangents(B, T, H, d, dk=d, seed=seed + 1, device=device)
    g = torch.empty_like(inp["z"])
    kda.kda_gate_fwd(inp["z"], inp["A_log"], g)
    f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=device)
    grads = dict(dq=f32(B, T, H, d), dk=f32(B, T, H, d), dv=f32(B, T, H, d),
                 dg=f32(B, T, H, d), dbeta=f32(B, T, H), d_init=f32(B, H, d, d))
    ws = torch.empty(kda.kda_recurrent_bwd_workspace_size(B, T, H, d, d), dtype=torch.uint8,
                     device=device)

    def run():
        kda.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], g, inp["beta"], cot["dout"], grads,
                              ws, init_state=inp["init_state"], d_final=cot["d_final"])

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    alg = B * T * H * BWD_BYTES_PER_TOKEN_HEAD + B * H * d * d * 4 * 3
    return ms, alg, B * T


# ------------------------------------------------------- oracle baseline
def oracle_prefill_parallel_sample(wl, inp, cu, budget_s=15.0):
    """Same as above but runs the oracle's own thread pool over a batch of
    units at once (what `cores` reports)."""
    import numpy as np

    import oracle
    H = wl["H"]
    nthreads = oracle.default_threads()
    q = inp["q"]
    if cu is None:
        B, T = q.shape[0], q.shape[1]
        n_b = 1
        sl = (slice(0, n_b),)
        per_unit = T
        units_per_b = H
        # one batch element at a time: H units of T tokens each
        t_used, done = 0.0, 0
        b = 0
        while t_used < budget_s and b < B:
            part = {k: inp[k][b:b + 1].detach().to("cpu", torch.float64).numpy()
                    for k in ("q", "k", "v", "z", "beta")}
            A_log = inp["A_log"].detach().cpu().double().numpy()
            t0 = time.perf_counter()
            g = oracle.gate(part["z"], A_log, -5.0)
            oracle.forward(part["q"], part["k"], part["v"], g, part["beta"], nthreads=nthreads)
            t_used += time.perf_counter() - t0
            done += per_unit * units_per_b
            b += 1
            if t_used * (b + 1) / b > budget_s * 1.5:
                break
        sample = f"{b} of {B} batch rows ({b * H} (sequence, head) units x {T} tokens)"
        return done / t_used / H, nthreads, sample, t_used
    cu_l = cu.cpu().tolist()
    Ns = len(cu_l) - 1
    t_used, done, n = 0.0, 0, 0
    A_log = inp["A_log"].detach().cpu().double().numpy()
    while t_used < budget_s and n < Ns:
        a, b = cu_l[n], cu_l[n + 1]
        part = {k: inp[k][:, a:b].detach().to("cpu", torch.float64).numpy()
                for k in ("q", "k", "v", "z", "beta")}
        S0 = inp["init_state"][n:n + 1].detach().cpu().double().numpy()
        t0 = time.perf_counter()
        g = oracle.gate(part["z"], A_log, -5.0)
        oracle.forward(part["q"], part["k"], part["v"], g, part["beta"], init_state=S0,
                       nthreads=nthreads)
        t_used += time.perf_counter() - t0
        done += (b - a) * H
        n += 1
    sample = f"{n} of {Ns} sequences (all {H} heads each)"
    return done / t_used / H, nthreads, sample, t_used


def oracle_decode_sample(wl, budget_s=10.0):
    import numpy as np

    import oracle
    N, H, dk, dv = wl["N"], wl["H"], wl["dk"], wl["dv"]
    nthreads = oracle.default_threads()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    S = W.make_decode_state(N, H, dk, dv, wl["seed"], dev).cpu().double().numpy()
    A_log = W.make_decode_gate_params(H, wl["seed"] + 1000, dev).cpu().double().numpy()
    t_used, steps = 0.0, 0
    while t_used < budget_s and steps < wl["steps"]:
        x = W.make_decode_step_inputs(N, H, dk, dv, torch.bfloat16, wl["seed"] + steps, dev)
        part = {k: x[k].detach().to("cpu", torch.float64).numpy()[:, None]
                for k in ("q", "k", "v", "z", "beta")}
        t0 = time.perf_counter()
        g = oracle.gate(part["z"], A_log, -5.0)
        _, S = oracle.forward(part["q"], part["k"], part["v"], g, part["beta"], init_state=S,
                              nthreads=nthreads)
        t_used += time.perf_counter() - t0
        steps += 1
    return steps / t_used, nthreads, f"{steps} of {wl['steps']} steps (all {N * H} heads)", t_used


def oracle_spec_sample(wl, budget_s=10.0):
    """The oracle verifying the K draft tokens of every head from its
    committed state (the recurrence over K tokens, outputs kept, the state
    left as it was), repeated until the budget is spent."""
    import oracle
    N, H, d, K = wl["N"], wl["H"], wl["dk"], wl["K"]
    nthreads = oracle.default_threads()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_prefill_inputs(N, K, H, d, d, torch.bfloat16, seed=wl["seed"], device=dev)
    S = W.make_decode_state(N, H, d, d, wl["seed"] + 1, dev).cpu().double().numpy()
    x = {k: inp[k].detach().to("cpu", torch.float64).numpy() for k in ("q", "k", "v", "z", "beta")}
    A_log = inp["A_log"].detach().cpu().double().numpy()
    t_used, launches = 0.0, 0
    while t_used < budget_s and launches < 1000:
        t0 = time.perf_counter()
        g = oracle.gate(x["z"], A_log, -5.0)
        oracle.forward(x["q"], x["k"], x["v"], g, x["beta"], init_state=S, nthreads=nthreads)
        t_used += time.perf_counter() - t0
        launches += 1
    return (launches * N * K / t_used, nthreads,
            f"{launches} verify launches (all {N * H} heads, K = {K})", t_used)


def bench_spec_line(args, wl, world, rank, peaks):
    """Speculative decoding on its own line: verify (the step) and replay."""
    dev = torch.device("cuda", torch.cuda.current_device())
    N, K = wl["N"], wl["K"]
    reps = max(args.steps, 20)
    clocks = None if args.no_clocks else ClockSampler(dev.index)
    barrier(world)
    res, bv, br, _ = run_spec_decode(dev, N=N, H=wl["H"], d=wl["dk"], K=K, reps=reps,
                                     seed=wl["seed"])
    clk = clocks.stop() if clocks else None
    vms = max_over_ranks(res["verify"], world)
    rms = max_over_ranks(res["replay"], world)
    vach, rach = bv / (vms * 1e-3) / 1e9, br / (rms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(N * K * world / (vms * 1e-3) / 1e6, 3),
        "unit": "M draft tokens/s (verify)", "n_gpus": world, "steps": reps, "warmup": 3,
        "ms_per_step": round(vms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "parallelism": f"dp{world} (independent batches)",
                   "l2": "state (537 MB) larger than L2",
                   "step": "kda_decode_verify (gate fused)"},
        "roofline": {"bound": "hbm", "achieved": round(vach, 1), "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": round(vach / peaks["hbm"], 4), "traffic": None,
                     "kernel": "decode_multi_kernel (verify)", "kernel_ms": round(vms, 4),
                     "algorithmic_bytes": bv},
        "replay": {"ms": round(rms, 4),
                   "roofline": {"bound": "hbm", "achieved": round(rach, 1), "peak": peaks["hbm"],
                                "unit": "GB/s", "frac": round(rach / peaks["hbm"], 4),
                                "algorithmic_bytes": br}},
        "gpu_launches": 2 * reps, "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, secs = oracle_spec_sample(wl)
        line["cpu_baseline"] = {"value": round(v / 1e6, 6), "unit": "M draft tokens/s (verify)",
                                "cores": cores, "kind": "oracle",
                                "sample": sample + f", {secs:.1f} s"}
    return line


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="libkda", choices=["libkda", "reference"])
    ap.add_argument("--workload", default="prefill", choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--kcp", action="store_true",
                    help="with --workload long: split the one sequence across the torchrun "
                         "ranks (context parallelism) instead of replicating it")
    ap.add_argument("--no-long", action="store_true",
                    help="leave the 1M-token prefill out of the default line")
    ap.add_argument("--no-varlen", action="store_true",
                    help="leave the varlen prefill out of the default line")
    ap.add_argument("--no-clocks", action="store_true",
                    help="skip nvidia-smi clock sampling (profiling runs)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B of a dense prefill workload (smaller profiling captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world, rank, local = dist_setup()
    wl = dict(WORKLOADS[args.workload])
    if args.batch is not None and args.workload == "decode":
        wl["N"] = args.batch
        wl["name"] = wl["name"].replace("N256 ", f"N{args.batch} ")
    elif args.batch is not None and not wl.get("varlen", True):
        wl["B"] = args.batch
        wl["name"] = wl["name"].replace(f"B{WORKLOADS[args.workload]['B']} ", f"B{args.batch} ")
    peaks = load_peaks()

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    if args.kcp and args.workload != "long":
        ap.error("--kcp applies to --workload long")
    if args.kcp:
        line = bench_kcp_line(args, wl, world, rank, peaks)
    elif args.workload == "decode":
        line = bench_decode_line(args, wl, world, rank, peaks)
    elif args.workload == "backward":
        line = bench_backward_line(args, wl, world, rank, peaks)
    elif args.workload == "spec_decode":
        line = bench_spec_line(args, wl, world, rank, peaks)
    else:
        line = bench_prefill_line(args, wl, world, rank, peaks)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def measure_prefill(wl, dev, steps, warmup, world, with_clocks):
    """Times `steps` gated chunkwise-forward steps of workload `wl` on resident
    inputs; returns the inputs, the step and the measured figures."""
    inp, cu, T, N = make_prefill(wl, dev)
    H, dk, dv = wl["H"], wl["dk"], wl["dv"]
    B = inp["q"].shape[0]
    step = PrefillStep(inp, cu, N)
    clocks = ClockSampler(dev.index) if with_clocks else None
    total_ms, chunk_ms = time_steps(step, steps, warmup, world)
    clk = clocks.extend_window(step) if clocks else None
    st, _ = kda.kda_get_device_status(step.ws)
    if st != kda.KDA_OK:
        raise RuntimeError(f"device status {kda.kda_status_string(st)}")
    ms_per_step = total_ms / steps
    tokens = B * T  # per rank
    tok_heads = tokens * H
    alg_bytes = tok_heads * prefill_bytes_per_token_head(wl) + N * H * dk * dv * 4 * (
        2 if inp["init_state"] is not None else 1)
    achieved = alg_bytes / (chunk_ms * 1e-3) / 1e9
    return dict(inp=inp, cu=cu, T=T, N=N, B=B, H=H, dk=dk, dv=dv, step=step, clk=clk,
                ms_per_step=ms_per_step, chunk_ms=chunk_ms, tokens=tokens, tok_heads=tok_heads,
                alg_bytes=alg_bytes, achieved=achieved,
                value=tokens * world / (ms_per_step * 1e-3) / 1e6)


def prefill_roofline(m, peaks, wl):
    dk, dv = m["dk"], m["dv"]
    f32 = m["tok_heads"] * prefill_flops_per_token_head(32, dk, dv)
    f64 = m["tok_heads"] * prefill_flops_per_token_head(64, dk, dv)
    secs = m["chunk_ms"] * 1e-3
    return {"bound": "hbm", "achieved": round(m["achieved"], 1), "peak": peaks["hbm"],
            "unit": "GB/s", "frac": round(m["achieved"] / peaks["hbm"], 4),
            "traffic": (chunk_traffic(m["B"], m["H"], m["T"])
                        if not wl.get("varlen") and wl.get("dtype", "bf16") == "bf16" else None),
            "kernel": ("chunk_tc_kernel (kda_chunk_fwd_gated)" if wl.get("dtype", "bf16") == "bf16"
                       else "bwd_keyside (key-side matrices of every chunk) + fwd_f32_scan_tc "
                            "(tcgen05 scan; kda_chunk_fwd_gated, fp32 inputs)"),
            "kernel_ms": round(m["chunk_ms"], 4), "algorithmic_bytes": m["alg_bytes"],
            "peak_source": peaks["src"],
            "tensor_frac": round(f32 / secs / (peaks["tc"] * 1e12), 4),
            "tensor_flops_count": "C(3dk+2dv)+C^2/3+6dk dv per token-head at C=32 "
                                  "(the chunk the kernel runs)",
            "tensor_frac_c64_count": round(f64 / secs / (peaks["tc"] * 1e12), 4)}


def check_input_sensitivity(step):
    """Outside the timed region: the step's output must follow its inputs.
    One value of v (token 0, head 0, channel 0) is changed, the step rerun, the
    output compared with the previous one (it must differ at token 0 of head 0),
    then the input is restored and the step rerun once more (it must give the
    original output back bit for bit)."""
    inp = step.inp
    before = step.out.clone()
    keep = inp["v"][0, 0, 0, 0].clone()
    inp["v"][0, 0, 0, 0] = keep + 1.0
    step()
    changed = not torch.equal(step.out[0, 0, 0], before[0, 0, 0])
    inp["v"][0, 0, 0, 0] = keep
    step()
    restored = torch.equal(step.out, before)
    torch.cuda.synchronize()
    if not (changed and restored):
        raise RuntimeError(f"output does not follow the input (changed={changed}, "
                           f"restored={restored})")
    return True


def bench_prefill_line(args, wl, world, rank, peaks):
    dev = torch.device("cuda", torch.cuda.current_device())
    m = measure_prefill(wl, dev, args.steps, args.warmup, world, not args.no_clocks)
    sensitivity = check_input_sensitivity(m["step"])
    inp, cu, T, N, B, H = m["inp"], m["cu"], m["T"], m["N"], m["B"], m["H"]
    dk, dv, step, tokens = m["dk"], m["dv"], m["step"], m["tokens"]
    line = {
        "metric": METRIC, "value": round(m["value"], 3), "unit": "Mtokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(m["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.get("dtype", "bf16"), "data": "synthetic",
        "config": {"workload": wl["name"], "global_batch": B * world, "seq_len": T,
                   "heads": H, "dk": dk, "dv": dv, "parallelism": f"dp{world} (independent batches)",
                   "l2": "inputs larger than L2 (no flush needed)",
                   "step": "kda_chunk_fwd_gated (gate fused)"},
        "roofline": prefill_roofline(m, peaks, wl),
        "gpu_launches": args.steps * kernels_per_step(wl, B, T),
        "clocks": m["clk"],
        "input_sensitivity": "checked: one value of v changed changes the output; restored gives "
                             "it back bit for bit" if sensitivity else None,
    }
    if not args.no_e2e and wl.get("dtype", "bf16") == "bf16":  # the host-buffer entry is bf16
        e2e_ms, h2d, d2h = e2e_prefill(wl, inp, cu, N, max(2, min(args.steps, 5)))
        line["e2e"] = {"value": round(tokens * world / (e2e_ms * 1e-3) / 1e6, 3),
                       "unit": "Mtokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, secs = oracle_prefill_parallel_sample(wl, inp, cu, budget_s=15.0)
        line["cpu_baseline"] = {"value": round(v / 1e6, 6), "unit": "Mtokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample + f", {secs:.1f} s"}
    del step, inp, m
    torch.cuda.empty_cache()
    if args.workload == "prefill":
        for name, skip, steps in (("long", args.no_long, 3), ("varlen", args.no_varlen, 10)):
            if skip:
                continue
            swl = WORKLOADS[name]
            sm = measure_prefill(swl, dev, steps, 3, world, not args.no_clocks)
            nk = kernels_per_step(swl, sm["B"], sm["T"])
            roof = prefill_roofline(sm, peaks, swl)
            if nk == 3:
                roof["kernel"] = ("chunk_tc_kernel (segment transitions) + segment_combine_kernel + "
                                  "chunk_tc_kernel (segment outputs): one kda_chunk_fwd_gated call")
            elif swl.get("varlen"):
                roof["kernel"] = "varlen_plan_kernel + chunk_tc_kernel (kda_chunk_fwd_gated)"
            line[name] = {
                "workload": swl["name"], "value": round(sm["value"], 3), "unit": "Mtokens/s",
                "steps": steps, "warmup": 3, "ms_per_step": round(sm["ms_per_step"], 4),
                "tokens_per_step": sm["tokens"], "heads": sm["H"],
                "roofline": roof, "gpu_launches": steps * nk,
                "clocks": sm["clk"]}
            del sm
            torch.cuda.empty_cache()
    if not args.no_decode and args.workload == "prefill":
        dwl = WORKLOADS["decode"]
        total, dec_ms, bpl = run_decode(dwl, dev)
        dach = bpl / (dec_ms * 1e-3) / 1e9
        line["decode"] = {"workload": dwl["name"], "value": round(dwl["steps"] / (total * 1e-3), 2),
                          "unit": "steps/s", "ms_per_step": round(total / dwl["steps"], 4),
                          "roofline": {"bound": "hbm", "achieved": round(dach, 1),
                                       "peak": peaks["hbm"], "unit": "GB/s",
                                       "frac": round(dach / peaks["hbm"], 4),
                                       "kernel": "decode_kernel (kda_decode_step_gated)",
                                       "kernel_ms": round(dec_ms, 4),
                                       "algorithmic_bytes": bpl}}
        res, bv, br, K = run_spec_decode(dev)
        line["spec_decode"] = {
            "workload": f"verify/replay N256 H32 d128, K={K} draft tokens",
            "verify_ms": round(res["verify"], 4),
            "verify_tokens_per_s": round(256 * K / (res["verify"] * 1e-3), 1),
            "verify_roofline": {"bound": "hbm", "achieved": round(bv / (res["verify"] * 1e-3) / 1e9, 1),
                                "peak": peaks["hbm"], "unit": "GB/s",
                                "frac": round(bv / (res["verify"] * 1e-3) / 1e9 / peaks["hbm"], 4)},
            "replay_ms": round(res["replay"], 4),
            "replay_roofline": {"bound": "hbm", "achieved": round(br / (res["replay"] * 1e-3) / 1e9, 1),
                                "peak": peaks["hbm"], "unit": "GB/s",
                                "frac": round(br / (res["replay"] * 1e-3) / 1e9 / peaks["hbm"], 4)}}
    if not args.no_backward and args.workload == "prefill":
        torch.cuda.empty_cache()
        ms, alg, ntok = run_backward(dev)
        ach = alg / (ms * 1e-3) / 1e9
        line["backward"] = {
            "workload": "backward B8 H32 T4096 d128, bf16 q/k/v/dout, fp32 gradients",
            "value": round(ntok / (ms * 1e-3) / 1e6, 4), "unit": "Mtokens/s",
            "ms_per_call": round(ms, 3),
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"],
                         "unit": "GB/s", "frac": round(ach / peaks["hbm"], 4),
                         "kernel": "bwd_keyside + bwd_fwd_scan_tc + bwd_state_grad_scan_tc + bwd_chunk_grads "
                                   "(one kda_recurrent_bwd call)", "algorithmic_bytes": alg}}
    return line


def bench_decode_line(args, wl, world, rank, peaks):
    dev = torch.device("cuda", torch.cuda.current_device())
    clocks = None if args.no_clocks else ClockSampler(dev.index)
    barrier(world)
    total, dec_ms, bpl = run_decode(wl, dev)
    clk = clocks.stop() if clocks else None
    total = max_over_ranks(total, world)
    dach = bpl / (dec_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(wl["steps"] / (total * 1e-3) * world, 2),
        "unit": "steps/s", "n_gpus": world, "steps": wl["steps"], "warmup": 3,
        "ms_per_step": round(total / wl["steps"], 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "parallelism": f"dp{world} (independent batches)",
                   "l2": "state (1 GiB) larger than L2"},
        "roofline": {"bound": "hbm", "achieved": round(dach, 1), "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": round(dach / peaks["hbm"], 4), "traffic": None,
                     "kernel": "decode_kernel (kda_decode_step_gated)",
                     "kernel_ms": round(dec_ms, 4)},
        "gpu_launches": wl["steps"], "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, secs = oracle_decode_sample(wl)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": "steps/s", "cores": cores,
                                "kind": "oracle", "sample": sample + f", {secs:.1f} s"}
    return line


def bench_backward_line(args, wl, world, rank, peaks):
    dev = torch.device("cuda", torch.cuda.current_device())
    B, T, H, d = wl["B"], wl["T"], wl["H"], wl["dk"]
    clocks = None if args.no_clocks else ClockSampler(dev.index)
    barrier(world)
    ms, alg, ntok = run_backward(dev, B=B, H=H, T=T, d=d, reps=args.steps)
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(ms, world)
    ach = alg / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(ntok * world / (ms * 1e-3) / 1e6, 4),
        "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps, "warmup": 3,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["name"], "global_batch": B * world, "seq_len": T,
                   "parallelism": f"dp{world} (independent batches)",
                   "l2": "inputs and workspace larger than L2",
                   "step": "kda_recurrent_bwd (bf16 q/k/v/dout, fp32 gradients)"},
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": round(ach / peaks["hbm"], 4), "traffic": None,
                     "kernel": "bwd_keyside + bwd_fwd_scan_tc + bwd_state_grad_scan_tc + bwd_chunk_grads "
                               "(one kda_recurrent_bwd call)", "kernel_ms": round(ms, 3),
                     "algorithmic_bytes": alg},
        "gpu_launches": 4 * args.steps, "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, secs = oracle_backward_sample(T=T, d=d)
        line["cpu_baseline"] = {"value": round(v, 6), "unit": "Mtokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample + f", {secs:.1f} s"}
    return line


def run_reference(args, wl, world):
    """The fp64 oracle as the reference arm, on this arm's config/metric."""
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if args.workload == "backward":
        vals = []
        for _ in range(args.steps):
            v, cores, sample, secs = oracle_backward_sample(T=wl["T"], d=wl["dk"], budget_s=5.0)
            vals.append(v)
        value = statistics.mean(vals)
        unit = "Mtokens/s"
        cfg = {"workload": wl["name"], "global_batch": wl["B"], "seq_len": wl["T"]}
    elif args.workload == "decode":
        t_per = []
        for _ in range(args.steps):
            v, cores, sample, secs = oracle_decode_sample(wl, budget_s=5.0)
            t_per.append(1.0 / v)
        value = 1.0 / statistics.mean(t_per)
        unit = "steps/s"
        cfg = {"workload": wl["name"]}
    elif args.workload == "spec_decode":
        vals = []
        for _ in range(args.steps):
            v, cores, sample, secs = oracle_spec_sample(wl, budget_s=5.0)
            vals.append(v / 1e6)
        value = statistics.mean(vals)
        unit = "M draft tokens/s (verify)"
        cfg = {"workload": wl["name"]}
    else:
        inp, cu, T, N = make_prefill(wl, dev)
        vals = []
        for _ in range(args.steps):
            v, cores, sample, secs = oracle_prefill_parallel_sample(wl, inp, cu, budget_s=8.0)
            vals.append(v / 1e6)
        value = statistics.mean(vals)
        unit = "Mtokens/s"
        cfg = {"workload": wl["name"], "global_batch": inp["q"].shape[0], "seq_len": T}
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
