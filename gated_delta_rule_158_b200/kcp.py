"""Cross-device context parallelism (KCP) for one long sequence.

"NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Infrastructure > KDA kernels
(KCP): cut a sequence into consecutive segments, one per device; the state a
segment leaves is S_end = S~ + M S_in, with S~ the state it leaves from a
zero state and M the product of its per-token transitions.  So each rank

  1. computes the pair (S~, M) of its own segment (every head),
  2. exchanges the pairs with one all-gather (fixed size: 2 x 64 KB per head),
  3. folds the pairs of the ranks before it into its incoming state, starting
     from the sequence's initial state,
  4. computes its outputs and the state its segment leaves from that state.

The last rank's end state is the sequence's final state.  The compute steps
run in libkda's kernels (LibkdaBackend); the exchange is torch.distributed
(NCCL between GPUs).  A backend object with the same three methods can be
passed in (with a `pair_dtype` attribute, the dtype of the exchanged pairs),
which is how the host logic is tested without a GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib as K


def segment_bounds(T: int, parts: int, chunk: int = 32):
    """Split T tokens into `parts` consecutive segments of whole chunks (the
    last takes the remainder); returns [(start, end)] in order."""
    if parts <= 0 or T < 0:
        raise ValueError("parts must be positive and T non-negative")
    chunks = (T + chunk - 1) // chunk
    base, extra = divmod(chunks, parts)
    bounds, start = [], 0
    for r in range(parts):
        n = base + (1 if r < extra else 0)
        end = min(T, start + n * chunk)
        bounds.append((start, end))
        start = end
    return bounds


class LibkdaBackend:
    """The three compute steps on the local GPU through libkda.  Segment
    inputs are dicts of device tensors: q, k, v bf16 [B, T, H, 128];
    z fp32 [B, T, H, 128]; A_log fp32 [H]; beta fp32 [B, T, H]."""

    pair_dtype = torch.float32

    def __init__(self, g_min: float = -5.0, scale: float = 1.0):
        self.g_min, self.scale = g_min, scale

    def transition(self, seg):
        q = seg["q"]
        B, T, H, dk = q.shape
        pairs = torch.empty((B, H, 2, dk, dk), dtype=torch.float32, device=q.device)
        ws = torch.zeros(256, dtype=torch.uint8, device=q.device)
        K.kda_chunk_segment_transition(seg["q"], seg["k"], seg["v"], seg["z"], seg["A_log"],
                                       seg["beta"], pairs, ws, g_min=self.g_min)
        return pairs

    def prefix(self, gathered, index, init_state):
        B, H, dk, dv = gathered.shape[1], gathered.shape[2], gathered.shape[-2], gathered.shape[-1]
        out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=gathered.device)
        K.kda_chunk_state_prefix(gathered, index, out, init_state=init_state)
        return out

    def forward(self, seg, state_in):
        q, v = seg["q"], seg["v"]
        B, T, H, dk = q.shape
        out = torch.empty((B, T, H, v.shape[-1]), dtype=q.dtype, device=q.device)
        fin = torch.empty((B, H, dk, v.shape[-1]), dtype=torch.float32, device=q.device)
        ws = torch.zeros(K.kda_chunk_fwd_workspace_size(B, T, H, dk, v.shape[-1]),
                         dtype=torch.uint8, device=q.device)
        K.kda_chunk_fwd_gated(seg["q"], seg["k"], seg["v"], seg["z"], seg["A_log"], seg["beta"],
                              out, ws, g_min=self.g_min, init_state=state_in, final_state=fin,
                              scale=self.scale)
        return out, fin


def kcp_prefill(seg, init_state=None, group=None, backend=None):
    """Run this rank's segment of a sequence split across the ranks of
    `group` (rank r holds the r-th segment in token order).  Returns (o of
    the local segment, state after it); on the last rank that state is the
    sequence's final state.  init_state: the sequence's initial state
    [B, H, dk, dv] fp32 or None (zeros), the same on every rank."""
    backend = backend or LibkdaBackend()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    q, v = seg["q"], seg["v"]
    B, T, H, dk = q.shape
    if rank < world - 1 and T > 0:
        pairs = backend.transition(seg)
    else:  # the last segment's pair is never read; an empty segment is (0, I)
        pairs = torch.zeros((B, H, 2, dk, dk), dtype=backend.pair_dtype, device=q.device)
        if T == 0:
            pairs[:, :, 1] = torch.eye(dk, dtype=pairs.dtype, device=pairs.device)
    parts = [torch.empty_like(pairs) for _ in range(world)]
    dist.all_gather(parts, pairs.contiguous(), group=group)
    state_in = backend.prefix(torch.stack(parts), rank, init_state)
    if T == 0:
        return torch.empty((B, 0, H, v.shape[-1]), dtype=v.dtype, device=v.device), state_in
    return backend.forward(seg, state_in)
