"""Window-aligned sharding of a batch across GPUs, one process per GPU.

The forward has no exchange across windows: a window is whole 100-frame chunks
of one request and attention never crosses a window (aut_encoder page, module
docstring; openarchlab "1A . AuT Audio Encoder", section 4, window isolation),
and every other step is per token.  So a batch splits exactly along window
boundaries: whole requests, or a long request cut at multiples of
n_window_infer frames.  Pieces are assigned to ranks longest-first onto the
least-loaded rank (LPT), by token count.  Token counts come from the library's
planner (aut_plan); nothing here computes any step of the encoder.

Each rank encodes its pieces as one packed batch through aut_encode.  The rows
stay on the rank that computed them unless the caller asks for them to be
gathered (one all-gather over the process group: NCCL between GPUs, gloo on
CPU).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import _lib as A


@dataclasses.dataclass(frozen=True, order=True)
class Piece:
    request: int   # index in the batch
    frame0: int    # first frame of the piece inside its request (a window boundary)
    frames: int    # frames in the piece


def pieces(lens, n_window_infer: int, max_frames: int | None = None) -> list[Piece]:
    """Cut requests longer than `max_frames` (rounded down to whole windows)
    at window boundaries; shorter requests stay whole.  Empty requests give no
    piece."""
    out = []
    step = None
    if max_frames is not None:
        step = max(n_window_infer, (max_frames // n_window_infer) * n_window_infer)
    for r, n in enumerate(lens):
        if n <= 0:
            continue
        if step is None or n <= step:
            out.append(Piece(r, 0, n))
        else:
            for f0 in range(0, n, step):
                out.append(Piece(r, f0, min(step, n - f0)))
    return out


def frame_tokens(cfg: A.aut_config, frame_counts) -> list[int]:
    """Token count of each frame span (a span starting on a chunk boundary
    yields what a request of that length yields), from aut_plan."""
    if not len(frame_counts):
        return []
    return A.aut_plan(cfg, [int(f) for f in frame_counts])[0]


def assign(ps: list[Piece], world: int, cfg: A.aut_config) -> list[list[Piece]]:
    """Longest-processing-time-first assignment of pieces to `world` ranks (by
    token count); each rank's pieces in batch order."""
    tok = dict(zip(ps, frame_tokens(cfg, [p.frames for p in ps])))
    loads = [0] * world
    shards = [[] for _ in range(world)]
    for p in sorted(ps, key=lambda p: (-tok[p], p.request, p.frame0)):
        k = min(range(world), key=lambda i: (loads[i], i))
        shards[k].append(p)
        loads[k] += tok[p]
    for s in shards:
        s.sort(key=lambda p: (p.request, p.frame0))
    return shards


def reassemble(cfg: A.aut_config, shards, outputs):
    """Concatenate per-rank outputs (rows of each rank's pieces, in its shard
    order) back into the unsharded packed order: requests in input order,
    pieces in frame order.  Works on numpy arrays and torch tensors."""
    rows = {}
    for shard, out in zip(shards, outputs):
        at = 0
        for p, n in zip(shard, frame_tokens(cfg, [p.frames for p in shard])):
            rows[(p.request, p.frame0)] = out[at:at + n]
            at += n
    keys = sorted(rows)
    if not keys:
        return None
    parts = [rows[k] for k in keys]
    if isinstance(parts[0], np.ndarray):
        return np.concatenate(parts, axis=0)
    import torch
    return torch.cat(parts, dim=0)


def shard_features(features, shard: list[Piece]):
    """The sub-batch of a rank's pieces: [len(shard), mel_bins, max frames]
    (piece i's frames first, zeros after), from the batch's features
    [B, mel_bins, T_max] (numpy array or torch tensor, on any device)."""
    n = max((p.frames for p in shard), default=1)
    if isinstance(features, np.ndarray):
        sub = np.zeros((len(shard), features.shape[1], n), features.dtype)
    else:
        import torch
        sub = torch.zeros((len(shard), features.shape[1], n), dtype=features.dtype,
                          device=features.device)
    for i, p in enumerate(shard):
        sub[i, :, :p.frames] = features[p.request, :, p.frame0:p.frame0 + p.frames]
    return sub


def encode_sharded(enc, features, lens, rank: int, world: int, max_frames: int | None = None,
                   gather: bool = False, group=None):
    """One rank's part of a sharded forward.  `enc` is this rank's Encoder
    (weights replicated on every GPU), `features` the whole batch on this
    rank's GPU.  Returns (rows of this rank's pieces in shard order, shards);
    with gather=True also all-gathers every rank's rows (padded to the longest
    shard) and returns the whole batch's output in packed order instead."""
    ps = pieces(lens, enc.cfg.n_window_infer, max_frames)
    shards = assign(ps, world, enc.c)
    mine = shards[rank]
    if mine:
        sub = shard_features(features, mine)
        out = enc.encode(sub, [p.frames for p in mine])
    else:
        import torch
        out = torch.zeros((0, enc.cfg.output_dim), dtype=torch.float32, device=enc.device)
    if not gather:
        return out, shards
    import torch
    import torch.distributed as dist
    counts = [sum(frame_tokens(enc.c, [p.frames for p in s])) for s in shards]
    cap = max(counts + [1])
    padded = torch.zeros((cap, out.shape[1]), dtype=out.dtype, device=out.device)
    padded[:out.shape[0]] = out
    bufs = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(bufs, padded, group=group)
    return reassemble(enc.c, shards, [b[:c] for b, c in zip(bufs, counts)]), shards
