"""The N > 1 path on CPU: two gloo ranks each encode a window-aligned shard of
one batch (through the oracle, since no GPU is here); the gathered rows equal
the unsharded forward.  Also checks the shard planner's invariants."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import aut_synth as S
import oracle as O
from audio_encoder_aut_b200 import shard as SH


def test_pieces_and_assignment_cover_the_batch():
    lens = [0, 5, 99, 100, 801, 2500, 1600, 4321]
    ps = SH.pieces(lens, 800, max_frames=1700)
    # every frame of every request appears exactly once, cut on window boundaries
    for r, n in enumerate(lens):
        mine = sorted((p.frame0, p.frames) for p in ps if p.request == r)
        covered = 0
        for f0, nf in mine:
            assert f0 == covered and f0 % 800 == 0
            covered += nf
        assert covered == n
    shards = SH.assign(ps, 3)
    assert sorted(p for s in shards for p in s) == sorted(ps)
    loads = [sum(SH._tokens(p.frames) for p in s) for s in shards]
    assert max(loads) - min(loads) <= max(SH._tokens(p.frames) for p in ps)
    # token counts of the pieces add up to the requests' token counts
    for r, n in enumerate(lens):
        assert sum(SH._tokens(p.frames) for p in ps if p.request == r) == \
            O.tokens_for_frames(S.TINY, n)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, lens, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = S.TINY
        w = S.weights(cfg, conv_scale=10.0)
        feats = S.features(lens)
        shards = SH.assign(SH.pieces(lens, cfg.n_window_infer, max_frames=400), world)
        mine = shards[rank]
        if mine:
            sub_lens = [p.frames for p in mine]
            sub = np.zeros((len(mine), feats.shape[1], max(sub_lens)), np.float32)
            for i, p in enumerate(mine):
                sub[i, :, :p.frames] = feats[p.request, :, p.frame0:p.frame0 + p.frames]
            out, _ = O.forward(cfg, w, sub, sub_lens)
        else:
            out = np.zeros((0, cfg.output_dim))
        gathered = [None] * world
        dist.all_gather_object(gathered, out)
        if rank == 0:
            got = SH.reassemble(lens, shards, gathered)
            ref, _ = O.forward(cfg, w, feats, lens)
            np.save(result_path, np.stack([np.abs(got - ref).max(), float(got.shape[0] == ref.shape[0])]))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_forward_equals_unsharded(tmp_path):
    lens = [1234, 90, 610, 0, 333]
    path = str(tmp_path / "res.npy")
    mp.spawn(_rank_main, args=(2, _free_port(), lens, path), nprocs=2, join=True)
    err, same_rows = np.load(path)
    assert same_rows == 1.0
    # fp64; BLAS blocks shorter matrices differently, so rows agree to rounding
    assert err < 1e-12
