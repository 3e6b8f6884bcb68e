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
from audio_encoder_aut_b200 import _lib as A
from audio_encoder_aut_b200 import shard as SH

CFG = A.make_config(S.TINY)


def _tok(frames):
    return SH.frame_tokens(CFG, [frames])[0]


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
    shards = SH.assign(ps, 3, CFG)
    assert sorted(p for s in shards for p in s) == sorted(ps)
    loads = [sum(_tok(p.frames) for p in s) for s in shards]
    assert max(loads) - min(loads) <= max(_tok(p.frames) for p in ps)
    # token counts of the pieces add up to the requests' token counts
    for r, n in enumerate(lens):
        assert sum(_tok(p.frames) for p in ps if p.request == r) == \
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
        shards = SH.assign(SH.pieces(lens, cfg.n_window_infer, max_frames=400), world,
                           A.make_config(cfg))
        mine = shards[rank]
        if mine:
            sub_lens = [p.frames for p in mine]
            sub = SH.shard_features(feats, mine)
            out, _ = O.forward(cfg, w, sub, sub_lens)
        else:
            out = np.zeros((0, cfg.output_dim))
        gathered = [None] * world
        dist.all_gather_object(gathered, out)
        if rank == 0:
            got = SH.reassemble(A.make_config(cfg), shards, gathered)
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


def test_shard_planner_properties_random():
    """Random batches, window sizes, cut lengths and rank counts: the pieces
    tile every request on window boundaries, their token counts add up to the
    oracle's, every piece lands on exactly one rank, the LPT loads stay within
    one piece of each other, and reassembling per-rank rows that carry their
    own coordinates gives the unsharded packed order."""
    rng = np.random.default_rng(123)
    for trial in range(200):
        nwi = 100 * int(rng.integers(1, 9))
        lens = [int(x) for x in rng.integers(0, 6000, size=int(rng.integers(1, 12)))]
        max_frames = int(rng.integers(nwi, 5000)) if trial % 3 else None
        world = int(rng.integers(1, 6))
        ps = SH.pieces(lens, nwi, max_frames=max_frames)
        for r, n in enumerate(lens):
            mine = sorted((p.frame0, p.frames) for p in ps if p.request == r)
            covered = 0
            for f0, nf in mine:
                assert f0 == covered and f0 % nwi == 0 and nf > 0
                covered += nf
            assert covered == n
            assert sum(_tok(p.frames) for p in ps if p.request == r) == \
                O.tokens_for_frames(S.TINY, n)
        shards = SH.assign(ps, world, CFG)
        assert len(shards) == world
        assert sorted(p for s in shards for p in s) == sorted(ps)
        if ps:
            loads = [sum(_tok(p.frames) for p in s) for s in shards]
            assert max(loads) - min(loads) <= max(_tok(p.frames) for p in ps)
        # each rank's "output" rows hold (request, token index within the request)
        outputs = []
        for s in shards:
            rows = []
            for p in s:
                t0 = _tok(p.frame0)
                rows += [(p.request, t0 + i) for i in range(_tok(p.frames))]
            outputs.append(np.array(rows, dtype=np.int64).reshape(-1, 2))
        got = SH.reassemble(CFG, shards, outputs)
        want = [(r, i) for r, n in enumerate(lens) for i in range(O.tokens_for_frames(S.TINY, n))]
        if want:
            assert got.tolist() == [list(w) for w in want]
        else:
            assert got is None
