"""Encoder parity on the GPU through the C ABI against the CPU oracle on the
same seeded bf16 inputs: stage-wise (stem output before the positions, x0,
after layer 0, after the last layer) and the final output, on every workload;
the full-size long-form and throughput batches on sampled windows (a window is
whole chunks of one request, so the oracle computes it from its own frames);
bit-exact invariants (window isolation, packing order); edge cases."""
import numpy as np
import pytest

import aut_synth as S
import oracle as O
from gpu_util import assert_rows_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from audio_encoder_aut_b200 import _lib as A  # noqa: E402
from audio_encoder_aut_b200.encoder import Encoder  # noqa: E402

_ENC = {}


def encoder(name, **wkw):
    key = (name, tuple(sorted(wkw.items())))
    if key not in _ENC:
        cfg = S.WORKLOADS.get(name, S.OMNI)
        w = S.weights(cfg, **wkw)
        _ENC[key] = (cfg, w, Encoder(cfg, w, 0))
    return _ENC[key]


def run(enc, feats, lens):
    out = enc.encode(enc.features_to_device(feats), lens)
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK
    return out.float().cpu().numpy()


def test_plan_device_agrees_with_oracle_layout():
    cfg, w, enc = encoder("tiny")
    tpr, cu, total, nw, nch = enc.plan([237, 0, 1000])
    lay = O.plan(cfg, [237, 0, 1000])
    assert cu == lay.cu_seqlens and tpr == lay.tokens_per_request


@pytest.mark.parametrize("variant", [dict(), dict(conv_scale=25.0, conv_out_bias=True)])
def test_tiny_stagewise_and_final(variant):
    cfg, w, enc = encoder("tiny", **variant)
    lens = S.request_lengths("tiny")
    feats = S.features(lens)
    fd = enc.features_to_device(feats)
    # stem output (conv_out) before the positions
    ref_hidden = {}
    ref_out, lay = O.forward(cfg, w, feats, lens, hidden=ref_hidden)
    h = enc.frontend(fd, lens, with_positions=False)
    torch.cuda.synchronize()
    assert_rows_close(h.cpu().numpy(), ref_hidden["stem"], "stem")
    x0 = enc.frontend(fd, lens)
    torch.cuda.synchronize()
    assert_rows_close(x0.cpu().numpy(), ref_hidden["x0"], "x0")
    x = x0.clone()
    enc.encode_packed(x, lay.cu_seqlens, 1, with_projector=False)
    torch.cuda.synchronize()
    assert_rows_close(x.cpu().numpy(), ref_hidden[0], "after layer 0")
    out = run(enc, feats, lens)
    assert_rows_close(out, ref_out, "final")


def _stage_and_final(name, dtype=np.float32, **wkw):
    cfg, w, enc = encoder(name, **wkw)
    lens = S.request_lengths(name)
    feats = S.features(lens)
    ref_hidden = {}
    ref_out, lay = O.forward(cfg, w, feats, lens, dtype=dtype, hidden=ref_hidden)
    fd = enc.features_to_device(feats)
    h = enc.frontend(fd, lens, with_positions=False)
    torch.cuda.synchronize()
    assert_rows_close(h.cpu().numpy(), ref_hidden["stem"], "stem")
    x0 = enc.frontend(fd, lens)
    torch.cuda.synchronize()
    assert_rows_close(x0.cpu().numpy(), ref_hidden["x0"], "x0")
    x = x0.clone()
    enc.encode_packed(x, lay.cu_seqlens, 1, with_projector=False)
    torch.cuda.synchronize()
    assert_rows_close(x.cpu().numpy(), ref_hidden[0], "after layer 0")
    x = x0.clone()
    out = enc.encode_packed(x, lay.cu_seqlens, cfg.encoder_layers, with_projector=True)
    torch.cuda.synchronize()
    assert_rows_close(x.cpu().numpy(), ref_hidden[cfg.encoder_layers - 1], "after last layer")
    assert_rows_close(out.float().cpu().numpy(), ref_out, "projector output (packed entry)")
    assert_rows_close(run(enc, feats, lens), ref_out, "final")


def test_asr06b_30s_stagewise_and_final():
    _stage_and_final("asr06b_30s")


def test_omni_16req_stagewise_and_final():
    _stage_and_final("omni_16req")


def test_asr06b_nonlinear_stem():
    cfg, w, enc = encoder("asr06b_30s", conv_scale=25.0)
    lens = [1234, 77]
    feats = S.features(lens)
    h = enc.frontend(enc.features_to_device(feats), lens, with_positions=False)
    torch.cuda.synchronize()
    assert_rows_close(h.cpu().numpy(), O.frontend(cfg, w, feats, lens, np.float32,
                                                  with_positions=False), "stem x25")


@pytest.mark.parametrize("C", [64, 192, 240, 256, 384, 512])
def test_stem_channel_counts(C):
    """The stem at other supported conv widths: C = 64 .. 512 on the tensor-core
    conv1 (accumulator halves of N = min(C, 256) and C - 256: one half up to
    C = 256, two from 384; epilogue groups without a block at C = 64), C = 240
    on the CUDA-core conv1; partial last chunks; GELUs in their non-linear range
    (conv weights x 25)."""
    import dataclasses
    cfg = dataclasses.replace(S.TINY, downsample_hidden_size=C)
    w = S.weights(cfg, conv_scale=25.0)
    enc = Encoder(cfg, w, 0)
    lens = [237, 1000, 450]
    feats = S.features(lens)
    h = enc.frontend(enc.features_to_device(feats), lens, with_positions=False)
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK
    assert_rows_close(h.cpu().numpy(), O.frontend(cfg, w, feats, lens, np.float32,
                                                  with_positions=False), f"stem C={C}")


def _sampled_windows(cfg, w, enc, lens, picks):
    """GPU on the whole batch; oracle on each picked (request, window) alone."""
    feats = S.features(lens)
    out = run(enc, feats, lens)
    lay = O.plan(cfg, lens)
    wt = O.window_tokens(cfg)
    row0 = np.cumsum([0] + lay.tokens_per_request)
    for r, k in picks:
        f0 = k * cfg.n_window_infer
        n = min(cfg.n_window_infer, lens[r] - f0)
        ref, _ = O.forward(cfg, w, feats[r:r + 1, :, f0:f0 + n], [n], dtype=np.float32)
        a = row0[r] + k * wt
        assert_rows_close(out[a:a + ref.shape[0]], ref, f"request {r} window {k}")
    return out


@pytest.mark.parametrize("name", ["omni_20min", "omni_20min_ragged"])
def test_long_form_sampled_windows(name):
    cfg, w, enc = encoder("omni_20min")
    lens = S.request_lengths(name)
    nwin = -(-O.tokens_for_frames(cfg, lens[0]) // O.window_tokens(cfg))
    out = _sampled_windows(cfg, w, enc, lens, [(0, 0), (0, 71), (0, nwin - 1)])
    assert out.shape[0] == O.plan(cfg, lens).total_tokens


def test_throughput_batch_sampled_windows():
    cfg, w, enc = encoder("omni_256req")
    lens = S.request_lengths("omni_256req")
    rng = np.random.default_rng(9)
    picks = [(0, 0), (255, 0)]
    for r in rng.choice(256, 3, replace=False):
        nwin = -(-O.tokens_for_frames(cfg, lens[r]) // O.window_tokens(cfg))
        picks.append((int(r), int(nwin - 1)))
    _sampled_windows(cfg, w, enc, lens, picks)


def test_window_isolation_bit_exact():
    """openarchlab 1A, section 4, on the GPU: changing the second window's
    frames leaves the first window's output rows bit-identical."""
    cfg, w, enc = encoder("omni_16req")
    lens = [1700]
    feats = S.features(lens)
    a = run(enc, feats, lens)
    f2 = feats.copy()
    f2[0, :, 800:1600] = S.round_bf16(f2[0, :, 800:1600] * 0.5 + 0.25)
    b = run(enc, f2, lens)
    assert np.array_equal(a[:104], b[:104])
    assert not np.array_equal(a[104:208], b[104:208])


def test_packing_order_bit_exact():
    cfg, w, enc = encoder("omni_16req")
    lens = [437, 1250, 90, 2001]
    feats = S.features(lens)
    a = run(enc, feats, lens)
    perm = [3, 1, 0, 2]
    b = run(enc, feats[perm], [lens[i] for i in perm])
    ta = [O.tokens_for_frames(cfg, n) for n in lens]
    sa = np.cumsum([0] + ta)
    sb = np.cumsum([0] + [ta[i] for i in perm])
    for j, i in enumerate(perm):
        assert np.array_equal(a[sa[i]:sa[i + 1]], b[sb[j]:sb[j + 1]])


def test_edge_cases_empty_and_tiny_requests():
    cfg, w, enc = encoder("tiny")
    lens = [0, 1, 8, 9, 100, 0, 101]
    feats = S.features(lens, t_max=128 + 1, fill_beyond=7.0)  # garbage past each length
    ref, lay = O.forward(cfg, w, S.features(lens, t_max=129), lens)
    out = run(enc, feats, lens)
    assert out.shape == ref.shape
    assert_rows_close(out, ref, "ragged tiny requests")
    out = enc.encode(enc.features_to_device(feats), [0, 0])
    torch.cuda.synchronize()
    assert out.shape[0] == 0


def test_stem_group_boundaries():
    """More chunks than one conv group: groups of conv_chunksize chunks give the
    same rows as one group."""
    import dataclasses
    cfg = dataclasses.replace(S.TINY, conv_chunksize=3)
    w = S.weights(cfg, conv_scale=25.0)
    enc = Encoder(cfg, w, 0)
    lens = [737, 250, 99]
    feats = S.features(lens)
    out = run(enc, feats, lens)
    ref, _ = O.forward(cfg, w, feats, lens)
    assert_rows_close(out, ref, "grouped stem")


def test_cuda_graph_replay_matches_eager_bit_exact():
    """The forward captured once into a CUDA graph (plan built on the host,
    outside the graph) and replayed on new features gives the eager result."""
    cfg, w, enc = encoder("omni_16req")
    lens = [777, 1203, 64]
    fa, fb = S.features(lens, seed=11), S.features(lens, seed=12)
    feats_dev = enc.features_to_device(fa)
    graph, out = enc.capture(feats_dev, lens)
    feats_dev.copy_(enc.features_to_device(fb))
    graph.replay()
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK
    got = out.cpu().numpy().copy()
    eager = run(enc, fb, lens)
    assert np.array_equal(got, eager)
    ref, _ = O.forward(cfg, w, fb, lens, dtype=np.float32)
    assert_rows_close(got, ref, "graph replay")


def test_pipelined_host_stream_matches_eager_bit_exact():
    """Encoder.encode_stream: five batches from pinned host memory, copies on a
    second stream overlapping the neighbours' compute, two device buffer sets;
    every host output equals the eager forward of its own batch."""
    cfg, w, enc = encoder("omni_16req")
    lens = [777, 1203, 64]
    batches = [S.features(lens, seed=20 + i) for i in range(5)]
    host_in = [torch.from_numpy(b).to(torch.bfloat16).pin_memory() for b in batches]
    total = enc.plan(lens)[2]
    host_out = [torch.full((total, cfg.output_dim), float("nan")).pin_memory() for _ in batches]
    graphs, (e0, e1) = enc.encode_stream(host_in, lens, host_out)
    torch.cuda.synchronize()
    assert enc.check() == A.AUT_OK
    assert e0.elapsed_time(e1) > 0
    for b, h in zip(batches, host_out):
        assert np.array_equal(h.numpy(), run(enc, b, lens))
    # the returned graphs serve a second sequence, written into other host buffers
    host_out2 = [torch.empty_like(h).pin_memory() for h in host_out[:2]]
    enc.encode_stream(host_in[3:], lens, host_out2, graphs=graphs)
    torch.cuda.synchronize()
    for b, h in zip(batches[3:], host_out2):
        assert np.array_equal(h.numpy(), run(enc, b, lens))


@pytest.mark.parametrize("name,lens,max_frames,world", [
    ("omni_16req", [1734, 90, 610, 2999, 333, 1201], 1600, 3),
    ("tiny", [1234, 90, 610, 0, 333], 400, 4),
])
def test_sharded_pieces_reassemble_bit_exact(name, lens, max_frames, world):
    """The multi-GPU split on one device: a `world`-rank plan of window-aligned
    pieces (long requests cut at window boundaries), every rank's pieces
    encoded as its own packed batch through aut_encode, reassembled into
    packed order, equals the unsharded forward bit for bit (window isolation,
    aut_encoder page module docstring; openarchlab 1A, section 4)."""
    from audio_encoder_aut_b200 import shard as SH
    cfg, w, enc = encoder(name)
    feats = S.features(lens)
    whole = run(enc, feats, lens)
    shards = SH.assign(SH.pieces(lens, cfg.n_window_infer, max_frames), world, enc.c)
    assert sum(len(s) > 0 for s in shards) >= 2
    fd = enc.features_to_device(feats)
    outs = []
    for s in shards:
        if s:
            o = enc.encode(SH.shard_features(fd, s), [p.frames for p in s])
            torch.cuda.synchronize()
            assert enc.check() == A.AUT_OK
            outs.append(o.cpu().numpy())
        else:
            outs.append(np.zeros((0, cfg.output_dim), np.float32))
    got = SH.reassemble(enc.c, shards, outs)
    assert got.shape == whole.shape
    assert np.array_equal(got, whole)
