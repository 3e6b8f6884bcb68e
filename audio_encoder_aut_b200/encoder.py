"""PyTorch plumbing around the C ABI: device buffers for the weights, the
workspace and the outputs, and the current CUDA stream.  Nothing here computes
any step of the encoder; every step runs in libaut.so."""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib as A


def _dev_bf16(arr, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device=device, dtype=torch.bfloat16).contiguous()


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def current_stream_handle(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


class Encoder:
    """Holds one encoder's weights on a GPU and runs it through libaut.so.

    `cfg` has AuTEncoderConfig-style attributes; `weights` is a dict of arrays
    in PyTorch layouts (see include/aut.h), e.g. from aut_synth.weights()."""

    def __init__(self, cfg, weights: dict, device: int | str = 0):
        if not torch.cuda.is_available():
            raise RuntimeError("the AuT encoder runs on a CUDA GPU only")
        self.device = torch.device("cuda", torch.device(device).index
                                   if isinstance(device, str) else device)
        self.cfg = cfg
        self.c = A.make_config(cfg)
        A.lib()
        dev = self.device
        self._keep = []

        def up(a):
            if a is None:
                return None
            t = _dev_bf16(a, dev)
            self._keep.append(t)
            return t

        w = A.aut_weights()
        for k in ["conv1_w", "conv1_b", "conv2_w", "conv2_b", "conv3_w", "conv3_b",
                  "conv_out_w", "conv_out_b", "ln_post_w", "ln_post_b", "proj1_w", "proj1_b",
                  "proj2_w", "proj2_b"]:
            setattr(w, k, _ptr(up(weights.get(k))))
        n = len(weights["layers"])
        self._layers = (A.aut_layer_weights * max(1, n))()
        for i, lw in enumerate(weights["layers"]):
            for k in A.LAYER_FIELDS:
                setattr(self._layers[i], k, _ptr(up(lw[k])))
        w.layers = ctypes.cast(self._layers, ctypes.POINTER(A.aut_layer_weights))
        self._src = w
        nbytes = A.aut_prepared_bytes(self.c)
        if nbytes == 0:
            raise A.AutError(A.AUT_ERR_UNSUPPORTED, "aut_prepared_bytes")
        self._prepared_buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        with torch.cuda.device(dev):
            self.prepared = A.aut_prepare_weights(self.c, self._src, self._prepared_buf.data_ptr(),
                                                  nbytes, current_stream_handle(dev))
        self._ws = None
        self._lm_ws = None

    # ------------------------------------------------------------------
    def plan(self, feature_lens):
        return A.aut_plan(self.c, feature_lens)

    def workspace(self, total_tokens: int, num_windows: int, num_chunks: int) -> torch.Tensor:
        need = A.aut_workspace_bytes(self.c, total_tokens, num_windows, num_chunks)
        if need == 0:
            raise A.AutError(A.AUT_ERR_UNSUPPORTED, "aut_workspace_bytes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def logmel(self, waveform: torch.Tensor, sample_lens, t_max: int | None = None):
        """16 kHz mono waveform, device fp32 [B, S_max] -> (features bf16
        [B, 128, T_max] on the device, feature_lens), through aut_logmel."""
        waveform = waveform.contiguous()
        frames = [int(n) // 160 for n in sample_lens]
        t = max(frames + [1]) if t_max is None else t_max
        feats = torch.empty((len(sample_lens), 128, t), dtype=torch.bfloat16, device=self.device)
        need = A.aut_logmel_workspace_bytes(len(sample_lens), t)
        if self._lm_ws is None or self._lm_ws.numel() < need:
            self._lm_ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        st, lens = A.aut_logmel(waveform.data_ptr(), waveform.shape[-1], sample_lens,
                                feats.data_ptr(), t, self._lm_ws.data_ptr(), self._lm_ws.numel(),
                                current_stream_handle(self.device))
        if st != A.AUT_OK:
            raise A.AutError(st, "aut_logmel")
        return feats, lens

    def features_to_device(self, feats: np.ndarray) -> torch.Tensor:
        return _dev_bf16(feats, self.device)

    def encode(self, features: torch.Tensor, feature_lens, out: torch.Tensor | None = None,
               trace: A.aut_trace | None = None):
        """features: bf16 [B, 128, T_max] on the device -> fp32 [total_tokens, output_dim]."""
        _, _, total, nw, nch = self.plan(feature_lens)
        ws = self.workspace(total, nw, nch)
        if out is None:
            out = torch.empty((total, self.cfg.output_dim), dtype=torch.float32, device=self.device)
        st = A.aut_encode_traced(self.c, self.prepared, features.data_ptr(), features.shape[-1],
                                 feature_lens, out.data_ptr(), ws.data_ptr(), ws.numel(),
                                 current_stream_handle(self.device), trace)
        if st != A.AUT_OK:
            raise A.AutError(st, "aut_encode")
        return out

    def frontend(self, features: torch.Tensor, feature_lens, with_positions: bool = True):
        """-> fp32 [total_tokens, d_model] packed chunk embeddings."""
        _, _, total, nw, nch = self.plan(feature_lens)
        ws = self.workspace(total, nw, nch)
        x0 = torch.empty((total, self.cfg.d_model), dtype=torch.float32, device=self.device)
        st = A.aut_frontend(self.c, self.prepared, features.data_ptr(), features.shape[-1],
                            feature_lens, x0.data_ptr(), with_positions, ws.data_ptr(), ws.numel(),
                            current_stream_handle(self.device))
        if st != A.AUT_OK:
            raise A.AutError(st, "aut_frontend")
        return x0

    def encode_packed(self, hidden: torch.Tensor, cu_seqlens, n_layers: int,
                      with_projector: bool = True):
        """Runs layers [0, n_layers) on `hidden` (fp32 [T, d], updated in place) and
        optionally the projector; returns the projector output or None."""
        T = hidden.shape[0]
        ws = self.workspace(T, len(cu_seqlens) - 1, 0)
        out = None
        if with_projector:
            out = torch.empty((T, self.cfg.output_dim), dtype=torch.float32, device=self.device)
        st = A.aut_encode_packed(self.c, self.prepared, hidden.data_ptr(), T, cu_seqlens, n_layers,
                                 _ptr(out), ws.data_ptr(), ws.numel(),
                                 current_stream_handle(self.device))
        if st != A.AUT_OK:
            raise A.AutError(st, "aut_encode_packed")
        return out

    def capture(self, features: torch.Tensor, feature_lens, out: torch.Tensor | None = None,
                warmup: int = 2, trace: A.aut_trace | None = None):
        """Records one aut_encode of this exact batch shape into a CUDA graph and
        returns (graph, out).  The plan is built on the host once, outside the
        graph (aut_encoder page, module docstring: the runner's plan is built
        outside the graph so the block loop replays as a CUDA graph); replaying
        the graph re-runs the whole forward on whatever `features` then holds.
        The graph keeps this encoder's workspace, so it must not be replayed
        concurrently with another call on the same encoder.  With `trace`, the
        graph also records trace.events[i] after launch i (an event node between
        launches, which orders them fully: no launch overlaps its predecessor)."""
        if out is None:
            _, _, total, _, _ = self.plan(feature_lens)
            out = torch.empty((total, self.cfg.output_dim), dtype=torch.float32, device=self.device)
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            for _ in range(warmup):  # one-time kernel attributes, workspace sizing
                self.encode(features, feature_lens, out=out)
        torch.cuda.current_stream(self.device).wait_stream(side)
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.encode(features, feature_lens, out=out, trace=trace)
        return graph, out

    def encode_stream(self, host_features, feature_lens, host_outs, graphs=None,
                      before_each=None):
        """Encodes a sequence of batches of one shape from pinned host memory
        into pinned host outputs: host_features[i] (bf16 [B, 128, T_max]) ->
        host_outs[i] (fp32 [total_tokens, output_dim]).  Every batch is copied
        in, encoded and copied back, and the copies of batches i + 1 and i - 1
        run on a second stream while batch i computes (two device buffer sets,
        each with its captured forward).  `graphs`, as returned by a previous
        call, skips the captures; `before_each`, if given, is called on the
        compute stream before every batch.  Returns (graphs, (start, end) CUDA
        events) around the whole sequence; the caller synchronises."""
        dev = self.device
        if graphs is None:
            graphs = []
            for _ in range(2):
                fd = torch.empty(host_features[0].shape, dtype=torch.bfloat16, device=dev)
                fd.copy_(host_features[0])
                out = torch.empty(host_outs[0].shape, dtype=torch.float32, device=dev)
                g, _ = self.capture(fd, feature_lens, out=out)
                graphs.append((g, fd, out))
        comp = torch.cuda.current_stream(dev)
        copy = torch.cuda.Stream(dev)
        h2d = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        d2h = [torch.cuda.Event() for _ in range(2)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = len(host_features)
        copy.wait_stream(comp)
        start.record(copy)
        with torch.cuda.stream(copy):
            graphs[0][1].copy_(host_features[0], non_blocking=True)
        h2d[0].record(copy)
        for i in range(n):
            j, jn = i % 2, (i + 1) % 2
            if i + 1 < n:  # next batch in, once batch i - 1 no longer reads that buffer
                if i >= 1:
                    copy.wait_event(done[jn])
                with torch.cuda.stream(copy):
                    graphs[jn][1].copy_(host_features[i + 1], non_blocking=True)
                h2d[jn].record(copy)
            comp.wait_event(h2d[j])
            if i >= 2:  # batch i - 2's result has left this output buffer
                comp.wait_event(d2h[j])
            if before_each is not None:
                before_each()
            graphs[j][0].replay()
            done[j].record(comp)
            copy.wait_event(done[j])
            with torch.cuda.stream(copy):
                host_outs[i].copy_(graphs[j][2], non_blocking=True)
            d2h[j].record(copy)
        end.record(copy)
        comp.wait_stream(copy)
        return graphs, (start, end)

    def check(self) -> int:
        """Device status of the latest call on this encoder's workspace."""
        return A.aut_check(self._ws.data_ptr()) if self._ws is not None else A.AUT_OK
