"""Full-shape streaming runs for the GPU tests: every frame's K/V generated once on the host
(threads; seeded per (layer, kind, frame) by `synth`) and held on the device, so that a layer's
cache for a chunk is a device-side concatenation of frame runs instead of a host rebuild.

At the 1.3B shape one layer's frames 0..56 are 57 x 4.8 MB per K or V in bf16 (30 layers:
16.4 GB of device memory).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import synth
from streaming_video_attention_b200 import ispa
from streaming_video_attention_b200.session import IspaSession


class DeviceFrames:
    """K and V of frames [0, n_frames) of every layer as bf16 [n_frames * tpf, heads, head_dim]
    device tensors (bit-exact copies of synth.frame_kv)."""

    def __init__(self, cfg: synth.IspaConfig, n_frames: int, threads: Optional[int] = None):
        assert cfg.dtype == "bf16"
        self.cfg, self.n_frames = cfg, n_frames
        tpf, h, d = cfg.tpf, cfg.heads, cfg.head_dim
        threads = threads or max(1, min(32, os.cpu_count() or 8))
        self.kv: List[List[torch.Tensor]] = []
        host = np.empty((2, n_frames * tpf, cfg.D), dtype=np.uint16)

        def fill(which, f):
            x = synth.frame_kv(cfg, layer, f, "k" if which == 0 else "v").reshape(tpf, cfg.D)
            host[which, f * tpf:(f + 1) * tpf] = synth.bf16_bits_from_f32(x)

        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            for layer in range(cfg.layers):
                list(ex.map(lambda j: fill(*j), [(w, f) for w in range(2) for f in range(n_frames)]))
                t = torch.from_numpy(host.view(np.int16)).cuda().view(torch.bfloat16)
                self.kv.append([t[0].reshape(n_frames * tpf, h, d).clone(), t[1].reshape(n_frames * tpf, h, d).clone()])
                del t

    def cache(self, layer: int, frames: Sequence[int]):
        """(K, V) of `frames` (time order) stacked on the device."""
        tpf = self.cfg.tpf
        runs, start, prev = [], frames[0], frames[0]
        for f in list(frames[1:]) + [None]:
            if f is not None and f == prev + 1:
                prev = f
                continue
            runs.append((start, prev + 1))
            if f is not None:
                start = prev = f
        out = []
        for which in range(2):
            src = self.kv[layer][which]
            out.append(torch.cat([src[a * tpf:b * tpf] for a, b in runs], dim=0))
        return out[0], out[1]


def q_device(cfg: synth.IspaConfig, layer: int, t: int) -> torch.Tensor:
    bits = synth.bf16_bits_from_f32(synth.chunk_q(cfg, layer, t))
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def episode(cfg: synth.IspaConfig, store: DeviceFrames, K: int, n_chunks: int, rewarm: str = "cut",
            sample: Optional[Dict[tuple, np.ndarray]] = None):
    """A streaming run through IspaSession, as in the scaled-down configuration tests:
    rewarm "cut" re-enters the warmup at the workload's scene cut; "auto" monitors every F-layer
    after a transition and re-enters the warmup at the chunk after the trigger fired.
    sample maps (chunk, layer) -> query rows whose attention output (O: the full output of an
    F-layer, the local output of an L-layer) is returned for the oracle."""
    L = cfg.layers
    sess = IspaSession(L, cfg.heads, cfg.head_dim, cfg.lam, K, "bf16")
    W = []
    for l in range(L):
        bits = synth.bf16_bits_from_f32(synth.w_out(cfg, l))
        W.append(torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16))
    sess.set_weights(W)
    sess.reserve(cfg.n_q)
    sess.rewarm()
    hist_from: List[Optional[int]] = [None] * L
    warm_start, pending = 0, False
    transitions, fired, live, rows_out, frames_used = [], [], [], {}, {}
    o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.heads, cfg.n_q), device="cuda")
    y = torch.empty((cfg.n_q, cfg.D), dtype=torch.bfloat16, device="cuda")
    for t in range(n_chunks):
        scheduled = rewarm == "cut" and cfg.cut_chunk is not None and t == cfg.cut_chunk
        if scheduled or pending:
            for l in range(L):
                if sess.is_local[l]:
                    hist_from[l] = cfg.chunk_start_frame(t)
            sess.rewarm()
            warm_start, pending = t, False
        in_warmup = warm_start <= t < warm_start + cfg.warmup_chunks
        watch = rewarm == "auto" and sess.transitions > 0 and not in_warmup
        for l in range(L):
            q = q_device(cfg, l, t)
            if sess.is_local[l]:
                s0 = cfg.chunk_start_frame(t)
                frames = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))
                k, v = store.cache(l, frames)
                sess.local_attention(l, q, k, v, o, lse, y)
            else:
                frames = synth.cache_frames(cfg, t, hist_from[l])
                lay = synth.chunk_layout(cfg, frames, t)
                k, v = store.cache(l, frames)
                sess.full_attention(l, q, k, v, (lay["sink_begin"], lay["sink_end"]),
                                    (lay["chunk_begin"], lay["chunk_end"]), o, lse, collect=in_warmup, monitor=watch)
            if sample is not None and (t, l) in sample:
                rows_out[(t, l)] = o.float().cpu().numpy()[sample[(t, l)]].astype(np.float64)
                frames_used[(t, l)] = (list(frames), bool(sess.is_local[l]))
        if in_warmup:
            sess.flush_stats()
        if watch:
            live.append((t, sess.live_errors()))
            f = sess.rewarm_layers()
            fired.append((t, f))
            if f:
                pending = True
        if in_warmup and t == warm_start + cfg.warmup_chunks - 1:
            idx = sess.transition()
            transitions.append(dict(chunk=t, eps=list(sess.eps_host), idx=idx, is_local=list(sess.is_local)))
    torch.cuda.synchronize()
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    return dict(transitions=transitions, fired=fired, live=live, rows=rows_out, frames=frames_used)
