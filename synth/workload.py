"""Workload shapes and seeded input generation for the ISPA warmup path.

Shapes follow the video models the ISPA paper evaluates ("Towards Memory-Efficient
Autoregressive Video Generation via Instance-Specific Parametric Absorption", §4.1
Experimental Settings: 1.3B to 14B autoregressive video models). The paper's own videos,
prompts and weights are not available; every tensor here is drawn from a seeded normal
distribution instead:

* Q, K, V ~ N(0, 1), W_o ~ N(0, 1/D); values are rounded to bf16 (round to nearest even)
  for the bf16 workloads, so the oracle and the GPU read identical numbers.
* K/V are drawn per (layer, frame), so a frame holds the same keys and values in every
  chunk that sees it. Q is drawn per (layer, chunk).
* The "structured" workload plants absorbable layers: in even layers every frame's K/V is
  a fixed rank-16 template U·B plus 0.1·N(0, 1) drift; a scene cut redraws B.

The frame timeline (which frames sit in a layer's cache when chunk t is generated) is
part of the workload description and lives here too: frame 0 is the sink frame, chunk t
holds frames [f0 + c·t, f0 + c·t + c), and a full-attention layer keeps the sink plus the
(window - 1) most recent frames before the chunk (§3.1 Overall Framework; §3.3 for the
re-warmup after a scene cut). With f0 = h_max - c·(W - 1), the last warmup chunk sees
exactly h_max frames before it.

Random streams: numpy PCG64 seeded by SeedSequence(seed, spawn_key=(layer, kind, sub,
index)), so any single frame can be regenerated on its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

# spawn-key kinds
KIND_Q, KIND_K, KIND_V, KIND_W, KIND_U, KIND_B, KIND_DRIFT, KIND_AUX = range(8)


def make_rng(seed: int, *key: int) -> np.random.Generator:
    """PCG64 stream for one (layer, kind, sub, index) key."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(int(k) for k in key))))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    r = (b >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += b                      # finite values never wrap past 2^32
    r >>= 16
    return r.astype(np.uint16)


def f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _to_dtype_grid(x: np.ndarray, dtype: str) -> np.ndarray:
    """Return float32 values that are exactly representable in the workload dtype."""
    if dtype == "bf16":
        return f32_from_bf16_bits(bf16_bits_from_f32(x))
    return np.ascontiguousarray(x, dtype=np.float32)


@dataclass(frozen=True)
class IspaConfig:
    """One workload. Frame counts include the sink frame; `h_max` is the number of cached
    frames (sink included) in front of the last warmup chunk."""

    name: str
    layers: int
    heads: int
    head_dim: int
    tpf: int                  # tokens per latent frame
    chunk_frames: int         # frames generated per chunk (c)
    h_max: int                # cached frames before the last warmup chunk, sink included
    warmup_chunks: int        # W
    lam: float                # ridge regulariser
    K: int                    # layers switched to local attention
    dtype: str                # "fp32" | "bf16"
    sink_frames: int = 1
    window: Optional[int] = None        # cached frames kept by F-layers (default h_max)
    structured: bool = False
    planted_rank: int = 16
    drift: float = 0.1
    cut_chunk: Optional[int] = None     # scene cut: re-warmup starts at this chunk
    total_chunks: Optional[int] = None  # chunks in one streaming run (default W + 1)
    seed: int = 0
    sweep_K: Tuple[int, ...] = field(default_factory=tuple)

    @property
    def D(self) -> int:
        return self.heads * self.head_dim

    @property
    def n_q(self) -> int:
        return self.tpf * self.chunk_frames

    @property
    def first_chunk_frame(self) -> int:
        return self.h_max - self.chunk_frames * (self.warmup_chunks - 1)

    @property
    def kv_window(self) -> int:
        return self.window if self.window is not None else self.h_max

    @property
    def n_chunks(self) -> int:
        return self.total_chunks if self.total_chunks is not None else self.warmup_chunks + 1

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    def chunk_start_frame(self, t: int) -> int:
        return self.first_chunk_frame + self.chunk_frames * t

    def planted(self, layer: int) -> bool:
        return self.structured and layer % 2 == 0

    def epoch_of_frame(self, frame: int) -> int:
        if self.cut_chunk is None or frame < self.chunk_start_frame(self.cut_chunk):
            return 0
        return 1

    def n_kv_at_h(self, h_frames: int) -> int:
        return h_frames * self.tpf + self.n_q


def cache_frames(cfg: IspaConfig, t: int, hist_from: Optional[int] = None) -> List[int]:
    """Frames (time order) in a full-attention layer's cache while chunk t is generated:
    sink frame(s), then the most recent history frames, then the chunk's own frames.
    `hist_from` drops history frames older than that frame (a layer that evicted its
    history and started collecting again)."""
    start = cfg.chunk_start_frame(t)
    keep = cfg.kv_window - cfg.sink_frames
    lo = max(cfg.sink_frames, start - keep)
    if hist_from is not None:
        lo = max(lo, hist_from)
    sink = list(range(cfg.sink_frames))
    hist = list(range(lo, start)) if lo < start else []
    chunk = list(range(start, start + cfg.chunk_frames))
    return sink + hist + chunk


def chunk_layout(cfg: IspaConfig, frames: List[int], t: int) -> dict:
    """Row ranges of the sink and of the chunk inside a KV tensor built from `frames`."""
    start = cfg.chunk_start_frame(t)
    pos = {f: i for i, f in enumerate(frames)}
    sink_rows = (0, cfg.sink_frames * cfg.tpf)
    c0 = pos[start] * cfg.tpf
    return {
        "n_kv": len(frames) * cfg.tpf,
        "sink_begin": sink_rows[0],
        "sink_end": sink_rows[1],
        "chunk_begin": c0,
        "chunk_end": c0 + cfg.n_q,
    }


def _template(cfg: IspaConfig, layer: int, which: int, epoch: int) -> np.ndarray:
    """Rank-`planted_rank` frame template U·B for one layer and K (which=1) or V (which=2)."""
    r = cfg.planted_rank
    s = np.float32(r ** -0.25)        # U, B ~ N(0, 1/sqrt(r)) each: unit element variance (1/4 each at r = 16)
    U = make_rng(cfg.seed, layer, KIND_U, which, 0).standard_normal((cfg.tpf, r), dtype=np.float32) * s
    B = make_rng(cfg.seed, layer, KIND_B, which, epoch).standard_normal((r, cfg.D), dtype=np.float32) * s
    return U @ B


def frame_kv(cfg: IspaConfig, layer: int, frame: int, which: str) -> np.ndarray:
    """K (which='k') or V (which='v') of one frame: float32 [tpf, heads, head_dim]."""
    w = 1 if which == "k" else 2
    if cfg.planted(layer):
        base = _template(cfg, layer, w, cfg.epoch_of_frame(frame))
        noise = make_rng(cfg.seed, layer, KIND_DRIFT, w, frame).standard_normal(base.shape, dtype=np.float32)
        x = base + np.float32(cfg.drift) * noise
    else:
        x = make_rng(cfg.seed, layer, KIND_K if w == 1 else KIND_V, 0, frame).standard_normal(
            (cfg.tpf, cfg.D), dtype=np.float32)
    return _to_dtype_grid(x, cfg.dtype).reshape(cfg.tpf, cfg.heads, cfg.head_dim)


def chunk_q(cfg: IspaConfig, layer: int, t: int) -> np.ndarray:
    """Queries of chunk t in one layer: float32 [n_q, heads, head_dim]."""
    x = make_rng(cfg.seed, layer, KIND_Q, 0, t).standard_normal((cfg.n_q, cfg.D), dtype=np.float32)
    return _to_dtype_grid(x, cfg.dtype).reshape(cfg.n_q, cfg.heads, cfg.head_dim)


def w_out(cfg: IspaConfig, layer: int) -> np.ndarray:
    """Attention output projection W_o of one layer, stored [D_in, D_out] (y = A @ W_o)."""
    x = make_rng(cfg.seed, layer, KIND_W, 0, 0).standard_normal((cfg.D, cfg.D), dtype=np.float32)
    x *= np.float32(1.0 / np.sqrt(cfg.D))
    return _to_dtype_grid(x, cfg.dtype)


def kv_tensor(cfg: IspaConfig, layer: int, frames: List[int], which: str) -> np.ndarray:
    """Stack the K or V of `frames` into [len(frames)*tpf, heads, head_dim]."""
    return np.concatenate([frame_kv(cfg, layer, f, which) for f in frames], axis=0)


def normal_tensor(seed: int, key: Tuple[int, ...], shape: Tuple[int, ...], dtype: str, std: float = 1.0) -> np.ndarray:
    """Generic seeded N(0, std^2) tensor on the workload grid (used for unit-level cases)."""
    x = make_rng(seed, KIND_AUX, *key).standard_normal(shape, dtype=np.float32) * np.float32(std)
    return _to_dtype_grid(x, dtype)


# The five workloads. Sizes: tokens per frame, chunk frames and history frames from the
# 1.3B (12 heads x 128) and 14B (40 heads x 128) video models.
CONFIGS = {
    "tiny_fp32": IspaConfig(
        name="tiny_fp32", layers=1, heads=2, head_dim=64, tpf=64, chunk_frames=2, h_max=8,
        warmup_chunks=4, lam=1e-2, K=1, dtype="fp32"),
    "1p3b_bf16": IspaConfig(
        name="1p3b_bf16", layers=30, heads=12, head_dim=128, tpf=1560, chunk_frames=3, h_max=21,
        warmup_chunks=3, lam=1e-2, K=15, dtype="bf16"),
    "long_bf16": IspaConfig(
        name="long_bf16", layers=30, heads=12, head_dim=128, tpf=1560, chunk_frames=3, h_max=120,
        warmup_chunks=3, lam=1e-2, K=15, dtype="bf16"),
    "14b_bf16": IspaConfig(
        name="14b_bf16", layers=40, heads=40, head_dim=128, tpf=1560, chunk_frames=3, h_max=21,
        warmup_chunks=3, lam=1e-2, K=20, dtype="bf16"),
    "structured_bf16": IspaConfig(
        name="structured_bf16", layers=30, heads=12, head_dim=128, tpf=1560, chunk_frames=3, h_max=21,
        warmup_chunks=3, lam=1e-2, K=15, dtype="bf16", structured=True, cut_chunk=10, total_chunks=20,
        sweep_K=(7, 15)),
}
