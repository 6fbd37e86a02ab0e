"""The seeded workload generator: determinism, frame reuse, dtype grid and the frame timeline."""
import numpy as np

import synth


def test_generation_is_deterministic_and_keyed():
    cfg = synth.CONFIGS["tiny_fp32"]
    a = synth.frame_kv(cfg, 0, 3, "k")
    b = synth.frame_kv(cfg, 0, 3, "k")
    assert np.array_equal(a, b)
    assert not np.array_equal(a, synth.frame_kv(cfg, 0, 4, "k"))
    assert not np.array_equal(a, synth.frame_kv(cfg, 0, 3, "v"))
    assert a.shape == (cfg.tpf, cfg.heads, cfg.head_dim) and a.dtype == np.float32


def test_bf16_workloads_sit_on_the_bf16_grid():
    cfg = synth.IspaConfig(name="t", layers=2, heads=2, head_dim=16, tpf=8, chunk_frames=2, h_max=4,
                           warmup_chunks=2, lam=1e-2, K=1, dtype="bf16")
    for x in (synth.frame_kv(cfg, 1, 2, "v"), synth.chunk_q(cfg, 0, 1), synth.w_out(cfg, 1)):
        bits = synth.bf16_bits_from_f32(x)
        assert np.array_equal(synth.f32_from_bf16_bits(bits), x)


def test_distributions():
    cfg = synth.CONFIGS["1p3b_bf16"]
    k = synth.frame_kv(cfg, 5, 7, "k")
    assert abs(k.mean()) < 5e-3 and abs(k.std() - 1) < 5e-3
    w = synth.w_out(cfg, 0)
    assert abs(w.std() * np.sqrt(cfg.D) - 1) < 1e-2


def test_timeline_1p3b():
    cfg = synth.CONFIGS["1p3b_bf16"]
    assert cfg.first_chunk_frame == 15
    sizes = []
    for t in range(4):
        fr = synth.cache_frames(cfg, t)
        lay = synth.chunk_layout(cfg, fr, t)
        sizes.append(len(fr) - cfg.chunk_frames)
        assert fr[0] == 0 and fr[-cfg.chunk_frames:] == list(range(15 + 3 * t, 18 + 3 * t))
        assert lay["chunk_end"] == lay["n_kv"] and lay["sink_end"] == cfg.tpf
    assert sizes == [15, 18, 21, 21]                      # warmup H = 15, 18, 21, then the window
    assert synth.chunk_layout(cfg, synth.cache_frames(cfg, 2), 2)["n_kv"] == 37440
    assert synth.cache_frames(cfg, 3)[1] == 4             # sink + the 20 most recent frames


def test_timeline_tiny_and_long():
    tiny = synth.CONFIGS["tiny_fp32"]
    assert [len(synth.cache_frames(tiny, t)) - 2 for t in range(4)] == [2, 4, 6, 8]
    assert synth.chunk_layout(tiny, synth.cache_frames(tiny, 3), 3)["n_kv"] == 640
    long = synth.CONFIGS["long_bf16"]
    assert [len(synth.cache_frames(long, t)) - 3 for t in range(3)] == [114, 117, 120]
    assert synth.chunk_layout(long, synth.cache_frames(long, 2), 2)["n_kv"] == 191880


def test_structured_template_and_cut():
    cfg = synth.IspaConfig(name="s", layers=2, heads=2, head_dim=16, tpf=32, chunk_frames=2, h_max=6,
                           warmup_chunks=3, lam=1e-2, K=1, dtype="fp32", structured=True, planted_rank=4,
                           cut_chunk=4, total_chunks=6)
    a = synth.frame_kv(cfg, 0, 1, "k").reshape(cfg.tpf, -1)
    b = synth.frame_kv(cfg, 0, 2, "k").reshape(cfg.tpf, -1)
    # same template, independent drift of std 0.1
    assert abs((a - b).std() - 0.1 * np.sqrt(2)) < 0.02
    cut_frame = cfg.chunk_start_frame(4)
    c = synth.frame_kv(cfg, 0, cut_frame, "k").reshape(cfg.tpf, -1)
    assert (a - c).std() > 1.0                            # the basis was redrawn at the cut
    # i.i.d. layer: no template shared between frames
    d1 = synth.frame_kv(cfg, 1, 1, "k").reshape(cfg.tpf, -1)
    d2 = synth.frame_kv(cfg, 1, 2, "k").reshape(cfg.tpf, -1)
    assert (d1 - d2).std() > 1.3
    assert cfg.planted(0) and not cfg.planted(1)


def test_history_restart_after_eviction():
    cfg = synth.CONFIGS["structured_bf16"]
    t = cfg.cut_chunk
    fr = synth.cache_frames(cfg, t, hist_from=cfg.chunk_start_frame(t))
    assert fr == [0] + list(range(cfg.chunk_start_frame(t), cfg.chunk_start_frame(t) + 3))
