#!/usr/bin/env python
"""Benchmark of the ISPA warmup hot path on B200.

One step = one streaming episode of the 1.3B-shaped workload on every GPU (replicas):
  * 3 warmup chunks x 30 layers of split attention with fused ridge statistics
    (history 15, 18, 21 frames: n_kv = 28,080 / 32,760 / 37,440 rows, n_q = 4,680),
  * the transition: absorb solve + reconstruction error for 30 layers (D = 1536),
    selection of K = 15 L-layers on the host, W_new = W + dW,
  * one post-transition chunk: 15 L-layers of local attention (sink + chunk, 6,240 rows)
    with the W_new projection, 15 F-layers of full attention (sink + 20 frames + chunk).
value = query tokens through the model per second = (4 chunks x 4,680 queries x N GPUs) /
step time (max over ranks). Inputs are seeded synthetic tensors (same recipe as the
oracle tests), resident in HBM before the timed region; ~20 GB are touched per step, far
more than L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ispa|reference]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "query tokens/s through split attention+absorb stats; % of BF16 tensor peak"
UNIT = "query tokens/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ispa", "reference"], default="ispa")
    ap.add_argument("--config", default="1p3b_bf16")
    ap.add_argument("--e2e-steps", type=int, default=10,
                    help="timed steps of the end-to-end leg (its first step's copies are the pipeline fill)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shapes", action="store_true",
                    help="skip the one-layer call timings of the 1.3B, long-history and 14B shapes")
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--mode", choices=["episode", "call", "local", "solve", "stats"], default="episode",
                    help="episode: the full step (default). call / local / solve: one layer's fused split "
                         "attention at the last warmup chunk, one L-layer local attention with projection, or "
                         "the batched solve alone, or one warmup chunk's batched statistics launch (kernel-level "
                         "timing, also the target of ncu captures)")
    ap.add_argument("--stats-layers", type=int, default=0,
                    help="stats mode: layers in the batched statistics launch (default: the workload's layers)")
    ap.add_argument("--i8", action="store_true",
                    help="call mode: the 8-bit split attention (int8 Q and K, quantised inside the timed call)")
    ap.add_argument("--w8a8", action="store_true",
                    help="local mode: the L-layer projection through int8 weights and activations")
    ap.add_argument("--attn-kernel", choices=["auto", "single", "pair", "two_group"], default="auto",
                    help="bf16 head_dim-128 attention kernel: one CTA per query tile, CTA pairs "
                         "(cta_group::2), or one CTA with two softmax groups; auto = the library's default")
    return ap.parse_args(argv)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum, ncu) per launch of the kernels the
# roofline object describes, each tied to the sha256 of the sources it was captured from: a figure
# is reported only while those sources are unchanged, otherwise the line's traffic is null.
# The path is the episode's: one ispa_attn_split_ops launch per warmup layer call and one batched
# ispa_accum_ops launch per chunk, whose bytes are charged to the chunk's layers equally.
# None: not yet captured for the current sources.
_PTX = ("streaming_video_attention_b200/csrc/ptx.cuh",
        "0353fca5187d1129c0e7936a8baa86b17e79672c07a933ea5a5f127e77d94af0")
CAPTURED_TRAFFIC = {
    "workload": "1p3b_bf16",
    # the 90 warmup launches of one timed episode, averaged (n_kv 28,080 / 32,760 / 37,440)
    "attention": {"two_group": (240.3e6, dict([_PTX, ("streaming_video_attention_b200/csrc/attn2g_sm100.cu",
                                                      "3bed3806f2e152d01cb932a529d3f79da812540a4b19e6fbb52febc93f129433")]))},
    # the episode's three 30-layer statistics launches (3.08 GB each), per layer
    "stats_per_layer": (102.75e6, dict([_PTX, ("streaming_video_attention_b200/csrc/stats_sm100.cu",
                                               "b6b42e9369b57a364c239b9be97ce127908ae56800a6f12cfa6448475cd0e748")])),
}


def captured_traffic(cfg, attn_kernel: str):
    """DRAM bytes per warmup layer call on the timed path (attention launch + its share of the
    chunk's statistics launch), or None."""
    import hashlib
    kernel = "two_group" if attn_kernel == "auto" else attn_kernel
    if cfg.name != CAPTURED_TRAFFIC["workload"] or kernel not in CAPTURED_TRAFFIC["attention"]:
        return None
    total = 0.0
    for nbytes, sources in (CAPTURED_TRAFFIC["attention"][kernel], CAPTURED_TRAFFIC["stats_per_layer"]):
        if nbytes is None:
            return None
        for rel, digest in sources.items():
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        total += nbytes
    return total


DATASHEET_DENSE_BF16_TFLOPS = 2250.0   # B200 dense bf16 (the 2:4-sparse figure halved)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# --------------------------------------------------------------------------- workload
class Workload:
    """Host (pinned) and device copies of one episode's inputs."""

    def __init__(self, cfg: synth.IspaConfig, threads: int):
        self.cfg = cfg
        W = cfg.warmup_chunks
        self.post_t = W
        self.n_frames = cfg.chunk_start_frame(W) + cfg.chunk_frames       # frames 0 .. last post-chunk frame
        tpf, h, d = cfg.tpf, cfg.heads, cfg.head_dim
        L = cfg.layers
        self.kv_host = [[torch.empty((self.n_frames * tpf, h, d), dtype=torch.bfloat16, pin_memory=True)
                         for _ in range(2)] for _ in range(L)]
        self.q_host = [torch.empty((W + 1, cfg.n_q, h, d), dtype=torch.bfloat16, pin_memory=True) for _ in range(L)]
        self.w_host = [torch.empty((cfg.D, cfg.D), dtype=torch.bfloat16, pin_memory=True) for _ in range(L)]

        def bits(t):
            return t.view(torch.int16).numpy().view(np.uint16)

        def fill_frame(l, f, which):
            x = synth.frame_kv(cfg, l, f, which)
            bits(self.kv_host[l][0 if which == "k" else 1])[f * tpf:(f + 1) * tpf] = synth.bf16_bits_from_f32(x)

        def fill_q(l, t):
            bits(self.q_host[l])[t] = synth.bf16_bits_from_f32(synth.chunk_q(cfg, l, t))

        def fill_w(l):
            bits(self.w_host[l])[:] = synth.bf16_bits_from_f32(synth.w_out(cfg, l))

        jobs = [(fill_frame, (l, f, wh)) for l in range(L) for f in range(self.n_frames) for wh in ("k", "v")]
        jobs += [(fill_q, (l, t)) for l in range(L) for t in range(W + 1)]
        jobs += [(fill_w, (l,)) for l in range(L)]
        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda j: j[0](*j[1]), jobs))

        # per-chunk KV geometry
        self.warm = []
        for t in range(W):
            fr = synth.cache_frames(cfg, t)
            lay = synth.chunk_layout(cfg, fr, t)
            assert fr == list(range(len(fr))), "warmup caches are contiguous frame prefixes"
            self.warm.append(lay)
        self.post_frames = synth.cache_frames(cfg, self.post_t)
        self.post_layout = synth.chunk_layout(cfg, self.post_frames, self.post_t)
        s0 = cfg.chunk_start_frame(self.post_t)
        self.local_frames = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))

    def h2d_bytes(self) -> int:
        b = 0
        for l in range(self.cfg.layers):
            b += sum(t.numel() * 2 for t in self.kv_host[l]) + self.q_host[l].numel() * 2 + self.w_host[l].numel() * 2
        return b


class DeviceInputs:
    def __init__(self, wl: Workload, device):
        cfg = wl.cfg
        tpf = cfg.tpf
        L = cfg.layers
        self.wl = wl
        self.kv = [[torch.empty_like(wl.kv_host[l][i], device=device) for i in range(2)] for l in range(L)]
        self.q = [torch.empty_like(wl.q_host[l], device=device) for l in range(L)]
        self.w = [torch.empty_like(wl.w_host[l], device=device) for l in range(L)]
        n_post, n_loc = len(wl.post_frames) * tpf, len(wl.local_frames) * tpf
        h, d = cfg.heads, cfg.head_dim
        self.kv_post = [[torch.empty((n_post, h, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
                        for _ in range(L)]
        self.kv_loc = [[torch.empty((n_loc, h, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
                       for _ in range(L)]

    def upload(self, stream=None):
        """Host -> device copies of the step's inputs, then the derived post-transition caches."""
        self.upload_h2d()
        self.derive()

    def upload_h2d(self):
        """Host -> device copies of the step's inputs (on the current stream)."""
        wl = self.wl
        for l in range(wl.cfg.layers):
            for i in range(2):
                self.kv[l][i].copy_(wl.kv_host[l][i], non_blocking=True)
            self.q[l].copy_(wl.q_host[l], non_blocking=True)
            self.w[l].copy_(wl.w_host[l], non_blocking=True)

    def derive(self):
        wl = self.wl
        tpf = wl.cfg.tpf
        for l in range(wl.cfg.layers):
            for i in range(2):
                src = self.kv[l][i]
                for dst, frames in ((self.kv_post[l][i], wl.post_frames), (self.kv_loc[l][i], wl.local_frames)):
                    # frames are runs of consecutive indices: copy run by run
                    pos = 0
                    start = frames[0]
                    prev = frames[0]
                    for f in frames[1:] + [None]:
                        if f is not None and f == prev + 1:
                            prev = f
                            continue
                        n = prev - start + 1
                        dst[pos * tpf:(pos + n) * tpf].copy_(src[start * tpf:(prev + 1) * tpf], non_blocking=True)
                        pos += n
                        if f is not None:
                            start = prev = f


class Outputs:
    def __init__(self, cfg, device):
        L = cfg.layers
        self.o = [torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device=device)
                  for _ in range(L)]
        self.lse = [torch.empty((cfg.heads, cfg.n_q), dtype=torch.float32, device=device) for _ in range(L)]
        self.y = [torch.empty((cfg.n_q, cfg.D), dtype=torch.bfloat16, device=device) for _ in range(L)]


def _timed(timers, flops, fn, kind):
    if timers is None:
        fn()
        return
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    fn()
    ev1.record()
    timers.append((ev0, ev1, flops, kind))


def run_episode(sess, dev: DeviceInputs, out: Outputs, timers=None):
    """One streaming episode: warmup chunks -> transition -> one post-transition chunk. Each
    warmup chunk runs every layer's split attention (writing its statistics operands), then one
    statistics launch for all layers."""
    cfg = dev.wl.cfg
    sess.rewarm()
    for t, lay in enumerate(dev.wl.warm):
        n_kv = lay["n_kv"]
        sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
        for l in range(cfg.layers):
            _timed(timers, 4.0 * cfg.n_q * n_kv * cfg.head_dim * cfg.heads,
                   lambda: sess.full_attention(l, dev.q[l][t], dev.kv[l][0][:n_kv], dev.kv[l][1][:n_kv], sink, chunk,
                                               out.o[l], out.lse[l], collect=True), "attention")
        _timed(timers, cfg.layers * 4.0 * cfg.n_q * cfg.D * cfg.D, sess.flush_stats, "statistics")
    sess.transition()
    t = dev.wl.post_t
    lay = dev.wl.post_layout
    sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
    for l in range(cfg.layers):
        if sess.is_local[l]:
            sess.local_attention(l, dev.q[l][t], dev.kv_loc[l][0], dev.kv_loc[l][1], out.o[l], out.lse[l], out.y[l])
        else:
            sess.full_attention(l, dev.q[l][t], dev.kv_post[l][0], dev.kv_post[l][1], sink, chunk, out.o[l],
                                out.lse[l], collect=False)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = os.path.join("/tmp", f"ispa_clocks_{os.getpid()}_{gpu_index}.csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(gpu_index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def physical_gpu_index(local_rank: int) -> int:
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    if local_rank < len(vis) and vis[local_rank].isdigit():
        return int(vis[local_rank])
    return local_rank


# --------------------------------------------------------------------------- CPU oracle sample
def oracle_parts(cfg, rows: int) -> dict:
    """Time the oracle on one bounded sample of the episode's calls: `rows` query rows of one
    layer's last warmup call -- the split attention over explicit masks, and the statistics of
    those rows -- and the same rows through one L-layer call (attention over the sink and chunk
    rows, projection with W + dW). Returns seconds per part and the sample's KV row counts."""
    import oracle
    t = cfg.warmup_chunks - 1
    frames = synth.cache_frames(cfg, t)
    lay = synth.chunk_layout(cfg, frames, t)
    q = synth.chunk_q(cfg, 0, t)[:rows]
    k = synth.kv_tensor(cfg, 0, frames, "k")
    v = synth.kv_tensor(cfg, 0, frames, "v")
    s0 = cfg.chunk_start_frame(t)
    loc = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))
    pos = {f: i for i, f in enumerate(frames)}
    loc_rows = np.concatenate([np.arange(pos[f] * cfg.tpf, (pos[f] + 1) * cfg.tpf) for f in loc])
    W = synth.w_out(cfg, 0).astype(np.float64)
    t0 = time.perf_counter()
    res = oracle.split_attention(q, k, v, (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"]),
                                 cfg.scale)
    t1 = time.perf_counter()
    st = oracle.stats_init(cfg.D)
    oracle.stats_update(st, res["A_loc"], res["A_full"], cfg.dtype)
    t2 = time.perf_counter()
    A, _ = oracle.local_attention(q, k[loc_rows], v[loc_rows], cfg.scale)
    oracle.project(A, W)
    t3 = time.perf_counter()
    return {"attn": t1 - t0, "stats": t2 - t1, "local": t3 - t2, "n_kv": lay["n_kv"], "n_loc": len(loc_rows),
            "rows": rows}


def oracle_transition(cfg) -> float:
    """The oracle's transition in full: absorb solve (dense LU) + reconstruction error for every
    layer and the selection, on statistics of three warmup chunks' rows built once from seeded
    operands outside the timing. Returns seconds."""
    import oracle
    n = cfg.warmup_chunks * cfg.n_q
    a = synth.normal_tensor(5, (1,), (n, cfg.D), cfg.dtype, std=0.05).astype(np.float64)
    r = synth.normal_tensor(5, (2,), (n, cfg.D), cfg.dtype, std=0.05).astype(np.float64)
    st = oracle.stats_init(cfg.D)
    oracle.stats_update(st, a.reshape(n, cfg.heads, -1), (a + r).reshape(n, cfg.heads, -1), cfg.dtype)
    Ws = [synth.w_out(cfg, l).astype(np.float64) for l in range(cfg.layers)]
    t0 = time.perf_counter()
    eps = []
    for W in Ws:
        dW = oracle.absorb_solve(st["G"], st["C"], W, cfg.lam)
        eps.append(oracle.reconstruction_error(st["G"], st["C"], st["H"], W, dW)["eps"])
    oracle.select_layers(eps, cfg.K)
    return time.perf_counter() - t0


def oracle_episode_seconds(cfg, parts: dict, t_transition: float) -> float:
    """The oracle's time for one episode: each warmup call's attention scaled from the sample
    linearly in query rows and KV rows, its statistics linearly in query rows (their cost does
    not depend on the KV rows), the transition as timed, then the post-transition chunk (F-layers:
    split attention; L-layers: local attention + projection)."""
    per_row = cfg.n_q / parts["rows"]
    est = 0.0
    for t in range(cfg.warmup_chunks):
        n_kv = synth.chunk_layout(cfg, synth.cache_frames(cfg, t), t)["n_kv"]
        est += cfg.layers * (parts["attn"] * per_row * n_kv / parts["n_kv"] + parts["stats"] * per_row)
    est += t_transition
    post = synth.chunk_layout(cfg, synth.cache_frames(cfg, cfg.warmup_chunks), cfg.warmup_chunks)["n_kv"]
    est += (cfg.layers - cfg.K) * parts["attn"] * per_row * post / parts["n_kv"]
    est += cfg.K * parts["local"] * per_row
    return est


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


# --------------------------------------------------------------------------- arms
def cpu_baseline_block(cfg, rows: int, parts_list, t_transition: float) -> dict:
    """The oracle's throughput on this host's cores from sampled calls and a timed transition."""
    parts = {key: statistics.mean(p[key] for p in parts_list) for key in ("attn", "stats", "local")}
    parts.update(n_kv=parts_list[0]["n_kv"], n_loc=parts_list[0]["n_loc"], rows=rows)
    episode_s = oracle_episode_seconds(cfg, parts, t_transition)
    sampled = sum(p["attn"] + p["stats"] + p["local"] for p in parts_list)
    sample = (f"{rows} query rows of one layer's last warmup call (n_kv {parts['n_kv']}): float64 split attention "
              f"over explicit masks {parts['attn']:.2f} s, statistics {parts['stats']:.2f} s, L-layer local attention "
              f"(n_kv {parts['n_loc']}) + projection {parts['local']:.2f} s (mean of {len(parts_list)}), scaled "
              f"linearly to every call of the episode (attention in rows x KV rows, the rest in rows); the "
              f"transition (dense-LU absorb solve + error for {cfg.layers} layers at D = {cfg.D}, selection) timed "
              f"in full: {t_transition:.2f} s")
    return {"value": (cfg.warmup_chunks + 1) * cfg.n_q / episode_s, "unit": UNIT, "cores": cpu_threads(),
            "kind": "oracle", "sample": sample, "extrapolated": True, "episode_s_estimate": episode_s,
            "sampled_s": sampled + t_transition, "transition_s": t_transition}


def reference_arm(args, cfg, rank):
    """The oracle timed on the host's cores. Each step is a bounded sample of the episode (one
    layer call's sampled rows through the attention, the statistics and the L-layer call); the
    transition is timed in full once; the line's value is the episode's query tokens over the
    oracle's estimated episode time, and ms_per_step is the time of a sampled step as run."""
    if rank != 0:
        return 0
    rows = args.cpu_rows
    for _ in range(args.warmup):
        oracle_parts(cfg, max(8, rows // 8))
    parts_list = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        parts_list.append(oracle_parts(cfg, rows))
    step_ms = (time.perf_counter() - t0) / max(1, args.steps) * 1e3
    t_transition = oracle_transition(cfg)
    cpu = cpu_baseline_block(cfg, rows, parts_list, t_transition)
    value = cpu["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, args.gpus), "extrapolated": True,
        "episode_ms_estimate": cpu["episode_s_estimate"] * 1e3,
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def kv_block(cfg, is_local):
    """K/V bytes held per replica before the transition (every layer F) and after it (the
    selected L-layers keep only the sink and the chunk)."""
    from streaming_video_attention_b200.session import kv_cache_bytes
    hist = cfg.kv_window - cfg.sink_frames
    args = (hist, cfg.chunk_frames, cfg.sink_frames, cfg.tpf, cfg.D, 2)
    before = kv_cache_bytes([0] * cfg.layers, *args)
    after = kv_cache_bytes(is_local, *args)
    return {"before_bytes": before, "after_bytes": after, "removed_frac": (before - after) / before,
            "l_layers": int(sum(is_local))}


def config_block(cfg, n):
    return {
        "workload": (f"{cfg.name}: ISPA episode, {cfg.layers} layers x {cfg.heads} heads x {cfg.head_dim}, "
                     f"{cfg.tpf} tokens/frame, chunk {cfg.chunk_frames} frames ({cfg.n_q} queries), warmup history "
                     f"{[len(synth.cache_frames(cfg, t)) - cfg.chunk_frames for t in range(cfg.warmup_chunks)]} "
                     f"frames, transition (solve + error + select K={cfg.K}), 1 post-transition chunk"),
        "layers": cfg.layers, "heads": cfg.heads, "head_dim": cfg.head_dim, "n_q": cfg.n_q,
        "warmup_chunks": cfg.warmup_chunks, "K": cfg.K, "lambda": cfg.lam,
        "l2": "inputs larger than L2 (about 20 GB touched per step)", "parallelism": f"replicas x{n}",
    }


def ispa_arm(args, cfg, rank, world, local_rank):
    from streaming_video_attention_b200 import ispa, replicas
    from streaming_video_attention_b200.session import IspaSession

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    ispa.lib()
    cfg = replicas.replica_config(cfg, rank)
    threads = max(1, (os.cpu_count() or 8) // max(1, int(os.environ.get("LOCAL_WORLD_SIZE", world))))
    t0 = time.time()
    wl = Workload(cfg, threads)
    gen_s = time.time() - t0
    dev = DeviceInputs(wl, device)
    dev.upload()
    out = Outputs(cfg, device)
    sess = IspaSession(cfg.layers, cfg.heads, cfg.head_dim, cfg.lam, cfg.K, "bf16", str(device))
    sess.set_weights(dev.w)
    sess.reserve(cfg.n_q)
    torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        run_episode(sess, dev, out)
    torch.cuda.synchronize()
    assert ispa.ispa_device_status() == ispa.ISPA_OK

    # ---- timed region: device-resident inputs
    clocks = ClockSampler(physical_gpu_index(local_rank))
    time.sleep(0.4)
    timers = []
    launches0 = ispa.ispa_kernel_launches()
    replicas.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        run_episode(sess, dev, out, timers)
    e1.record()
    torch.cuda.synchronize()
    replicas.barrier()
    launches = ispa.ispa_kernel_launches() - launches0
    clk = clocks.stop()
    value, elapsed = replicas.job_throughput(args.steps * (cfg.warmup_chunks + 1) * cfg.n_q,
                                             e0.elapsed_time(e1) / 1e3, device)
    ms_per_step = elapsed / args.steps * 1e3

    # roofline of the warmup's split attention + statistics (the dominant kernel pair): every
    # layer call and every chunk's statistics launch of the timed episodes
    flops = 0.0
    secs = 0.0
    by_kind = {"attention": [0.0, 0], "statistics": [0.0, 0]}
    for ev0, ev1, f, kind in timers:
        dt = ev0.elapsed_time(ev1) / 1e3
        secs += dt
        flops += f
        by_kind[kind][0] += dt
        by_kind[kind][1] += 1
    burst, sustained, hbm, peak_kind = peaks()
    achieved = flops / secs / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
            "frac": achieved / sustained, "traffic": captured_traffic(cfg, args.attn_kernel),
            "kernel": "warmup split attention (ispa_attn_split_ops) + statistics GEMM (ispa_accum_ops, one launch "
                      "per chunk for all layers)",
            "attn_kernel": "two_group" if args.attn_kernel == "auto" else args.attn_kernel,
            "peak_kind": f"{peak_kind} sustained bf16 (timed inside a long step)",
            "frac_of_burst_peak": achieved / burst,
            "frac_of_datasheet_dense_bf16": achieved / DATASHEET_DENSE_BF16_TFLOPS,
            "per_call_ms": secs / max(1, args.steps * cfg.warmup_chunks * cfg.layers) * 1e3,
            "attention_ms_per_call": by_kind["attention"][0] / max(1, by_kind["attention"][1]) * 1e3,
            "statistics_ms_per_chunk_of_all_layers": by_kind["statistics"][0] / max(1, by_kind["statistics"][1]) * 1e3}

    # ---- end to end through the public API, host buffers in the timed region
    e2e = None
    if not args.no_e2e:
        # A streaming caller prefetches: the next step's inputs are copied host -> device on a
        # copy stream (into the second of two device buffers) while the current step computes.
        # Every step's copies, its episode, the read-back of its outputs and of its errors lie
        # inside the timed region.
        host_o = [torch.empty_like(out.o[l], device="cpu").pin_memory() for l in range(cfg.layers)]
        d2h = sum(o.numel() * 2 for o in host_o) + cfg.layers * 4
        bufs = [dev, DeviceInputs(wl, device)]
        copy_stream = torch.cuda.Stream(device=device)
        main = torch.cuda.current_stream(device)
        released = [None, None]   # compute is done with that buffer

        def upload_into(b, after):
            copy_stream.wait_event(after)
            if released[b] is not None:
                copy_stream.wait_event(released[b])
            with torch.cuda.stream(copy_stream):
                bufs[b].upload_h2d()
            ev = torch.cuda.Event()
            ev.record(copy_stream)
            return ev

        def run_pipelined(steps):
            start = torch.cuda.Event()
            start.record(main)
            ready = upload_into(0, start)
            for step in range(steps):
                b = step % 2
                nxt = upload_into(1 - b, start) if step + 1 < steps else None
                main.wait_event(ready)
                # the post-transition caches are derived on the compute stream, which has slack,
                # so that the copy stream carries only host -> device traffic
                bufs[b].derive()
                sess.set_weights(bufs[b].w)   # this step's copy of W, not the one being refilled
                run_episode(sess, bufs[b], out)
                for l in range(cfg.layers):
                    host_o[l].copy_(out.o[l], non_blocking=True)
                released[b] = torch.cuda.Event()
                released[b].record(main)
                sess.eps.cpu()
                ready = nxt

        run_pipelined(2)
        torch.cuda.synchronize()
        replicas.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        run_pipelined(args.e2e_steps)
        f1.record()
        torch.cuda.synchronize()
        sess.set_weights(dev.w)
        e2e_value, et = replicas.job_throughput(args.e2e_steps * (cfg.warmup_chunks + 1) * cfg.n_q,
                                                f0.elapsed_time(f1) / 1e3, device)
        e2e = {"value": e2e_value, "unit": UNIT,
               "h2d_bytes_per_step": wl.h2d_bytes(), "d2h_bytes_per_step": d2h,
               "ms_per_step": et / args.e2e_steps * 1e3, "steps": args.e2e_steps,
               "overlap": "next step's host->device copies on a copy stream during this step's compute; "
                          "the first step's copies (pipeline fill) inside the timed region too"}

    assert ispa.ispa_device_status() == ispa.ISPA_OK

    shapes = None
    if world == 1 and not args.no_shapes:
        shapes = shape_calls(device, steps=5, warmup=3, threads=threads)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        parts = oracle_parts(cfg, args.cpu_rows)
        cpu = cpu_baseline_block(cfg, args.cpu_rows, [parts], oracle_transition(cfg))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_block(cfg, world),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches), "clocks": clk,
            "selection": {"idx": sess.idx, "margin": sess.selection_margin()},
            "kv_cache": kv_block(cfg, sess.is_local),
            "shapes": shapes,
            "input_generation_s": gen_s,
        }
        print(json.dumps(line), flush=True)
    return 0


def kv_device(cfg, layer: int, frames, which: str, device, threads: int) -> torch.Tensor:
    """K or V of `frames` (time order) on the device, bf16, generated frame by frame on `threads`
    host threads (the same bytes as synth.kv_tensor)."""
    tpf = cfg.tpf
    host = np.empty((len(frames) * tpf, cfg.D), dtype=np.uint16)

    def fill(i):
        x = synth.frame_kv(cfg, layer, frames[i], which).reshape(tpf, cfg.D)
        host[i * tpf:(i + 1) * tpf] = synth.bf16_bits_from_f32(x)

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(len(frames))))
    t = torch.from_numpy(host.view(np.int16)).to(device).view(torch.bfloat16)
    return t.reshape(len(frames) * tpf, cfg.heads, cfg.head_dim)


def shape_calls(device, steps: int, warmup: int, threads: int) -> dict:
    """One layer's warmup call (split attention with the statistics fused, the library's call for
    a single layer) at the last warmup chunk of each model shape, timed alone with CUDA events,
    L2 flushed (a 256 MB write) before every call; median of `steps`. The roofline fraction takes
    the measured burst peak (a kernel pair timed alone); hbm_gbs is the call's algorithmic bytes
    (Q, K, V, O and lse once) over its time."""
    from streaming_video_attention_b200.session import IspaSession

    burst, _, hbm, _ = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    out = {}
    for name in ("1p3b_bf16", "long_bf16", "14b_bf16"):
        cfg = synth.CONFIGS[name]
        t = cfg.warmup_chunks - 1
        frames = synth.cache_frames(cfg, t)
        lay = synth.chunk_layout(cfg, frames, t)
        n_kv = lay["n_kv"]
        q = torch.from_numpy(synth.bf16_bits_from_f32(synth.chunk_q(cfg, 0, t)).view(np.int16)).to(device)
        q = q.view(torch.bfloat16)
        k = kv_device(cfg, 0, frames, "k", device, threads)
        v = kv_device(cfg, 0, frames, "v", device, threads)
        sess = IspaSession(1, cfg.heads, cfg.head_dim, cfg.lam, 1, "bf16", str(device), batch_stats=False)
        sess.reserve(cfg.n_q)
        o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device=device)
        lse = torch.empty((cfg.heads, cfg.n_q), dtype=torch.float32, device=device)
        sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
        times = []
        for i in range(warmup + steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sess.full_attention(0, q, k, v, sink, chunk, o, lse, collect=True)
            e1.record()
            torch.cuda.synchronize()
            if i >= warmup:
                times.append(e0.elapsed_time(e1) / 1e3)
        dt = statistics.median(times)
        flops = 4.0 * cfg.n_q * n_kv * cfg.head_dim * cfg.heads + 4.0 * cfg.n_q * cfg.D * cfg.D
        nbytes = 2.0 * (2 * cfg.n_q + 2 * n_kv) * cfg.D + 4.0 * cfg.heads * cfg.n_q
        out[name] = {"n_q": cfg.n_q, "n_kv": n_kv, "heads": cfg.heads, "D": cfg.D, "ms": dt * 1e3,
                     "query_tokens_per_s": cfg.n_q / dt, "tflops": flops / dt / 1e12,
                     "frac_of_burst_peak": flops / dt / 1e12 / burst,
                     "hbm_gbs": nbytes / dt / 1e9, "frac_of_hbm_peak": nbytes / dt / 1e9 / hbm}
        del q, k, v, sess, o, lse
        torch.cuda.empty_cache()
    return out


def unit_arm(args, cfg):
    """Kernel-level timing of one unit of the path, inputs resident, L2 flushed between
    iterations (a 256 MB write)."""
    from streaming_video_attention_b200 import ispa
    from streaming_video_attention_b200.session import IspaSession

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)

    def up(x):
        return torch.from_numpy(synth.bf16_bits_from_f32(x).view(np.int16)).view(torch.bfloat16).to(device)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    t = cfg.warmup_chunks - 1
    D = cfg.D
    sess = IspaSession(1 if args.mode != "solve" else cfg.layers, cfg.heads, cfg.head_dim, cfg.lam, 1, "bf16",
                       str(device), w8a8=args.w8a8, batch_stats=False)   # one layer's call, statistics fused
    if args.mode in ("call", "local"):
        if args.mode == "call":
            frames = synth.cache_frames(cfg, t)
        else:
            t = cfg.warmup_chunks
            s0 = cfg.chunk_start_frame(t)
            frames = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))
        lay = synth.chunk_layout(cfg, frames, t)
        q = up(synth.chunk_q(cfg, 0, t))
        k = up(synth.kv_tensor(cfg, 0, frames, "k"))
        v = up(synth.kv_tensor(cfg, 0, frames, "v"))
        W = up(synth.w_out(cfg, 0))
        sess.set_weights([W])
        sess.W_new[0].copy_(W)
        sess.reserve(cfg.n_q)
        o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device=device)
        lse = torch.empty((cfg.heads, cfg.n_q), dtype=torch.float32, device=device)
        y = torch.empty((cfg.n_q, D), dtype=torch.bfloat16, device=device)
        n_kv = lay["n_kv"]
        if args.mode == "call":
            sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
            fn = lambda: sess.full_attention(0, q, k, v, sink, chunk, o, lse, collect=True)
            flops = 4.0 * cfg.n_q * n_kv * cfg.head_dim * cfg.heads + 4.0 * cfg.n_q * D * D
            what = f"fused split attention + statistics, one layer, n_q {cfg.n_q}, n_kv {n_kv}"
            if args.i8:
                desc = ispa.make_desc(cfg.n_q, n_kv, cfg.heads, cfg.head_dim, sink, chunk)
                q8 = torch.empty(q.shape, dtype=torch.int8, device=device)
                k8 = torch.empty(k.shape, dtype=torch.int8, device=device)
                qs = torch.empty((cfg.n_q, cfg.heads), dtype=torch.float32, device=device)
                ks = torch.empty((cfg.heads, ispa.ispa_k_blocks(desc)), dtype=torch.float32, device=device)
                ws = ispa.alloc_workspace(ispa.workspace_bytes(desc, 0, 0))
                st = sess.stats[0]

                def attn_only():
                    ispa.ispa_attn_split_i8(desc, q8, qs, k8, ks, v, o, lse, stats=st, ws=ws)

                def fn():
                    ispa.ispa_quantize_q_i8(q, q8, qs)
                    ispa.ispa_quantize_k_i8(desc, k, k8, ks)
                    attn_only()
                what = ("8-bit split attention (int8 Q/K quantised in the call) + statistics, one layer, "
                        f"n_q {cfg.n_q}, n_kv {n_kv}")
        else:
            sess.is_local = [1]
            if args.w8a8:
                sess.wq[0] = torch.empty(D, D, dtype=torch.int8, device=device)
                sess.wq_scale[0] = torch.empty(D, dtype=torch.float32, device=device)
                ispa.ispa_quantize_w8(sess.W_new[0], ispa.ISPA_BF16, sess.wq[0], sess.wq_scale[0])
            fn = lambda: sess.local_attention(0, q, k, v, o, lse, y)
            flops = 4.0 * cfg.n_q * n_kv * cfg.head_dim * cfg.heads + 2.0 * cfg.n_q * D * D
            what = (f"L-layer local attention + W_new projection{' (W8A8 int8)' if args.w8a8 else ''}, "
                    f"n_q {cfg.n_q}, n_kv {n_kv}")
    elif args.mode == "stats":
        # one warmup chunk's statistics: the operands of every layer [layers][n_q][D] (bf16) in one
        # ispa_accum_ops launch, as the session issues it after the chunk's attention calls
        layers = args.stats_layers or cfg.layers
        g = torch.Generator(device=device).manual_seed(0)
        a_ops = (torch.randn(layers, cfg.n_q, D, device=device, generator=g) * 0.05).to(torch.bfloat16)
        r_ops = (torch.randn(layers, cfg.n_q, D, device=device, generator=g) * 0.02).to(torch.bfloat16)
        stats = [ispa.Stats(D, device) for _ in range(layers)]
        fn = lambda: ispa.ispa_accum_ops(stats, a_ops, r_ops, cfg.n_q, ispa.ISPA_BF16)
        flops = layers * 4.0 * cfg.n_q * D * D
        what = f"batched statistics (G, C, H) of {layers} layers, n {cfg.n_q}, D {D}"
    else:
        Ws = [up(synth.w_out(cfg, l)) for l in range(cfg.layers)]
        sess.set_weights(Ws)
        # statistics of a representative warmup: random SPD-ish Grams from seeded operands
        g = torch.Generator(device="cpu").manual_seed(0)
        for st in sess.stats:
            a = (torch.randn(3 * cfg.n_q, D, generator=g) * 0.05).to(device)
            r = (torch.randn(3 * cfg.n_q, D, generator=g) * 0.05).to(device)
            st.G.copy_(a.T @ a)
            st.C.copy_(a.T @ r)
            st.H.copy_(r.T @ r)
        fn = lambda: sess.transition()
        flops = cfg.layers * (D ** 3 / 3 + 2 * D ** 3 + 2 * D ** 3 + 6 * D ** 3)
        what = f"absorb solve + error for {cfg.layers} layers, D {D}"
    for _ in range(max(3, args.warmup)):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    burst, sustained, hbm, kind = peaks()
    dt = statistics.median(times)
    tf = flops / dt / 1e12
    extra = {}

    def median_ms(f, steps):
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    if args.mode == "local" and not args.w8a8:
        # the L-layer step's two kernels apart (local attention; projection y = O W_new) and the
        # step replayed from a CUDA graph (no host launch work between the two kernels)
        att = lambda: sess.local_attention(0, q, k, v, o, lse)
        proj = lambda: ispa.ispa_project(o, sess.W_new[0], y)
        for f in (att, proj):
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream(device=device)
        s_cap.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(s_cap):
            fn()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s_cap):
                fn()
        torch.cuda.current_stream(device).wait_stream(s_cap)
        a_ms, p_ms = median_ms(att, args.steps), median_ms(proj, args.steps)
        g_ms = median_ms(g.replay, args.steps)
        extra = {"attention_only_ms": a_ms, "projection_only_ms": p_ms, "graph_step_ms": g_ms,
                 "step_minus_parts_ms": dt * 1e3 - a_ms - p_ms}
    if args.mode == "call" and args.i8:
        # the same call without the two quantisers (int8 Q/K already resident)
        t2 = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            attn_only()
            e1.record()
            torch.cuda.synchronize()
            t2.append(e0.elapsed_time(e1))
        extra = {"ms_without_quantisation": statistics.median(t2)}
    print(json.dumps({"mode": args.mode, "what": what, "ms": dt * 1e3, "ms_all": [x * 1e3 for x in times],
                      "tflops": tf, "frac_of_burst_peak": tf / burst, "peak_kind": kind,
                      "query_tokens_per_s": cfg.n_q / dt if args.mode in ("call", "local") else None} | extra),
          flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    cfg = synth.CONFIGS[args.config]
    if args.impl != "reference":
        from streaming_video_attention_b200 import ispa
        ispa.ispa_set_attn_kernel({"auto": ispa.ISPA_ATTN_AUTO, "single": ispa.ISPA_ATTN_SINGLE,
                                   "pair": ispa.ISPA_ATTN_PAIR,
                                   "two_group": ispa.ISPA_ATTN_TWO_GROUP}[args.attn_kernel])
    if args.mode != "episode":
        return unit_arm(args, cfg)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return reference_arm(args, cfg, rank)
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    try:
        return ispa_arm(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
