"""Parity of every workload configuration against the CPU oracle, through the product API
(IspaSession over the C ABI):

* tiny fp32 (1 layer, 2 x 64, 4 warmup chunks): the whole streaming run, element by element.
* structured bf16, scaled down (4 layers, cut + re-warmup, K sweep): the whole run.
* 1.3B shape: one planted and one i.i.d. layer through the whole warmup at full size (oracle on
  every row; dW through the whole bf16 chain).
* long history (n_kv 191,880): one layer, sampled query rows; then the L-layer call.
* 14B shape (40 x 128, D = 5120): one layer, sampled rows; the absorb solve at D = 5120.

Tolerances: fp32 1e-5 (attention), 1e-3 (dW, relative Frobenius), 1e-4 relative (eps);
bf16 attention 2e-2 relative Frobenius; eps through the bf16 chain 5e-2 relative (A_loc and
R carry about 4e-3 relative rounding noise into the statistics); selections bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from streaming_video_attention_b200 import ispa
from streaming_video_attention_b200.session import IspaSession
from tests.helpers import rel_fro, to_device, to_numpy, torch_dtype

pytestmark = pytest.mark.gpu


def gpu_episode(cfg, K=None, n_chunks=None, keep_layers=None, rewarm="cut", monitor=False):
    """Drive IspaSession through a streaming run laid out by `synth` (the caller owns the KV
    cache: it builds each layer's cache from the frames that layer still holds).

    rewarm: "cut" re-enters the warmup at the workload's scene cut, None never, "auto" at the
    chunk after the session's trigger fired (monitoring every F-layer after a transition).
    monitor: record the live errors (implied by "auto")."""
    K = cfg.K if K is None else K
    monitor = monitor or rewarm == "auto"
    live, fired = [], []
    pending_rewarm = False
    n_chunks = cfg.n_chunks if n_chunks is None else n_chunks
    L = cfg.layers
    td = torch_dtype(cfg.dtype)
    sess = IspaSession(L, cfg.heads, cfg.head_dim, cfg.lam, K, cfg.dtype)
    sess.set_weights([to_device(synth.w_out(cfg, l), cfg.dtype) for l in range(L)])
    sess.rewarm()
    hist_from = [None] * L
    warm_start = 0
    transitions, outputs = [], []
    for t in range(n_chunks):
        scheduled = rewarm == "cut" and cfg.cut_chunk is not None and t == cfg.cut_chunk
        if scheduled or pending_rewarm:
            for l in range(L):
                if sess.is_local[l]:
                    hist_from[l] = cfg.chunk_start_frame(t)
            sess.rewarm()
            warm_start = t
            pending_rewarm = False
        in_warmup = warm_start <= t < warm_start + cfg.warmup_chunks
        watch = monitor and sess.transitions > 0 and not in_warmup
        chunk_out = []
        for l in range(L):
            q = to_device(synth.chunk_q(cfg, l, t), cfg.dtype)
            o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=td, device="cuda")
            lse = torch.empty((cfg.heads, cfg.n_q), device="cuda")
            if sess.is_local[l]:
                s0 = cfg.chunk_start_frame(t)
                frames = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))
                k = to_device(synth.kv_tensor(cfg, l, frames, "k"), cfg.dtype)
                v = to_device(synth.kv_tensor(cfg, l, frames, "v"), cfg.dtype)
                y = torch.empty((cfg.n_q, cfg.D), dtype=td, device="cuda")
                sess.local_attention(l, q, k, v, o, lse, y)
                chunk_out.append(dict(O=o, y=y, local=True))
            else:
                frames = synth.cache_frames(cfg, t, hist_from[l])
                lay = synth.chunk_layout(cfg, frames, t)
                k = to_device(synth.kv_tensor(cfg, l, frames, "k"), cfg.dtype)
                v = to_device(synth.kv_tensor(cfg, l, frames, "v"), cfg.dtype)
                sess.full_attention(l, q, k, v, (lay["sink_begin"], lay["sink_end"]),
                                    (lay["chunk_begin"], lay["chunk_end"]), o, lse, collect=in_warmup,
                                    monitor=watch)
                chunk_out.append(dict(O=o, y=None, local=False))
        outputs.append(chunk_out)
        if watch:
            live.append((t, sess.live_errors()))
            f = sess.rewarm_layers()
            fired.append((t, f))
            if f and rewarm == "auto":
                pending_rewarm = True
        if in_warmup and t == warm_start + cfg.warmup_chunks - 1:
            idx = sess.transition()
            transitions.append(dict(chunk=t, eps=list(sess.eps_host), idx=idx, is_local=list(sess.is_local),
                                    dW=sess.dW.clone(), rows=[int(s.rows.item()) for s in sess.stats]))
    torch.cuda.synchronize()
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    return dict(transitions=transitions, outputs=outputs, live=live, fired=fired)


def _compare_runs(cfg, got, want, attn_tol, eps_tol, dW_tol=None, y_tol=None):
    assert len(got["transitions"]) == len(want["transitions"])
    for tg, tw in zip(got["transitions"], want["transitions"]):
        assert tg["chunk"] == tw["chunk"]
        assert tg["idx"] == tw["idx"], (tg["eps"], tw["eps"])
        assert tg["is_local"] == list(tw["is_local"])
        assert tg["rows"] == [s["rows"] for s in tw["stats"]]
        for l in range(cfg.layers):
            e_g, e_w = tg["eps"][l], tw["eps"][l]
            assert abs(e_g - e_w) <= eps_tol * abs(e_w) + 1e-7, (l, e_g, e_w)
            if dW_tol is not None:
                assert rel_fro(to_numpy(tg["dW"][l]), tw["dW"][l]) < dW_tol, l
    for t, (cg, cw) in enumerate(zip(got["outputs"], want["outputs"])):
        for l in range(cfg.layers):
            assert cg[l]["local"] == cw[l]["local"], (t, l)
            assert rel_fro(to_numpy(cg[l]["O"]), cw[l]["O"]) < attn_tol, (t, l)
            if cg[l]["local"] and y_tol is not None:
                assert rel_fro(to_numpy(cg[l]["y"]), cw[l]["y"]) < y_tol, (t, l)


def test_tiny_fp32_full_run():
    cfg = synth.CONFIGS["tiny_fp32"]
    got = gpu_episode(cfg)
    want = oracle.run_episode(cfg, keep_outputs=True)
    _compare_runs(cfg, got, want, attn_tol=1e-5, eps_tol=1e-4, dW_tol=1e-3, y_tol=1e-4)


def _small_structured(**kw):
    base = dict(name="structured_small", layers=4, heads=2, head_dim=128, tpf=64, chunk_frames=2, h_max=6,
                warmup_chunks=3, lam=1e-2, K=2, dtype="bf16", structured=True, cut_chunk=5, total_chunks=8)
    base.update(kw)
    return synth.IspaConfig(**base)


@pytest.mark.parametrize("K", [1, 2])
def test_structured_run_with_scene_cut_and_rewarmup(K):
    """Planted (even) layers absorb, i.i.d. layers do not; the cut at chunk 5 re-enters the
    warmup and selects again (25% and 50% of the layers)."""
    cfg = _small_structured()
    got = gpu_episode(cfg, K=K)
    want = oracle.run_episode(cfg, K=K, keep_outputs=True)
    assert [t["chunk"] for t in got["transitions"]] == [2, 7]
    # before the cut every planted layer absorbs; after it, planted F-layers still hold pre-cut
    # frames in their window (reading of the re-warmup), so only the first transition separates
    for tr in want["transitions"][:1]:
        planted = [tr["eps"][l] for l in range(cfg.layers) if cfg.planted(l)]
        iid = [tr["eps"][l] for l in range(cfg.layers) if not cfg.planted(l)]
        assert max(planted) < 0.25 * min(iid)
    _compare_runs(cfg, got, want, attn_tol=2e-2, eps_tol=5e-2, y_tol=5e-2)


def test_structured_live_error_detects_the_scene_cut():
    """Re-warmup trigger, no scheduled re-warmup: the live errors of the F-layers against the
    oracle's (eps tolerance of the bf16 chain), and the trigger fires at the cut chunk, for the
    planted F-layer only, as the oracle's statement of the rule does on the oracle's errors."""
    cfg = _small_structured(K=1)
    got = gpu_episode(cfg, K=1, rewarm=None, monitor=True)
    want = oracle.run_episode(cfg, K=1, rewarm_at=None, monitor=True)
    assert [t for t, _ in got["live"]] == [t for t, _ in want["live"]] == [3, 4, 5, 6, 7]
    prev = []
    for (t, lg), (_, lw), (_, fg) in zip(got["live"], want["live"], got["fired"]):
        assert sorted(lg) == sorted(lw)
        for l in lw:
            assert abs(lg[l] - lw[l]) <= 5e-2 * abs(lw[l]) + 1e-4, (t, l, lg[l], lw[l])
        assert fg == oracle.rewarm_trigger(prev, lw), (t, fg)
        prev.append(lw)
    first = next(t for t, f in got["fired"] if f)
    assert first == cfg.cut_chunk
    assert dict(got["fired"])[first] == [l for l in range(cfg.layers) if cfg.planted(l) and l not in got["transitions"][0]["idx"]]


def test_structured_run_with_automatic_rewarmup():
    """The trigger drives the re-warmup: it fires at the cut, the warmup restarts at the next
    chunk, and the whole run matches the oracle scheduled to re-warm there."""
    cfg = _small_structured(K=1, total_chunks=10)
    got = gpu_episode(cfg, K=1, rewarm="auto")
    want = oracle.run_episode(cfg, K=1, rewarm_at=cfg.cut_chunk + 1, keep_outputs=True)
    assert [t["chunk"] for t in got["transitions"]] == [2, cfg.cut_chunk + 3]
    _compare_runs(cfg, got, want, attn_tol=2e-2, eps_tol=5e-2, y_tol=5e-2)


@pytest.mark.parametrize("kind", ["planted", "iid"])
def test_1p3b_layer_full_warmup_chain(kind):
    """The 1.3B attention shape (12 x 128, n_q 4680, H = 15, 18, 21) through the whole warmup of
    one layer -- planted (rank-16 template + drift) or i.i.d. N(0, 1) -- the oracle on every row:
    attention outputs, eps, and dW through the whole bf16 chain (attention -> bf16 operands ->
    statistics -> solve) against the oracle's own float64 chain on the same inputs.

    dW bound, from an error model: the GPU's A_loc and R differ from the oracle's by the bf16
    rounding of P before the PV product (about 1.7e-3 relative RMS per element, independent across
    elements). Perturbing the oracle's own float64 attention outputs by noise of that size before
    the bf16 operand rounding moves its dW by 1.7e-3 relative Frobenius on the i.i.d. layer (G's
    eigenvalues 1.3 .. 1.7e3: the solve passes the noise through one for one) and by 5.3e-2 on the
    planted layer (G's eigenvalues 5e-3 .. 8.2e3 against lambda = 1e-2: the rank-16 template leaves
    weak directions in which the solve amplifies the noise about a hundredfold), while eps moves by
    5e-6 and 1.4e-3 relative. The 1e-3 that the solve meets on identical statistics
    (test_solve_absorb_matches_oracle) is therefore out of reach through any bf16 chain for the
    planted layer; the bounds are twice to three times the model's figures."""
    if kind == "planted":
        base = synth.CONFIGS["structured_bf16"]
        cfg = synth.IspaConfig(**{**base.__dict__, "layers": 1, "K": 1, "cut_chunk": None,
                                  "total_chunks": base.warmup_chunks, "name": "structured_1layer"})
        assert cfg.planted(0)
    else:
        base = synth.CONFIGS["1p3b_bf16"]
        cfg = synth.IspaConfig(**{**base.__dict__, "layers": 1, "K": 1, "total_chunks": base.warmup_chunks,
                                  "name": "1p3b_1layer"})
    got = gpu_episode(cfg, n_chunks=cfg.warmup_chunks)
    want = oracle.run_episode(cfg, n_chunks=cfg.warmup_chunks, keep_outputs=True)
    tg, tw = got["transitions"][0], want["transitions"][0]
    assert tg["rows"] == [3 * cfg.n_q]
    eps_err = abs(tg["eps"][0] - tw["eps"][0]) / tw["eps"][0]
    dW_err = rel_fro(to_numpy(tg["dW"][0]), tw["dW"][0])
    print(f"\n[{kind}] eps gpu {tg['eps'][0]:.6e} oracle {tw['eps'][0]:.6e} rel {eps_err:.3e}; "
          f"dW rel Frobenius {dW_err:.3e}")
    assert eps_err <= 5e-2, (tg["eps"], tw["eps"])
    assert dW_err < (1e-1 if kind == "planted" else 5e-3), dW_err
    for t in range(cfg.warmup_chunks):
        assert rel_fro(to_numpy(got["outputs"][t][0]["O"]), want["outputs"][t][0]["O"]) < 2e-2


def _layer_call(cfg, layer, t, rows):
    frames = synth.cache_frames(cfg, t)
    lay = synth.chunk_layout(cfg, frames, t)
    q = synth.chunk_q(cfg, layer, t)
    k = synth.kv_tensor(cfg, layer, frames, "k")
    v = synth.kv_tensor(cfg, layer, frames, "v")
    sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
    desc = ispa.make_desc(cfg.n_q, lay["n_kv"], cfg.heads, cfg.head_dim, sink, chunk, dtype=ispa.ISPA_BF16)
    st = ispa.Stats(cfg.D)
    ws = ispa.alloc_workspace(ispa.workspace_bytes(desc, 0, 0))
    o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    ol = torch.empty_like(o)
    lse = torch.empty((cfg.heads, cfg.n_q), device="cuda")
    ispa.ispa_attn_split(desc, to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), o, lse, ol,
                         stats=st, ws=ws)
    torch.cuda.synchronize()
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    want = oracle.split_attention(q[rows], k, v, sink, chunk, cfg.scale)
    assert rel_fro(to_numpy(o)[rows], want["A_full"]) < 2e-2
    assert rel_fro(to_numpy(ol)[rows], want["A_loc"]) < 2e-2
    assert np.max(np.abs(to_numpy(lse)[:, rows] - want["lse_full"])) < 2e-2
    G = to_numpy(st.G)
    a = to_numpy(ol).reshape(cfg.n_q, -1)
    assert abs(np.trace(G) - np.sum(a * a)) < 1e-4 * np.sum(a * a)
    assert int(st.rows.item()) == cfg.n_q
    return lay


def test_long_history_layer_sampled_rows():
    cfg = synth.CONFIGS["long_bf16"]
    rows = np.array([0, 1, 127, 128, 2000, 4095, 4600, 4679])
    lay = _layer_call(cfg, 2, cfg.warmup_chunks - 1, rows)
    assert lay["n_kv"] == 191880
    # the L-layer call after the switch: sink + chunk only, projection with a W_new
    t = cfg.warmup_chunks
    s0 = cfg.chunk_start_frame(t)
    frames = [0] + list(range(s0, s0 + cfg.chunk_frames))
    q = synth.chunk_q(cfg, 2, t)
    k = synth.kv_tensor(cfg, 2, frames, "k")
    v = synth.kv_tensor(cfg, 2, frames, "v")
    W = synth.w_out(cfg, 2)
    desc = ispa.make_desc(cfg.n_q, k.shape[0], cfg.heads, cfg.head_dim, dtype=ispa.ISPA_BF16)
    o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((cfg.n_q, cfg.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.heads, cfg.n_q), device="cuda")
    ispa.ispa_local_attn(desc, to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), o, lse,
                         to_device(W, "bf16"), y)
    torch.cuda.synchronize()
    A, _ = oracle.local_attention(q[rows], k, v, cfg.scale)
    assert rel_fro(to_numpy(o)[rows], A) < 2e-2
    assert rel_fro(to_numpy(y)[rows], oracle.project(A, W)) < 2e-2


def test_14b_layer_sampled_rows_and_solve():
    cfg = synth.CONFIGS["14b_bf16"]
    rows = np.array([0, 127, 128, 2500, 4679])
    _layer_call(cfg, 1, cfg.warmup_chunks - 1, rows)
    # the absorb solve at D = 5120 on statistics the oracle builds from seeded operands
    D, n = cfg.D, 6000
    a = synth.normal_tensor(91, (1,), (n, D), "bf16", std=0.05).astype(np.float64)
    r = synth.normal_tensor(91, (2,), (n, D), "bf16", std=0.05).astype(np.float64)
    ref = oracle.stats_init(D)
    oracle.stats_update(ref, a.reshape(n, cfg.heads, -1), (a + r).reshape(n, cfg.heads, -1), "bf16")
    st = ispa.Stats(D)
    for name in ("G", "C", "H"):
        getattr(st, name).copy_(torch.from_numpy(ref[name].astype(np.float32)))
    W = synth.w_out(cfg, 0)
    dW = torch.empty((1, D, D), device="cuda")
    eps = torch.empty(1, device="cuda")
    status = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = ispa.alloc_workspace(ispa.workspace_bytes(None, 1, D))
    ispa.ispa_solve_absorb([st], [to_device(W, "bf16")], ispa.ISPA_BF16, cfg.lam, dW, eps, None, None, status, ws)
    torch.cuda.synchronize()
    assert status.tolist() == [0]
    G32, C32, H32 = (ref[n_].astype(np.float32).astype(np.float64) for n_ in ("G", "C", "H"))
    dW_ref = oracle.absorb_solve(G32, C32, W, cfg.lam)
    assert rel_fro(to_numpy(dW[0]), dW_ref) < 1e-3
    e = oracle.reconstruction_error(G32, C32, H32, W, dW_ref)
    assert abs(float(eps[0]) - e["eps"]) <= 1e-3 * abs(e["eps"])
