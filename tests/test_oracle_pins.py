"""Pins of the CPU oracle against facts fixed by the ISPA pages and by mathematics.

Every check here compares the oracle with something other than itself: hand-derived
worked examples (tests/golden), closed forms, brute-force loops written out in plain
Python, library routines that reach the same result by another algorithm (least squares
by QR/SVD instead of the normal equations; torch's bf16 cast), and invariants.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_round_matches_torch_cast():
    x = np.random.default_rng(0).standard_normal(200000)
    x *= np.exp(np.random.default_rng(1).uniform(-20, 20, x.shape))
    x = x.astype(np.float32).astype(np.float64)        # float32-exact, so torch rounds once
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(x), ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 sits halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0).
    # 1 + 3*2^-8 sits halfway between 1 + 2^-7 and 1 + 2^-6: goes to 1 + 2^-6.
    vals = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -40])
    want = np.array([1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7])
    assert np.array_equal(oracle.bf16_round(vals), want)


def test_synth_bf16_bits_match_torch():
    x = np.random.default_rng(2).standard_normal(100000).astype(np.float32)
    bits = synth.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


# ---------------------------------------------------------------- attention (step a1)
def test_attention_golden_two_keys():
    g = _golden("attention_two_keys.json")
    q, k, v = (np.array(g[n], dtype=np.float64) for n in ("q", "k", "v"))
    res = oracle.split_attention(q, k, v, tuple(g["sink"]), tuple(g["chunk"]), 1 / math.sqrt(2))
    for name in ("A_full", "lse_full", "A_loc", "lse_loc", "A_hist", "lse_hist"):
        np.testing.assert_allclose(res[name], np.array(g[name]), rtol=0, atol=1e-12, err_msg=name)


def _brute_attention(q, k, v, rows, scale):
    """Per-query softmax with Python loops and math.exp (no max subtraction needed at these sizes)."""
    n_q, h, d = q.shape
    A = np.zeros((n_q, h, d))
    lse = np.full((h, n_q), -np.inf)
    for i in range(n_q):
        for hh in range(h):
            if not rows:
                continue
            ws = []
            for j in rows:
                s = scale * sum(q[i, hh, c] * k[j, hh, c] for c in range(d))
                ws.append(math.exp(s))
            tot = sum(ws)
            for c in range(d):
                A[i, hh, c] = sum(w * v[j, hh, c] for w, j in zip(ws, rows)) / tot
            lse[hh, i] = math.log(tot)
    return A, lse


@pytest.mark.parametrize("sink,chunk", [((0, 2), (5, 7)), ((0, 1), (3, 7)), ((0, 7), (7, 7)), ((0, 0), (0, 0))])
def test_attention_brute_force(sink, chunk):
    q, k, v = _rand((3, 2, 4), 10), _rand((7, 2, 4), 11), _rand((7, 2, 4), 12)
    scale = 0.5
    res = oracle.split_attention(q, k, v, sink, chunk, scale)
    local = sorted(set(range(*sink)) | set(range(*chunk)))
    hist = [j for j in range(7) if j not in local]
    for name, rows in (("full", list(range(7))), ("loc", local), ("hist", hist)):
        A, lse = _brute_attention(q, k, v, rows, scale)
        np.testing.assert_allclose(res["A_" + name], A, rtol=1e-12, atol=1e-13, err_msg=name)
        np.testing.assert_allclose(res["lse_" + name], lse, rtol=1e-12, atol=1e-13, err_msg=name)


def test_lse_merge_equals_full_softmax():
    q, k, v = _rand((40, 3, 16), 20), _rand((300, 3, 16), 21), _rand((300, 3, 16), 22)
    res = oracle.split_attention(q, k, v, (0, 50), (220, 300), 0.25)
    A, lse = oracle.lse_merge(res["A_loc"], res["lse_loc"], res["A_hist"], res["lse_hist"])
    np.testing.assert_allclose(A, res["A_full"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, res["lse_full"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(res["lse_full"], np.logaddexp(res["lse_loc"], res["lse_hist"]), rtol=1e-13)


def test_attention_closed_forms():
    # zero keys: every score is 0, softmax is uniform, A = mean of the masked V rows, lse = ln(n)
    q, v = _rand((5, 2, 8), 30), _rand((9, 2, 8), 31)
    k = np.zeros((9, 2, 8))
    res = oracle.split_attention(q, k, v, (0, 2), (6, 9), 0.3)
    np.testing.assert_allclose(res["A_full"], np.broadcast_to(v.mean(0), (5, 2, 8)), atol=1e-13)
    np.testing.assert_allclose(res["A_loc"], np.broadcast_to(v[[0, 1, 6, 7, 8]].mean(0), (5, 2, 8)), atol=1e-13)
    np.testing.assert_allclose(res["lse_hist"], np.full((2, 5), math.log(4)), atol=1e-13)
    # a single key row: A is that V row, lse = scale * q.k
    k1 = _rand((1, 2, 8), 32)
    v1 = _rand((1, 2, 8), 33)
    A, lse = oracle.local_attention(q, k1, v1, 0.3)
    np.testing.assert_allclose(A, np.broadcast_to(v1[0], (5, 2, 8)), atol=1e-13)
    np.testing.assert_allclose(lse, 0.3 * np.einsum("ihd,hd->hi", q, k1[0]), atol=1e-12)


def test_empty_history_partition():
    q, k, v = _rand((6, 2, 8), 40), _rand((10, 2, 8), 41), _rand((10, 2, 8), 42)
    res = oracle.split_attention(q, k, v, (0, 4), (4, 10), 0.35)
    assert np.array_equal(res["A_full"], res["A_loc"])
    assert np.all(np.isneginf(res["lse_hist"])) and np.all(res["A_hist"] == 0)


def test_local_attention_gather_equals_mask():
    q, k, v = _rand((7, 2, 8), 50), _rand((30, 2, 8), 51), _rand((30, 2, 8), 52)
    res = oracle.split_attention(q, k, v, (0, 5), (22, 30), 0.35)
    rows = list(range(5)) + list(range(22, 30))
    A, lse = oracle.local_attention(q, k[rows], v[rows], 0.35)
    np.testing.assert_allclose(A, res["A_loc"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, res["lse_loc"], rtol=1e-13)


# ---------------------------------------------------------------- statistics (step a2)
def test_stats_brute_force_and_invariants():
    n, h, d = 9, 2, 3
    D = h * d
    A_loc = _rand((n, h, d), 60)
    A_full = A_loc + 0.3 * _rand((n, h, d), 61)
    st = oracle.stats_init(D)
    oracle.stats_update(st, A_loc, A_full, "fp32")
    a = A_loc.reshape(n, D)
    r = A_full.reshape(n, D) - a
    G = np.zeros((D, D)); C = np.zeros((D, D)); H = np.zeros((D, D))
    for i in range(n):
        for p in range(D):
            for q_ in range(D):
                G[p, q_] += a[i, p] * a[i, q_]
                C[p, q_] += a[i, p] * r[i, q_]
                H[p, q_] += r[i, p] * r[i, q_]
    np.testing.assert_allclose(st["G"], G, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st["C"], C, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st["H"], H, rtol=1e-13, atol=1e-14)
    assert st["rows"] == n
    for M in (st["G"], st["H"]):
        assert np.allclose(M, M.T)
        assert np.linalg.eigvalsh(M).min() > -1e-12


def test_stats_chunkwise_equals_one_shot():
    A_loc = _rand((50, 2, 4), 70)
    A_full = A_loc + _rand((50, 2, 4), 71)
    one = oracle.stats_init(8)
    oracle.stats_update(one, A_loc, A_full, "bf16")
    parts = oracle.stats_init(8)
    for s in (slice(0, 13), slice(13, 14), slice(14, 50)):
        oracle.stats_update(parts, A_loc[s], A_full[s], "bf16")
    for name in ("G", "C", "H"):
        np.testing.assert_allclose(parts[name], one[name], rtol=1e-12, atol=1e-13)
    assert parts["rows"] == one["rows"] == 50


def test_stats_bf16_operands_are_rounded():
    # bf16-grid inputs keep R = A_full - A_loc exact in float32, so torch's float32 -> bf16
    # cast gives the correctly rounded operand to compare with.
    bf = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    A_loc = bf(_rand((20, 1, 6), 72))
    A_full = bf(A_loc + _rand((20, 1, 6), 73))
    st = oracle.stats_init(6)
    oracle.stats_update(st, A_loc, A_full, "bf16")
    a = A_loc.reshape(20, 6)
    r = bf((A_full - A_loc).reshape(20, 6))
    assert not np.array_equal(r, (A_full - A_loc).reshape(20, 6))   # rounding did something
    np.testing.assert_allclose(st["G"], a.T @ a, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st["C"], a.T @ r, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st["H"], r.T @ r, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- absorb solve (step a3)
def test_ridge_golden_scalar():
    g = _golden("ridge_scalar.json")
    G, C, H, W = (np.array(g[n]) for n in ("G", "C", "H", "W"))
    dW = oracle.absorb_solve(G, C, W, g["lambda"])
    np.testing.assert_allclose(dW, np.array(g["dW"]), rtol=1e-15)
    e = oracle.reconstruction_error(G, C, H, W, dW)
    assert abs(e["E2"] - g["E2"]) < 1e-12 and abs(e["T2"] - g["T2"]) < 1e-12
    assert abs(e["eps"] - g["eps"]) < 1e-15


def test_empty_history_gives_zero_update_and_error():
    q, k, v = _rand((12, 2, 4), 80), _rand((16, 2, 4), 81), _rand((16, 2, 4), 82)
    res = oracle.split_attention(q, k, v, (0, 4), (4, 16), 0.5)   # local covers all rows
    st = oracle.stats_init(8)
    oracle.stats_update(st, res["A_loc"], res["A_full"], "fp32")
    W = _rand((8, 8), 83, 1 / math.sqrt(8))
    dW = oracle.absorb_solve(st["G"], st["C"], W, 1e-2)
    assert np.all(dW == 0)
    e = oracle.reconstruction_error(st["G"], st["C"], st["H"], W, dW)
    assert e["eps"] == 0.0 and e["E2"] == 0.0


def test_planted_linear_residual_recovered_as_lambda_vanishes():
    n, D = 64, 8
    a = _rand((n, D), 90)
    P = _rand((D, D), 91)
    W = _rand((D, D), 92)
    A_loc = a.reshape(n, 2, 4)
    A_full = (a + a @ P).reshape(n, 2, 4)                         # R = A_loc P exactly
    st = oracle.stats_init(D)
    oracle.stats_update(st, A_loc, A_full, "fp32")
    dW = oracle.absorb_solve(st["G"], st["C"], W, 1e-10)
    np.testing.assert_allclose(dW, P @ W, rtol=1e-7, atol=1e-9)
    e = oracle.reconstruction_error(st["G"], st["C"], st["H"], W, dW)
    assert abs(e["eps"]) < 1e-9


def test_solve_agrees_with_least_squares():
    n, D, lam = 40, 6, 0.3
    a = _rand((n, D), 100)
    r = _rand((n, D), 101)
    W = _rand((D, D), 102)
    st = oracle.stats_init(D)
    oracle.stats_update(st, a.reshape(n, 2, 3), (a + r).reshape(n, 2, 3), "fp32")
    dW = oracle.absorb_solve(st["G"], st["C"], W, lam)
    Aaug = np.vstack([a, math.sqrt(lam) * np.eye(D)])
    Baug = np.vstack([r @ W, np.zeros((D, D))])
    ref = np.linalg.lstsq(Aaug, Baug, rcond=None)[0]
    np.testing.assert_allclose(dW, ref, rtol=1e-10, atol=1e-12)
    res = (st["G"] + lam * np.eye(D)) @ dW - st["C"] @ W
    assert np.linalg.norm(res) / np.linalg.norm(st["C"] @ W) < 1e-12


def test_error_traces_match_direct_norms():
    n, D, lam = 50, 6, 0.05
    a = _rand((n, D), 110)
    r = 0.5 * a @ _rand((D, D), 111) + 0.2 * _rand((n, D), 112)
    W = _rand((D, D), 113)
    st = oracle.stats_init(D)
    oracle.stats_update(st, a.reshape(n, 3, 2), (a + r).reshape(n, 3, 2), "fp32")
    for dW in (oracle.absorb_solve(st["G"], st["C"], W, lam), _rand((D, D), 114)):
        e = oracle.reconstruction_error(st["G"], st["C"], st["H"], W, dW)
        E2 = np.sum((a @ (W + dW) - (a + r) @ W) ** 2)
        T2 = np.sum(((a + r) @ W) ** 2)
        assert abs(e["E2"] - E2) < 1e-9 * T2
        assert abs(e["T2"] - T2) < 1e-10 * T2
        assert abs(e["eps"] - E2 / T2) < 1e-9


def test_project_golden_two_heads():
    """y = A W for A [n, heads, head_dim] (column h*head_dim + j) and W stored [D_in, D_out],
    against a hand-computed case whose W is neither square nor symmetric."""
    g = _golden("project_two_heads.json")
    A, W = np.array(g["A"]), np.array(g["W"])
    np.testing.assert_array_equal(oracle.project(A, W), np.array(g["y"]))


def test_project_residual_is_the_error_numerator():
    """||project(A_loc, W + dW) - project(A_full, W)||^2 summed over the warmup equals E^2 of
    the trace form (itself pinned to direct norms above), for attention outputs of a real
    split call, several heads and a non-symmetric W: a transposed W or a dropped dW in
    project would change the left side only."""
    n_q, n_kv, h, d = 12, 40, 3, 4
    D = h * d
    rng = np.random.default_rng(130)
    W = rng.standard_normal((D, D)) / math.sqrt(D)
    assert np.linalg.norm(W - W.T) > 0.5 * np.linalg.norm(W)
    st = oracle.stats_init(D)
    chunks = []
    for t in range(3):
        q, k, v = (rng.standard_normal(s) for s in ((n_q, h, d), (n_kv, h, d), (n_kv, h, d)))
        res = oracle.split_attention(q, k, v, (0, 6), (28, 40), 1 / math.sqrt(d))
        oracle.stats_update(st, res["A_loc"], res["A_full"], "fp32")
        chunks.append(res)
    for dW in (oracle.absorb_solve(st["G"], st["C"], W, 0.05), rng.standard_normal((D, D)) / D):
        e = oracle.reconstruction_error(st["G"], st["C"], st["H"], W, dW)
        E2 = sum(np.sum((oracle.project(c["A_loc"], W + dW) - oracle.project(c["A_full"], W)) ** 2) for c in chunks)
        T2 = sum(np.sum(oracle.project(c["A_full"], W) ** 2) for c in chunks)
        assert abs(E2 - e["E2"]) < 1e-10 * T2
        assert abs(T2 - e["T2"]) < 1e-10 * T2


def test_solution_minimises_the_ridge_objective():
    n, D, lam = 30, 5, 0.2
    a = _rand((n, D), 120)
    r = _rand((n, D), 121)
    W = _rand((D, D), 122)
    st = oracle.stats_init(D)
    oracle.stats_update(st, a.reshape(n, 1, 5), (a + r).reshape(n, 1, 5), "fp32")
    dW = oracle.absorb_solve(st["G"], st["C"], W, lam)

    def obj(X):
        return np.sum((a @ (W + X) - (a + r) @ W) ** 2) + lam * np.sum(X ** 2)

    base = obj(dW)
    rng = np.random.default_rng(123)
    for _ in range(20):
        assert obj(dW + 1e-3 * rng.standard_normal((D, D))) > base


# ---------------------------------------------------------------- selection (step a5)
def test_selection_golden():
    g = _golden("selection_examples.json")
    for case in g["cases"]:
        eps = [float("nan") if e == "nan" else e for e in case["eps"]]
        idx, flags = oracle.select_layers(eps, case["K"])
        assert idx == case["idx"], case
        assert flags == case["is_local"], case


# ---------------------------------------------------------------- whole episodes
def _small(structured=False, **kw):
    base = dict(name="small", layers=4, heads=2, head_dim=16, tpf=24, chunk_frames=2, h_max=6,
                warmup_chunks=3, lam=1e-2, K=2, dtype="fp32", structured=structured, planted_rank=4)
    base.update(kw)
    return synth.IspaConfig(**base)


def test_episode_structured_layers_are_absorbable():
    """The planted (rank-4 template + small drift) layers must reach a far lower error
    than the i.i.d. layers, and be the ones selected."""
    cfg = _small(structured=True)
    out = oracle.run_episode(cfg, n_chunks=cfg.warmup_chunks)
    eps = out["transitions"][0]["eps"]
    planted = [eps[l] for l in range(cfg.layers) if cfg.planted(l)]
    iid = [eps[l] for l in range(cfg.layers) if not cfg.planted(l)]
    assert max(planted) < 0.25 * min(iid), eps
    assert sorted(out["transitions"][0]["idx"]) == [0, 2]


def test_episode_rewarmup_after_cut():
    cfg = _small(structured=True, cut_chunk=5, total_chunks=8)
    out = oracle.run_episode(cfg)
    assert [tr["chunk"] for tr in out["transitions"]] == [2, 7]
    for tr in out["transitions"]:
        assert all(s["rows"] == cfg.warmup_chunks * cfg.n_q for s in tr["stats"])


def test_episode_warmup_schedule_rows():
    cfg = _small()
    out = oracle.run_episode(cfg, n_chunks=cfg.warmup_chunks, keep_outputs=True)
    tr = out["transitions"][0]
    assert tr["chunk"] == cfg.warmup_chunks - 1 and len(tr["idx"]) == cfg.K
    assert len(out["outputs"]) == cfg.warmup_chunks


# ------------------------------------------------------------------ re-warmup trigger (step 7)
def test_live_error_is_the_relative_residual_of_one_chunk():
    """eps_live from one chunk's statistics equals ||A_loc (W + dW) - A_full W||^2 /
    ||A_full W||^2 computed directly on that chunk (fp32 mode: no operand rounding)."""
    rng = np.random.default_rng(11)
    n, D = 60, 16
    a_loc = rng.standard_normal((n, 1, D))
    a_full = a_loc + 0.3 * rng.standard_normal((n, 1, D))
    W = rng.standard_normal((D, D)) / 4
    dW = 0.1 * rng.standard_normal((D, D))
    got = oracle.live_error(a_loc, a_full, "fp32", W, dW)
    A, F = a_loc.reshape(n, D), a_full.reshape(n, D)
    want = np.sum((A @ (W + dW) - F @ W) ** 2) / np.sum((F @ W) ** 2)
    assert got == pytest.approx(want, rel=1e-12)
    # no history at all: the residual is zero and dW = 0 reconstructs exactly
    assert oracle.live_error(a_loc, a_loc, "fp32", W, np.zeros((D, D))) == 0.0


def test_rewarm_trigger_rule_cases():
    hist = [{1: 0.01, 2: 2.0}, {1: 0.012, 2: 2.4}]
    assert oracle.rewarm_trigger(hist, {1: 0.3, 2: 2.2}) == [1]          # 30x its minimum, +0.29
    assert oracle.rewarm_trigger(hist, {1: 0.011, 2: 7.0}) == []         # 3.5x its minimum: not enough
    assert oracle.rewarm_trigger(hist, {1: 0.011, 2: 8.5}) == [2]        # 4.25x
    assert oracle.rewarm_trigger(hist, {1: 0.029, 2: 2.0}) == []         # 2.9x, below the ratio
    assert oracle.rewarm_trigger([{3: 1e-4}], {3: 9e-3}) == []           # 90x but a rise of 0.009 only
    assert oracle.rewarm_trigger([], {1: 5.0}) == []                     # no reference yet
    assert oracle.rewarm_trigger(hist, {4: 5.0}) == []                   # a layer never seen before


def test_live_error_fires_at_the_scene_cut_only():
    """Structured workload, no scheduled re-warmup: the planted layer that stayed an F-layer
    keeps a small live error until the cut, where it jumps; the i.i.d. layers stay put."""
    cfg = _small(structured=True, cut_chunk=5, total_chunks=8, K=1)
    out = oracle.run_episode(cfg, K=1, rewarm_at=None, monitor=True)
    assert [t for t, _ in out["live"]] == [3, 4, 5, 6, 7]
    fired, prev = {}, []
    for t, live in out["live"]:
        assert set(live) == {l for l in range(cfg.layers) if l not in out["transitions"][0]["idx"]}
        fired[t] = oracle.rewarm_trigger(prev, live)
        prev.append(live)
    planted_f = [l for l in range(cfg.layers) if cfg.planted(l) and l not in out["transitions"][0]["idx"]]
    assert planted_f and fired[3] == [] and fired[4] == [] and fired[5] == planted_f


# ------------------------------------------------------------------ W8A8 projection
def test_int8_quantization_hand_cases():
    q, s = oracle.quantize_int8(np.array([[1.0, -2.0, 0.5], [0.0, 0.0, 0.0]]), axis=1)
    assert q.tolist() == [[64, -127, 32], [0, 0, 0]]            # 63.5 rounds to even (64); 31.75 -> 32
    assert s[0] == np.float32(2.0) / np.float32(127.0) and s[1] == 0.0
    qc, sc = oracle.quantize_int8(np.array([[1.0, 4.0], [-3.0, 2.0]]), axis=0)
    assert qc.tolist() == [[42, 127], [-127, 64]]               # columns: amax 3 and 4; 42.33 -> 42, 63.5 -> 64
    assert sc.tolist() == [np.float32(3.0) / np.float32(127.0), np.float32(4.0) / np.float32(127.0)]


def test_int8_quantization_error_bound():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((40, 96)) * np.exp(rng.normal(0, 2, (40, 1)))).astype(np.float32)
    q, s = oracle.quantize_int8(x, axis=1)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-5) + 1e-30)
    assert np.all(np.abs(q).max(axis=1) == 127)                 # the largest element of a row maps to 127


def test_w8a8_scale_invariances_and_error_bound():
    """Per-row activation scales and per-column weight scales: doubling a row of A or a
    column of W doubles exactly that row or column of y; y is within the quantisation
    bound of the float64 product."""
    rng = np.random.default_rng(5)
    n, K, N = 24, 64, 40
    A = synth_bf16(rng.standard_normal((n, K)))
    W = synth_bf16(rng.standard_normal((K, N)) / 8)
    y = oracle.project_w8a8(A, W)
    A2 = A.copy(); A2[3] *= 2
    W2 = W.copy(); W2[:, 7] *= 2
    y2 = oracle.project_w8a8(A2, W)
    y3 = oracle.project_w8a8(A, W2)
    assert np.array_equal(y2[3], 2 * y[3]) and np.array_equal(np.delete(y2, 3, 0), np.delete(y, 3, 0))
    assert np.array_equal(y3[:, 7], 2 * y[:, 7]) and np.array_equal(np.delete(y3, 7, 1), np.delete(y, 7, 1))
    exact = A.astype(np.float64) @ W.astype(np.float64)
    sa = np.abs(A).max(axis=1, keepdims=True) / 127
    sw = np.abs(W).max(axis=0, keepdims=True) / 127
    # |A W - Aq Wq| <= sum_k (|a_k| e_w + |w_k| e_a + e_a e_w), e = half a step; plus bf16 rounding
    bound = (np.abs(A) @ np.ones((K, N))) * 0.5 * sw + 0.5 * sa * (np.ones((n, K)) @ np.abs(W)) + K * 0.25 * sa * sw
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-6) + np.abs(exact) * 2.0 ** -8 + 1e-12)


def synth_bf16(x):
    return oracle.bf16_round(np.asarray(x, np.float64)).astype(np.float32)


# ------------------------------------------------------------------ 8-bit (int8) split attention
def test_kv_blocks_cover_the_rows_once_and_respect_partitions():
    for n_kv, sink, chunk in [(1000, (0, 64), (900, 1000)), (300, (0, 0), (200, 300)), (640, (0, 130), (130, 640)),
                              (5, (0, 1), (1, 3)), (37440, (0, 1560), (32760, 37440))]:
        blocks = oracle.kv_blocks(n_kv, sink, chunk)
        rows = np.concatenate([np.arange(b, e) for b, e in blocks])
        assert np.array_equal(rows, np.arange(n_kv))                     # in order, each row once
        assert all(0 < e - b <= 128 for b, e in blocks)
        _, local, _ = oracle.partition_masks(n_kv, sink, chunk)
        for b, e in blocks:
            assert local[b:e].all() or not local[b:e].any()               # one partition per block
            in_sink = (sink[0] <= b < sink[1]) == (sink[0] <= e - 1 < sink[1])
            assert in_sink                                                # never across the sink edge
    assert oracle.kv_blocks(300, (0, 0), (200, 300)) == [(0, 128), (128, 200), (200, 300)]
    assert oracle.kv_blocks(1000, (0, 64), (900, 1000))[:3] == [(0, 64), (64, 192), (192, 320)]


def test_i8_quantizers_hand_cases_and_bounds():
    q = np.zeros((2, 1, 4), np.float32)
    q[0, 0] = [1.0, -2.0, 0.5, 0.25]
    q8, sq = oracle.quantize_i8_q(q)
    assert q8[0, 0].tolist() == [64, -127, 32, 16] and q8[1, 0].tolist() == [0, 0, 0, 0]   # 63.5 -> 64 (even)
    assert sq.shape == (2, 1) and sq[0, 0] == np.float32(2.0) / np.float32(127.0) and sq[1, 0] == 0.0
    rng = np.random.default_rng(9)
    k = synth_bf16(rng.standard_normal((300, 3, 64)) * np.exp(rng.normal(0, 1, (300, 1, 1))))
    blocks = oracle.kv_blocks(300, (0, 40), (200, 300))
    k8, sk = oracle.quantize_i8_k(k, blocks)
    assert sk.shape == (3, len(blocks))
    for i, (b, e) in enumerate(blocks):
        amax = np.abs(k[b:e]).max(axis=(0, 2))
        assert np.all(sk[:, i] == (amax / np.float32(127.0)).astype(np.float32))
        assert np.all(np.abs(k8[b:e]).max(axis=(0, 2)) == 127)        # the largest element maps to 127
        err = np.abs(k8[b:e].astype(np.float64) * sk[:, i][None, :, None] - k[b:e])
        assert np.all(err <= 0.5 * sk[:, i][None, :, None] * (1 + 1e-5))


def test_i8_attention_reduces_to_the_exact_one_on_the_grid():
    """Integer inputs whose per-row (Q) and per-block (K) maxima are 127 quantise to themselves
    with scale 1: the 8-bit split attention then equals the plain one exactly."""
    rng = np.random.default_rng(10)
    n_q, n_kv, h, d = 9, 300, 2, 32
    q = rng.integers(-126, 127, (n_q, h, d)).astype(np.float64)
    k = rng.integers(-126, 127, (n_kv, h, d)).astype(np.float64)
    q[:, :, 0] = 127.0
    for b, e in oracle.kv_blocks(n_kv, (0, 5), (200, 300)):
        k[b, :, 0] = -127.0
    v = synth_bf16(rng.standard_normal((n_kv, h, d)))
    scale = 1.0 / (127.0 * 127.0 * d)
    got = oracle.split_attention_i8(q, k, v, (0, 5), (200, 300), scale)
    want = oracle.split_attention(q, k, v, (0, 5), (200, 300), scale)
    assert np.all(got["q_scale"] == 1.0) and np.all(got["k_scale"] == 1.0)
    for key in ("A_full", "A_loc", "A_hist", "lse_full", "lse_loc", "lse_hist"):
        assert np.array_equal(got[key], want[key]), key


def test_i8_attention_error_against_unquantised():
    """On N(0,1) inputs with the 1/sqrt(d) scale the int8 scores move the outputs by about
    1 %: the bound here is the 2e-2 used for bf16 attention."""
    rng = np.random.default_rng(11)
    n_q, n_kv, h, d = 64, 300, 2, 128
    q, k, v = (synth_bf16(rng.standard_normal((n, h, d))) for n in (n_q, n_kv, n_kv))
    got = oracle.split_attention_i8(q, k, v, (0, 40), (200, 300), 1 / math.sqrt(d))
    want = oracle.split_attention(q, k, v, (0, 40), (200, 300), 1 / math.sqrt(d))
    for key in ("A_full", "A_loc", "A_hist"):
        rel = np.linalg.norm(got[key] - want[key]) / np.linalg.norm(want[key])
        assert rel < 2e-2, (key, rel)
