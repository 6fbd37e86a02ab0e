"""Plain, slow CPU oracle of the ISPA warmup path, in float64 NumPy. TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this module; the
product path never imports it, and it imports nothing from the product package.

Source: "Towards Memory-Efficient Autoregressive Video Generation via Instance-Specific
Parametric Absorption" (ISPA), paper text (paperpeel.com/paper/2607.00712), cited below as
[ISPA §x]; and the reading notes at paper.gecl.asia (arxiv-cs-cv-2607-00712, section
"Method"), cited as [notes: Method]. The paper's equations were lost from every page;
where a step is open, the plainest reading is taken and named "Reading" below.

What is computed (per layer, per warmup chunk, then once at the transition):

1. Attention over the layer's KV cache, split into two partitions [ISPA §3.1 step 1]:
   the local partition = sink frame rows + current-chunk rows, and the history partition =
   every other cached row. A_full attends to all rows, A_loc to the local rows, A_hist to
   the history rows, each a plain softmax over its own mask (scale 1/sqrt(head_dim)), with
   its log-sum-exp. No causal mask inside the chunk (Reading: the chunk is denoised
   jointly), no positional rotation (Q/K are taken as already positioned).
2. Statistics for the closed-form absorption [ISPA §3.2; notes: Method, "ridge
   regression" on the attention output projection]: R = A_full - A_loc and, summed over the
   warmup chunks, G = A_loc^T A_loc, C = A_loc^T R, H = R^T R (row count kept too).
   Reading (bf16 workloads): A_loc and R are rounded to bf16 before the products, because
   the GPU feeds them to the tensor cores in bf16; the sums stay in float64 here.
3. Absorption [ISPA §3.1 step 2, §3.2, §4.1 "Eq. 5", lambda]: the update of the output
   projection minimises sum_t ||A_loc,t (W + dW) - A_full,t W||^2 + lambda ||dW||^2, so
   (G + lambda I) dW = C W. Solved here with a dense LU solve (numpy.linalg.solve), not
   with a Cholesky factorisation, so that it shares no algorithm with the GPU.
4. Reconstruction error [ISPA §3.3]. Reading: eps = E^2 / T^2, the relative squared error
   of the reconstructed projected output over the warmup, from traces:
   E^2 = tr(dW^T G dW) - 2 tr(dW^T C W) + tr(W^T H W)  (= ||A_loc (W+dW) - A_full W||^2)
   T^2 = tr(W^T (G + C + C^T + H) W)                   (= ||A_full W||^2)
   eps = 0 when T^2 = 0.
5. Selection [ISPA §3.3]: rank layers by eps ascending (ties by the lower layer index,
   NaN ranks last); the first K become L-layers with W_new = W + dW [ISPA §3.1 step 3].
6. After the switch an L-layer attends to the sink + chunk rows only and projects with
   W_new [ISPA §3.1 step 3, §3.3].
7. Re-warmup trigger [ISPA §3.1 last paragraph, §3.3 last paragraph: the warmup is entered
   again when the scene changes; no trigger is given]. Reading: after a transition each
   F-layer still sees its history, so the statistics of one live chunk (step 2 on that chunk
   alone) and the dW solved at the transition give a live error eps_live (step 4 on those
   statistics). The warmup is re-entered when a monitored layer's eps_live exceeds both 4 x
   and 0.02 + the lowest eps_live that layer showed since the transition. The reference is
   that live minimum, not the eps of the selection: eps at the selection is an in-sample
   figure, and where the residual is not predictable from A_loc (i.i.d. layers) dW overfits
   the warmup, so a fresh chunk's error is far above it without any change of scene. L-layers
   cannot be monitored: their history is gone.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


# --------------------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even) of float64 values, directly from the
# definition: a bf16 number carries 8 significant bits.
# --------------------------------------------------------------------------------------
def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned as float64.
    Values are assumed to lie in bf16's normal range (true for every tensor here)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                # x = m * 2**e, 0.5 <= |m| < 1
    m = np.rint(m * 256.0) / 256.0    # 8 significant bits; rint rounds half to even
    return np.ldexp(m, e)


# --------------------------------------------------------------------------------------
# Step 1: attention over explicit masks [ISPA §3.1 step 1, §3.4].
# --------------------------------------------------------------------------------------
def partition_masks(n_kv: int, sink: Tuple[int, int], chunk: Tuple[int, int]):
    """Boolean masks over the KV rows: full, local (sink + chunk) and history (the rest)."""
    full = np.ones(n_kv, dtype=bool)
    local = np.zeros(n_kv, dtype=bool)
    local[sink[0]:sink[1]] = True
    local[chunk[0]:chunk[1]] = True
    hist = ~local
    return full, local, hist


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, scale: float):
    """Softmax attention restricted to the KV rows where `mask` is True.

    q [n_q, h, d], k/v [n_kv, h, d] -> A [n_q, h, d] (float64), lse [h, n_q] (natural log of
    the sum of exp(scale * q.k) over the masked rows). An empty mask gives A = 0, lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_q, h, d = q.shape
    A = np.zeros((n_q, h, d), dtype=np.float64)
    lse = np.full((h, n_q), NEG_INF, dtype=np.float64)
    if not mask.any():
        return A, lse
    km = k[mask]
    vm = v[mask]
    for head in range(h):
        S = scale * (q[:, head, :] @ km[:, head, :].T)          # [n_q, n_mask]
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        A[:, head, :] = (P @ vm[:, head, :]) / l
        lse[head] = (m + np.log(l))[:, 0]
    return A, lse


def split_attention(q, k, v, sink: Tuple[int, int], chunk: Tuple[int, int], scale: float) -> Dict[str, np.ndarray]:
    """A_full, A_loc and A_hist (with their log-sum-exps), each from its own mask."""
    full, local, hist = partition_masks(k.shape[0], sink, chunk)
    A_full, lse_full = masked_attention(q, k, v, full, scale)
    A_loc, lse_loc = masked_attention(q, k, v, local, scale)
    A_hist, lse_hist = masked_attention(q, k, v, hist, scale)
    return dict(A_full=A_full, lse_full=lse_full, A_loc=A_loc, lse_loc=lse_loc,
                A_hist=A_hist, lse_hist=lse_hist)


def lse_merge(A1, lse1, A2, lse2):
    """Decomposable attention [ISPA §3.4, "Online Softmax"]: combine the outputs of two
    disjoint key partitions into the output over their union.
    A, lse in the layouts of masked_attention. lse = log(e^lse1 + e^lse2); each partition
    is weighted by e^(lse_i - lse)."""
    lse = np.logaddexp(lse1, lse2)                               # [h, n_q]
    with np.errstate(invalid="ignore"):
        w1 = np.where(np.isneginf(lse1), 0.0, np.exp(lse1 - lse))
        w2 = np.where(np.isneginf(lse2), 0.0, np.exp(lse2 - lse))
    w1 = w1.T[:, :, None]                                        # [n_q, h, 1]
    w2 = w2.T[:, :, None]
    return w1 * A1 + w2 * A2, lse


def local_attention(q, k_loc, v_loc, scale: float):
    """L-layer attention after the switch: all given rows are local (sink + chunk)."""
    return masked_attention(q, k_loc, v_loc, np.ones(k_loc.shape[0], dtype=bool), scale)


# --------------------------------------------------------------------------------------
# Step 2: statistics [ISPA §3.2; notes: Method].
# --------------------------------------------------------------------------------------
def stats_init(D: int) -> Dict[str, np.ndarray]:
    return dict(G=np.zeros((D, D)), C=np.zeros((D, D)), H=np.zeros((D, D)), rows=0)


def stats_operands(A_loc: np.ndarray, A_full: np.ndarray, dtype: str):
    """Rows of A_loc and R = A_full - A_loc as [n, D] matrices (column h*d + j), rounded
    to bf16 in bf16 mode."""
    n = A_loc.shape[0]
    a = np.asarray(A_loc, dtype=np.float64).reshape(n, -1)
    r = np.asarray(A_full, dtype=np.float64).reshape(n, -1) - a
    if dtype == "bf16":
        a = bf16_round(a)
        r = bf16_round(r)
    return a, r


def stats_update(stats: Dict[str, np.ndarray], A_loc: np.ndarray, A_full: np.ndarray, dtype: str) -> None:
    """G += A_loc^T A_loc, C += A_loc^T R, H += R^T R, rows += n."""
    a, r = stats_operands(A_loc, A_full, dtype)
    stats["G"] += a.T @ a
    stats["C"] += a.T @ r
    stats["H"] += r.T @ r
    stats["rows"] += a.shape[0]


# --------------------------------------------------------------------------------------
# Steps 3-5: absorption, error, selection [ISPA §3.1-§3.3, §4.1].
# --------------------------------------------------------------------------------------
def absorb_solve(G: np.ndarray, C: np.ndarray, W: np.ndarray, lam: float) -> np.ndarray:
    """dW solving (G + lambda I) dW = C W (ridge normal equations), dense LU solve."""
    D = G.shape[0]
    M = np.asarray(G, dtype=np.float64) + lam * np.eye(D)
    return np.linalg.solve(M, np.asarray(C, dtype=np.float64) @ np.asarray(W, dtype=np.float64))


def reconstruction_error(G, C, H, W, dW) -> Dict[str, float]:
    """eps = E^2 / T^2 from the traces listed in the module docstring."""
    G = np.asarray(G, np.float64); C = np.asarray(C, np.float64); H = np.asarray(H, np.float64)
    W = np.asarray(W, np.float64); dW = np.asarray(dW, np.float64)
    CW = C @ W
    t_dgd = float(np.sum(dW * (G @ dW)))        # tr(dW^T G dW)
    t_dcw = float(np.sum(dW * CW))              # tr(dW^T C W)
    t_whw = float(np.sum(W * (H @ W)))          # tr(W^T H W)
    t_wgw = float(np.sum(W * (G @ W)))          # tr(W^T G W)
    t_wcw = float(np.sum(W * CW))               # tr(W^T C W) = tr(W^T C^T W)
    E2 = t_dgd - 2.0 * t_dcw + t_whw
    T2 = t_wgw + 2.0 * t_wcw + t_whw
    eps = 0.0 if T2 == 0.0 else E2 / T2
    return dict(eps=eps, E2=E2, T2=T2)


def select_layers(eps: Sequence[float], K: int) -> Tuple[List[int], List[int]]:
    """The K layers with the lowest eps (ties: lower layer index first; NaN last).
    Returns (idx in rank order, is_local flags)."""
    L = len(eps)
    key = [(math.inf if (e != e) else float(e), l) for l, e in enumerate(eps)]
    order = [l for _, l in sorted(key)]
    idx = order[:max(0, min(K, L))]
    is_local = [0] * L
    for l in idx:
        is_local[l] = 1
    return idx, is_local


def project(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = A W with A as [n, D] (column h*d + j) and W stored [D_in, D_out]."""
    n = A.shape[0]
    return np.asarray(A, np.float64).reshape(n, -1) @ np.asarray(W, np.float64)


# --------------------------------------------------------------------------------------
# W8A8 projection of the L-layers [ISPA §4.4: ISPA combined with 8-bit weights and
# activations for the linear layers; the scheme is not given]. Reading: int8, symmetric,
# one scale per activation row (token) and one per weight output column; scales and the
# quantisation in float32 (round to nearest, ties to even, clamp to +-127); exact integer
# accumulation; y = bf16((float32(acc) * s_row) * s_col). Every step is a plain float32 or
# integer operation, so the GPU result is reproducible bit for bit.
# --------------------------------------------------------------------------------------
def quantize_int8(x: np.ndarray, axis: int) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantisation along `axis` (the reduced axis). Returns (q, scale) with
    scale = amax / 127 (float32) and q = rint(x * (127 / amax)) clamped to [-127, 127]; an
    all-zero slice has scale 0 and q = 0."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=axis, keepdims=True).astype(np.float32)
    inv = np.zeros_like(amax)
    nz = amax > 0
    inv[nz] = np.float32(127.0) / amax[nz]
    q = np.clip(np.rint(x * inv), -127, 127).astype(np.int8)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    return q, np.squeeze(scale, axis=axis)


def project_w8a8(A: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = A W through the int8 path above; A [n, D_in] (or [n, h, d]), W [D_in, D_out].
    Returns the bf16-rounded values as float64."""
    n = A.shape[0]
    qa, sa = quantize_int8(np.asarray(A, np.float32).reshape(n, -1), axis=1)
    qw, sw = quantize_int8(np.asarray(W, np.float32), axis=0)
    acc = qa.astype(np.int64) @ qw.astype(np.int64)
    y = (acc.astype(np.float32) * sa[:, None]) * sw[None, :]
    return bf16_round(y.astype(np.float64))


# --------------------------------------------------------------------------------------
# 8-bit split attention [ISPA §3.4: the decomposition is built on 8-bit attention kernels
# (SageAttention, SageAttention2), whose scheme the pages do not give]. Reading: as in
# SageAttention, S = scale * Q K^T is taken from int8 copies of Q and K, everything after
# it (softmax, P, P V, the partition merge, the statistics operands) exactly as in the bf16
# path. Q is quantised per (token, head); K per (block, head), a block being 128 rows of
# one partition segment (the sink range, the chunk range and the history runs around them,
# each cut into blocks from its first row; the last block of a segment is shorter). Each
# scale is symmetric, as in quantize_int8: amax / 127, with q = rint(x * (127 / amax)) in
# float32 (ties to even), clamped to +-127. Then S_ij = scale * s_q,i * s_k,b(j) * (q8_i . k8_j),
# the dot product exact in integers. No smoothing of K: the softmax ignores a per-row
# shift, but the log-sum-exp output would have to be corrected for it.
# --------------------------------------------------------------------------------------
def kv_blocks(n_kv: int, sink: Tuple[int, int], chunk: Tuple[int, int], rows: int = 128) -> List[Tuple[int, int]]:
    """(begin, end) of the K quantisation blocks, in row order."""
    loc = sorted(r for r in (tuple(sink), tuple(chunk)) if r[1] > r[0])
    segs = list(loc)
    cur = 0
    for b, e in loc:
        if b > cur:
            segs.append((cur, b))
        cur = max(cur, e)
    if cur < n_kv:
        segs.append((cur, n_kv))
    blocks = []
    for b, e in sorted(segs):
        blocks += [(r, min(r + rows, e)) for r in range(b, e, rows)]
    return blocks


def _i8_symmetric(x: np.ndarray, amax: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    amax = np.asarray(amax, dtype=np.float32)
    inv = np.zeros_like(amax)
    nz = amax > 0
    inv[nz] = np.float32(127.0) / amax[nz]
    q = np.clip(np.rint(x * inv), -127, 127).astype(np.int8)
    return q, (amax / np.float32(127.0)).astype(np.float32)


def quantize_i8_q(q: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Q [n, h, d] -> (q8 [n, h, d] int8, s_q [n, h] float32)."""
    x = np.asarray(q, dtype=np.float32)
    q8, sc = _i8_symmetric(x, np.max(np.abs(x), axis=2, keepdims=True) if x.size else np.zeros(x.shape[:2] + (1,)))
    return q8, np.ascontiguousarray(sc[:, :, 0])


def quantize_i8_k(k: np.ndarray, blocks: Sequence[Tuple[int, int]]) -> Tuple[np.ndarray, np.ndarray]:
    """K [n, h, d] -> (k8 [n, h, d] int8, s_k [h, n_blocks] float32), blocks from kv_blocks."""
    x = np.asarray(k, dtype=np.float32)
    n, h, d = x.shape
    k8 = np.zeros((n, h, d), dtype=np.int8)
    sk = np.zeros((h, len(blocks)), dtype=np.float32)
    for i, (b, e) in enumerate(blocks):
        amax = np.max(np.abs(x[b:e]), axis=(0, 2)).reshape(1, h, 1)
        k8[b:e], sc = _i8_symmetric(x[b:e], amax)
        sk[:, i] = sc[0, :, 0]
    return k8, sk


def split_attention_i8(q, k, v, sink: Tuple[int, int], chunk: Tuple[int, int], scale: float) -> Dict[str, np.ndarray]:
    """split_attention with S taken from the int8 copies: S = scale * s_q s_k (q8 . k8)."""
    blocks = kv_blocks(k.shape[0], sink, chunk)
    q8, sq = quantize_i8_q(q)
    k8, sk = quantize_i8_k(k, blocks)
    q_deq = q8.astype(np.float64) * sq.astype(np.float64)[:, :, None]
    k_deq = np.zeros(k8.shape, dtype=np.float64)
    for i, (b, e) in enumerate(blocks):
        k_deq[b:e] = k8[b:e].astype(np.float64) * sk[:, i].astype(np.float64)[None, :, None]
    out = split_attention(q_deq, k_deq, v, sink, chunk, scale)
    out.update(q8=q8, q_scale=sq, k8=k8, k_scale=sk, blocks=blocks)
    return out


# --------------------------------------------------------------------------------------
# A whole streaming run, chunk by chunk [ISPA §3.1, §3.3 re-triggered warmup].
# --------------------------------------------------------------------------------------
def live_error(A_loc, A_full, dtype: str, W, dW) -> float:
    """Step 7: eps of a given dW on the statistics of one chunk."""
    st = stats_init(np.asarray(W).shape[0])
    stats_update(st, A_loc, A_full, dtype)
    return reconstruction_error(st["G"], st["C"], st["H"], W, dW)["eps"]


def rewarm_trigger(previous: Sequence[Dict[int, float]], eps_live: Dict[int, float], ratio: float = 4.0,
                   min_rise: float = 0.02) -> List[int]:
    """Step 7's rule: the monitored layers whose live error rose above the lowest live error
    they showed on the earlier chunks since the transition (`previous`, oldest first)."""
    fired = []
    for l, e in eps_live.items():
        seen = [p[l] for p in previous if l in p]
        if seen and e > ratio * min(seen) and e > min(seen) + min_rise:
            fired.append(l)
    return sorted(fired)


def run_episode(cfg, n_chunks: Optional[int] = None, K: Optional[int] = None,
                keep_outputs: bool = False, rewarm_at="cut", monitor: bool = False) -> Dict[str, object]:
    """Warmup -> transition -> L/F inference (-> re-warmup at a scene cut) for a workload
    from `synth`. Reading of the schedule: the warmup covers cfg.warmup_chunks chunks; at
    a scene cut every layer restores its original W, its statistics restart from zero and
    it becomes an F-layer again; a former L-layer's history restarts at the cut. The new
    dW replaces the old one.

    Returns per-transition eps/dW/selection and, if asked, per-chunk per-layer outputs: the
    attention output O (A_full for an F-layer, A_loc for an L-layer), y = O W_cur and
    whether the layer ran local.

    rewarm_at: the chunk where the warmup is re-entered -- "cut" (the workload's scene cut,
    the default), None (never), or a chunk index. The scene itself always changes at the
    workload's cut. monitor=True adds step 7: for every chunk after a transition, the live
    error of each F-layer (key "live": list of (chunk, {layer: eps_live})).
    """
    import synth  # seeded inputs only

    L = cfg.layers
    K = cfg.K if K is None else K
    n_chunks = cfg.n_chunks if n_chunks is None else n_chunks
    W0 = [synth.w_out(cfg, l).astype(np.float64) for l in range(L)]
    W_cur = [w.copy() for w in W0]
    is_local = [0] * L
    hist_from: List[Optional[int]] = [None] * L
    stats = [stats_init(cfg.D) for _ in range(L)]
    warm_start = 0
    transitions = []
    outputs = []
    live = []
    rewarm_chunk = cfg.cut_chunk if rewarm_at == "cut" else rewarm_at
    for t in range(n_chunks):
        if rewarm_chunk is not None and t == rewarm_chunk:
            for l in range(L):
                if is_local[l]:
                    hist_from[l] = cfg.chunk_start_frame(t)
                is_local[l] = 0
                W_cur[l] = W0[l].copy()
                stats[l] = stats_init(cfg.D)
            warm_start = t
        in_warmup = warm_start <= t < warm_start + cfg.warmup_chunks
        watch = monitor and transitions and not in_warmup
        chunk_live = {}
        chunk_out = []
        for l in range(L):
            q = synth.chunk_q(cfg, l, t)
            if is_local[l]:
                frames = list(range(cfg.sink_frames)) + list(range(cfg.chunk_start_frame(t),
                                                                    cfg.chunk_start_frame(t) + cfg.chunk_frames))
                k = synth.kv_tensor(cfg, l, frames, "k")
                v = synth.kv_tensor(cfg, l, frames, "v")
                O, _ = local_attention(q, k, v, cfg.scale)
            else:
                frames = synth.cache_frames(cfg, t, hist_from[l])
                lay = synth.chunk_layout(cfg, frames, t)
                k = synth.kv_tensor(cfg, l, frames, "k")
                v = synth.kv_tensor(cfg, l, frames, "v")
                res = split_attention(q, k, v, (lay["sink_begin"], lay["sink_end"]),
                                      (lay["chunk_begin"], lay["chunk_end"]), cfg.scale)
                O = res["A_full"]
                if in_warmup:
                    stats_update(stats[l], res["A_loc"], res["A_full"], cfg.dtype)
                elif watch:
                    chunk_live[l] = live_error(res["A_loc"], res["A_full"], cfg.dtype, W0[l],
                                               transitions[-1]["dW"][l])
            if keep_outputs:
                chunk_out.append(dict(O=O, y=project(O, W_cur[l]), local=bool(is_local[l])))
        if keep_outputs:
            outputs.append(chunk_out)
        if watch:
            live.append((t, chunk_live))
        if in_warmup and t == warm_start + cfg.warmup_chunks - 1:
            dWs, errs = [], []
            for l in range(L):
                s = stats[l]
                dW = absorb_solve(s["G"], s["C"], W0[l], cfg.lam)
                dWs.append(dW)
                errs.append(reconstruction_error(s["G"], s["C"], s["H"], W0[l], dW))
            eps = [e["eps"] for e in errs]
            idx, flags = select_layers(eps, K)
            for l in idx:
                W_cur[l] = W0[l] + dWs[l]
            is_local = list(flags)
            transitions.append(dict(chunk=t, eps=eps, errs=errs, dW=dWs, idx=idx, is_local=list(flags),
                                    stats=[dict(G=s["G"].copy(), C=s["C"].copy(), H=s["H"].copy(),
                                                rows=s["rows"]) for s in stats]))
    return dict(transitions=transitions, outputs=outputs, live=live)
