"""GPU parity of the three bf16 head_dim-128 split-attention kernels (one CTA per query tile;
CTA pairs with cta_group::2 MMAs; one CTA with two softmax groups on alternate KV tiles), each
against the CPU oracle on the same seeded inputs.

Tolerances: as for every bf16 attention check, 2e-2 relative Frobenius per output tensor and
2e-2 absolute on lse; the fused statistics 2e-2 relative. The two kernels against each other
on a full 1.3B-shaped layer: 1e-2 relative (all round P and the outputs to bf16; they differ
in accumulation order, and the two-group kernel also rounds each group's normalised local part
to bf16 before merging them).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from streaming_video_attention_b200 import ispa
from tests.helpers import rel_fro, to_numpy
from tests.test_gpu_parity import _attn_case, _check_attn, _run_split

pytestmark = pytest.mark.gpu

KERNELS = {"single": ispa.ISPA_ATTN_SINGLE, "pair": ispa.ISPA_ATTN_PAIR, "two_group": ispa.ISPA_ATTN_TWO_GROUP}


@pytest.fixture(params=sorted(KERNELS))
def attn_kernel(request):
    prev = ispa.ispa_set_attn_kernel(KERNELS[request.param])
    yield request.param
    ispa.ispa_set_attn_kernel(prev)


@pytest.mark.parametrize("layout", ["sink_hist_chunk", "no_history", "no_sink", "chunk_inside"])
def test_kernel_matches_oracle(attn_kernel, layout):
    tpf, heads, hd = 200, 3, 128
    n_q = 3 * tpf                    # 5 query tiles (the last ragged): the pair grid has an empty 6th
    if layout == "sink_hist_chunk":
        n_kv, sink, chunk = 8 * tpf, (0, tpf), (5 * tpf, 8 * tpf)
    elif layout == "no_history":
        n_kv, sink, chunk = 4 * tpf, (0, tpf), (tpf, 4 * tpf)
    elif layout == "no_sink":
        n_kv, sink, chunk = 7 * tpf + 37, (0, 0), (4 * tpf + 37, 7 * tpf + 37)
    else:
        n_kv, sink, chunk = 9 * tpf + 5, (3, 3 + tpf), (2 * tpf + 50, 5 * tpf + 50)
    q, k, v = _attn_case(31, n_q, n_kv, heads, hd, "bf16")
    got = _run_split(q, k, v, sink, chunk, "bf16")
    want = oracle.split_attention(q, k, v, sink, chunk, 1 / math.sqrt(hd))
    _check_attn(got, want, "bf16")


@pytest.mark.parametrize("n_q,n_kv,sink,chunk", [
    (1, 130, (0, 1), (2, 130)),          # one query row; history of one row
    (128, 64, (0, 10), (10, 64)),        # exactly one query tile; K/V shorter than a half tile
    (129, 129, (0, 64), (65, 129)),      # a 1-row query tail; a 1-row KV tail
    (256, 700, (0, 0), (300, 700)),      # exactly one tile pair; no sink
    (5, 3, (0, 1), (1, 3)),              # fewer keys than anything
    (128, 300, (0, 0), (200, 300)),      # one local tile, then history: the odd group hands over first
    (200, 1000, (0, 64), (900, 1000)),   # two local tiles; the history tiles alternate between groups
])
def test_kernel_edge_sizes(attn_kernel, n_q, n_kv, sink, chunk):
    q, k, v = _attn_case(77, n_q, n_kv, 2, 128, "bf16")
    got = _run_split(q, k, v, sink, chunk, "bf16")
    want = oracle.split_attention(q, k, v, sink, chunk, 1 / math.sqrt(128))
    _check_attn(got, want, "bf16")


def test_kernel_fused_stats(attn_kernel):
    tpf, heads, hd = 200, 2, 128
    n_q, n_kv, sink, chunk = 3 * tpf, 8 * tpf, (0, tpf), (5 * tpf, 8 * tpf)
    q, k, v = _attn_case(5, n_q, n_kv, heads, hd, "bf16")
    st = ispa.Stats(heads * hd)
    got = _run_split(q, k, v, sink, chunk, "bf16", stats=st)
    want = oracle.split_attention(q, k, v, sink, chunk, 1 / math.sqrt(hd))
    _check_attn(got, want, "bf16")
    ref = oracle.stats_init(heads * hd)
    oracle.stats_update(ref, want["A_loc"], want["A_full"], "bf16")
    for name in ("G", "C", "H"):
        assert rel_fro(to_numpy(getattr(st, name)), ref[name]) < 2e-2, name
    assert int(st.rows.item()) == n_q


def test_kernels_agree_on_full_1p3b_layer():
    """Every kernel against the single-CTA one on a 1.3B-shaped layer call (n_q 4680, n_kv 37440, 12 heads): every
    output element, not a sample."""
    cfg = synth.CONFIGS["1p3b_bf16"]
    t, layer = cfg.warmup_chunks - 1, 5
    frames = synth.cache_frames(cfg, t)
    lay = synth.chunk_layout(cfg, frames, t)
    q = synth.chunk_q(cfg, layer, t)
    k = synth.kv_tensor(cfg, layer, frames, "k")
    v = synth.kv_tensor(cfg, layer, frames, "v")
    sink, chunk = (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"])
    res = {}
    for name, choice in KERNELS.items():
        prev = ispa.ispa_set_attn_kernel(choice)
        try:
            res[name] = _run_split(q, k, v, sink, chunk, "bf16")
        finally:
            ispa.ispa_set_attn_kernel(prev)
    for other in sorted(set(KERNELS) - {"single"}):
        for key in res["single"]:
            a, b = res["single"][key], res[other][key]
            if key.startswith("A_"):
                assert rel_fro(b, a) < 1e-2, (other, key)
            else:
                assert np.array_equal(np.isfinite(a), np.isfinite(b)), (other, key)
                fin = np.isfinite(a)
                assert np.max(np.abs(a[fin] - b[fin])) < 1e-2, (other, key)

