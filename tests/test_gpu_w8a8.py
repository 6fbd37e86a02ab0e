"""W8A8 projection of the L-layers (int8 weights and activations, int32 accumulation on the
tensor cores) against the oracle's statement of the same scheme: bit-exact, since every step is
a plain float32 or integer operation (codes, scales and the bf16 outputs compared bit for bit)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from streaming_video_attention_b200 import ispa
from streaming_video_attention_b200.session import IspaSession
from tests.helpers import rel_fro, to_device, to_numpy

pytestmark = pytest.mark.gpu


def _quantize_gpu(W, dtype):
    d_in, d_out = W.shape
    wq = torch.empty(d_out, d_in, dtype=torch.int8, device="cuda")
    ws = torch.empty(d_out, dtype=torch.float32, device="cuda")
    ispa.ispa_quantize_w8(to_device(W, dtype), ispa.ISPA_BF16 if dtype == "bf16" else ispa.ISPA_FP32, wq, ws)
    return wq, ws


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_weight_codes_and_scales_are_bit_exact(dtype):
    W = synth.normal_tensor(3, (40,), (256, 384), dtype, std=0.05)
    W[:, 5] = 0.0                                         # a zero column: scale 0, codes 0
    wq, ws = _quantize_gpu(W, dtype)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_int8(W, axis=0)
    assert np.array_equal(wq.cpu().numpy(), q_ref.T)
    assert np.array_equal(ws.cpu().numpy(), s_ref)


@pytest.mark.parametrize("n", [1, 300, 512])
def test_projection_is_bit_exact(n):
    D_in, D_out = 256, 384
    A = synth.normal_tensor(4, (41,), (n, D_in), "bf16")
    if n > 3:
        A[2] = 0.0                                        # a zero row
    W = synth.normal_tensor(5, (42,), (D_in, D_out), "bf16", std=1 / math.sqrt(D_in))
    wq, wsc = _quantize_gpu(W, "bf16")
    y = torch.full((n, D_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = ispa.alloc_workspace(ispa.workspace_bytes(None, n, D_in))
    ispa.ispa_project_w8a8(to_device(A, "bf16"), wq, wsc, y, ws)
    torch.cuda.synchronize()
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    want = oracle.project_w8a8(A, W)
    assert np.array_equal(to_numpy(y), want)
    # and it stays close to the bf16 projection
    assert rel_fro(to_numpy(y), A.astype(np.float64) @ W.astype(np.float64)) < 2e-2


def test_full_size_1p3b_projection_sampled_rows():
    """n_q 4680, D 1536 (37 row tiles, the last ragged): rows sampled for the oracle, which
    quantises each row on its own and so needs only those rows; weights quantised in full."""
    n, D = 4680, 1536
    A = synth.normal_tensor(6, (43,), (n, D), "bf16", std=0.02)
    W = synth.normal_tensor(7, (44,), (D, D), "bf16", std=1 / math.sqrt(D))
    wq, wsc = _quantize_gpu(W, "bf16")
    y = torch.empty((n, D), dtype=torch.bfloat16, device="cuda")
    ws = ispa.alloc_workspace(ispa.workspace_bytes(None, n, D))
    ispa.ispa_project_w8a8(to_device(A, "bf16"), wq, wsc, y, ws)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, n, 97), [127, 128, 4607, 4608, n - 1]]))
    want = oracle.project_w8a8(A[rows], W)
    assert np.array_equal(to_numpy(y)[rows], want)


def test_session_l_layers_project_through_w8a8():
    """A session with w8a8=True: after the transition, the L-layer's y equals the oracle's W8A8
    projection of the same attention output with the same W_new, bit for bit."""
    cfg = synth.IspaConfig(name="w8a8_small", layers=2, heads=2, head_dim=128, tpf=64, chunk_frames=2, h_max=6,
                           warmup_chunks=3, lam=1e-2, K=1, dtype="bf16")
    sess = IspaSession(cfg.layers, cfg.heads, cfg.head_dim, cfg.lam, cfg.K, "bf16", w8a8=True)
    sess.set_weights([to_device(synth.w_out(cfg, l), "bf16") for l in range(cfg.layers)])
    sess.rewarm()
    for t in range(cfg.warmup_chunks):
        for l in range(cfg.layers):
            frames = synth.cache_frames(cfg, t)
            lay = synth.chunk_layout(cfg, frames, t)
            q = to_device(synth.chunk_q(cfg, l, t), "bf16")
            k = to_device(synth.kv_tensor(cfg, l, frames, "k"), "bf16")
            v = to_device(synth.kv_tensor(cfg, l, frames, "v"), "bf16")
            o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((cfg.heads, cfg.n_q), device="cuda")
            sess.full_attention(l, q, k, v, (lay["sink_begin"], lay["sink_end"]), (lay["chunk_begin"], lay["chunk_end"]),
                                o, lse, collect=True)
    idx = sess.transition()
    l = idx[0]
    t = cfg.warmup_chunks
    s0 = cfg.chunk_start_frame(t)
    frames = list(range(cfg.sink_frames)) + list(range(s0, s0 + cfg.chunk_frames))
    q = to_device(synth.chunk_q(cfg, l, t), "bf16")
    k = to_device(synth.kv_tensor(cfg, l, frames, "k"), "bf16")
    v = to_device(synth.kv_tensor(cfg, l, frames, "v"), "bf16")
    o = torch.empty((cfg.n_q, cfg.heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((cfg.n_q, cfg.D), dtype=torch.bfloat16, device="cuda")
    sess.local_attention(l, q, k, v, o, None, y)
    torch.cuda.synchronize()
    want = oracle.project_w8a8(to_numpy(o).reshape(cfg.n_q, -1), to_numpy(sess.W_new[l]))
    assert np.array_equal(to_numpy(y), want)
