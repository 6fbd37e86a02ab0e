"""ispa_attn_split_noalloc: the warmup call for callers that cannot allocate device memory
(a host framework that owns all device memory, a plugin interface without a workspace).
It runs the same kernels as ispa_attn_split with a caller workspace, only with the statistics
operands in the library's static scratch, so the attention outputs and the accumulated
statistics must be identical bit for bit, over two calls in a row (the statistics add up; the
static scratch keeps the previous call's contents, which must not leak into the next).
"""
import numpy as np
import pytest
import torch

import synth
from streaming_video_attention_b200 import ispa
from tests.helpers import to_device

pytestmark = pytest.mark.gpu

SLOT = 16 << 20   # bytes of one operand slot of the static scratch


def _inputs(seed, n_q, n_kv, heads, hd, dtype):
    q = synth.normal_tensor(seed, (1,), (n_q, heads, hd), dtype)
    k = synth.normal_tensor(seed, (2,), (n_kv, heads, hd), dtype)
    v = synth.normal_tensor(seed, (3,), (n_kv, heads, hd), dtype)
    return to_device(q, dtype), to_device(k, dtype), to_device(v, dtype)


def _compare_two_calls(n_q, n_kv, heads, hd, sink, chunk, dtype, seed0):
    code = ispa.ISPA_BF16 if dtype == "bf16" else ispa.ISPA_FP32
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    desc = ispa.make_desc(n_q, n_kv, heads, hd, sink, chunk, dtype=code)
    st_ws, st_na = ispa.Stats(heads * hd), ispa.Stats(heads * hd)
    ws = ispa.alloc_workspace(ispa.workspace_bytes(desc, 0, 0))
    for call in range(2):
        q, k, v = _inputs(seed0 + call, n_q, n_kv, heads, hd, dtype)
        outs = []
        for use_static in (False, True):
            o = torch.full((n_q, heads, hd), float("nan"), dtype=td, device="cuda")
            ol = torch.full_like(o, float("nan"))
            lse = torch.full((heads, n_q), float("nan"), device="cuda")
            if use_static:
                ispa.ispa_attn_split_noalloc(desc, q, k, v, o, lse, ol, stats=st_na)
            else:
                ispa.ispa_attn_split(desc, q, k, v, o, lse, ol, stats=st_ws, ws=ws)
            outs.append((o, ol, lse))
        torch.cuda.synchronize()
        assert ispa.ispa_device_status() == ispa.ISPA_OK
        for a, b in zip(*outs):
            assert torch.equal(a, b), call
        for name in ("G", "C", "H"):
            assert torch.equal(getattr(st_na, name), getattr(st_ws, name)), (call, name)
        assert int(st_na.rows.item()) == int(st_ws.rows.item()) == (call + 1) * n_q


@pytest.mark.parametrize("dtype,hd", [("bf16", 128), ("bf16", 64), ("fp32", 64)])
def test_noalloc_matches_workspace_entry_point_over_two_calls(dtype, hd):
    heads, tpf = 2, 200
    _compare_two_calls(3 * tpf, 8 * tpf, heads, hd, (0, tpf), (5 * tpf, 8 * tpf), dtype, 30)


def test_noalloc_full_1p3b_layer():
    """A 1.3B-shaped layer call (4680 x 12 x 128: 14.4 MB per operand, inside the 16 MiB slot)."""
    cfg = synth.CONFIGS["1p3b_bf16"]
    t = cfg.warmup_chunks - 1
    lay = synth.chunk_layout(cfg, synth.cache_frames(cfg, t), t)
    assert cfg.n_q * cfg.D * 2 <= SLOT
    _compare_two_calls(cfg.n_q, lay["n_kv"], cfg.heads, cfg.head_dim, (lay["sink_begin"], lay["sink_end"]),
                       (lay["chunk_begin"], lay["chunk_end"]), "bf16", 50)


def test_noalloc_size_limit_is_exact():
    """An operand of exactly 16 MiB is accepted (and matches the workspace call); one query row
    more is refused before any launch."""
    heads, hd = 2, 128
    n_max = SLOT // (heads * hd * 2)                    # 32768 rows of bf16
    _compare_two_calls(n_max, 256, heads, hd, (0, 64), (128, 256), "bf16", 70)
    desc = ispa.make_desc(n_max + 1, 256, heads, hd, (0, 64), (128, 256), dtype=ispa.ISPA_BF16)
    st = ispa.Stats(heads * hd)
    q, k, v = _inputs(71, n_max + 1, 256, heads, hd, "bf16")
    o = torch.empty_like(q)
    lse = torch.empty((heads, n_max + 1), device="cuda")
    launches = ispa.ispa_kernel_launches()
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split_noalloc(desc, q, k, v, o, lse, stats=st)
    assert ei.value.code == ispa.ISPA_ERR_UNSUPPORTED
    assert "16 MiB" in str(ei.value)
    assert ispa.ispa_kernel_launches() == launches


def test_noalloc_rejects_calls_beyond_the_static_scratch():
    # 4680 x 40 x 128 bf16 = 46.8 MB per operand > 16 MiB: refused before any launch
    desc = ispa.make_desc(4680, 37440, 40, 128, (0, 1560), (32760, 37440), dtype=ispa.ISPA_BF16)
    st = ispa.Stats(40 * 128)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split_noalloc(desc, x, x, x, x, torch.zeros(1, device="cuda"), stats=st)
    assert ei.value.code == ispa.ISPA_ERR_UNSUPPORTED
    assert "16 MiB" in str(ei.value)
