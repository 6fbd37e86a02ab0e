"""ispa_attn_split_noalloc: the warmup call for callers that cannot allocate device memory
(a host framework that owns all device memory, a plugin interface without a workspace).
It must give the same attention outputs and the same accumulated statistics as
ispa_attn_split with a caller workspace, over two calls in a row (the statistics add up;
the static scratch keeps the previous call's contents, which must not leak into the next).
"""
import math

import numpy as np
import pytest
import torch

import synth
from streaming_video_attention_b200 import ispa
from tests.helpers import rel_fro, to_device, to_numpy

pytestmark = pytest.mark.gpu


def _inputs(seed, n_q, n_kv, heads, hd):
    q = synth.normal_tensor(seed, (1,), (n_q, heads, hd), "bf16")
    k = synth.normal_tensor(seed, (2,), (n_kv, heads, hd), "bf16")
    v = synth.normal_tensor(seed, (3,), (n_kv, heads, hd), "bf16")
    return to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16")


def test_noalloc_matches_workspace_entry_point_over_two_calls():
    heads, hd, tpf = 2, 128, 200
    n_q, n_kv = 3 * tpf, 8 * tpf
    sink, chunk = (0, tpf), (5 * tpf, 8 * tpf)
    desc = ispa.make_desc(n_q, n_kv, heads, hd, sink, chunk, dtype=ispa.ISPA_BF16)
    st_ws, st_na = ispa.Stats(heads * hd), ispa.Stats(heads * hd)
    ws = ispa.alloc_workspace(ispa.workspace_bytes(desc, 0, 0))
    for call in range(2):
        q, k, v = _inputs(30 + call, n_q, n_kv, heads, hd)
        outs = []
        for use_static in (False, True):
            o = torch.full((n_q, heads, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
            lse = torch.full((heads, n_q), float("nan"), device="cuda")
            if use_static:
                ispa.ispa_attn_split_noalloc(desc, q, k, v, o, lse, stats=st_na)
            else:
                ispa.ispa_attn_split(desc, q, k, v, o, lse, stats=st_ws, ws=ws)
            outs.append((o, lse))
        torch.cuda.synchronize()
        assert ispa.ispa_device_status() == ispa.ISPA_OK
        (o_a, l_a), (o_b, l_b) = outs
        assert rel_fro(to_numpy(o_b), to_numpy(o_a)) < 2e-2
        assert np.max(np.abs(to_numpy(l_b) - to_numpy(l_a))) < 2e-2
        for name in ("G", "C", "H"):
            assert rel_fro(to_numpy(getattr(st_na, name)), to_numpy(getattr(st_ws, name))) < 1e-5, (call, name)
        assert int(st_na.rows.item()) == int(st_ws.rows.item()) == (call + 1) * n_q


def test_noalloc_rejects_calls_beyond_the_static_scratch():
    # 4680 x 40 x 128 bf16 = 46.8 MB per operand > 16 MiB: refused before any launch
    desc = ispa.make_desc(4680, 37440, 40, 128, (0, 1560), (32760, 37440), dtype=ispa.ISPA_BF16)
    st = ispa.Stats(40 * 128)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split_noalloc(desc, x, x, x, x, torch.zeros(1, device="cuda"), stats=st)
    assert ei.value.code == ispa.ISPA_ERR_UNSUPPORTED
    assert "16 MiB" in str(ei.value)
