"""Failure detection without faulting the GPU: a bounded device-side wait that runs out
reports ISPA_ERR_TIMEOUT through the device flag and leaves the context usable."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from streaming_video_attention_b200 import ispa
from tests.helpers import rel_fro, to_device, to_numpy

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    ispa.ispa_selftest_bounded_wait(2000)            # 2 ms; nothing ever arrives
    assert ispa.ispa_device_status() == ispa.ISPA_ERR_TIMEOUT
    assert ispa.ispa_device_status() == ispa.ISPA_OK  # the flag was cleared
    # the context still works
    q = synth.normal_tensor(3, (1,), (130, 2, 128), "bf16")
    k = synth.normal_tensor(3, (2,), (300, 2, 128), "bf16")
    v = synth.normal_tensor(3, (3,), (300, 2, 128), "bf16")
    desc = ispa.make_desc(130, 300, 2, 128, (0, 50), (170, 300), dtype=ispa.ISPA_BF16)
    o = torch.empty((130, 2, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 130), device="cuda")
    ispa.ispa_attn_split(desc, to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), o, lse)
    assert ispa.ispa_device_status() == ispa.ISPA_OK
    want = oracle.split_attention(q, k, v, (0, 50), (170, 300), 1 / math.sqrt(128))
    assert rel_fro(to_numpy(o), want["A_full"]) < 2e-2


def test_workspace_errors_are_reported():
    desc = ispa.make_desc(128, 256, 2, 128, (0, 64), (128, 256), dtype=ispa.ISPA_BF16)
    x = torch.zeros((256, 2, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((128, 2, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 128), device="cuda")
    st = ispa.Stats(256)
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split(desc, x[:128], x, x, o, lse, stats=st, ws=None)
    assert ei.value.code == ispa.ISPA_ERR_WORKSPACE
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split(desc, x[:128], x, x, o, lse, stats=st, ws=small)
    assert ei.value.code == ispa.ISPA_ERR_WORKSPACE
    bad = ispa.Stats(128)
    with pytest.raises(ispa.IspaError) as ei:
        ispa.ispa_attn_split(desc, x[:128], x, x, o, lse, stats=bad,
                             ws=ispa.alloc_workspace(ispa.workspace_bytes(desc, 0, 0)))
    assert ei.value.code == ispa.ISPA_ERR_INVALID_ARG


def test_fma_pipe_exponential_error_bound():
    """The softmax's FMA-pipe 2^x stays within 1e-4 relative of the exact value (bf16 rounding
    of the weights it feeds is 2^-9 = 2e-3), and agrees with CUDA's exp2f on the same inputs."""
    # odd length: pairs go through the packed form, the last element through the scalar one
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.99, 3.3])]).cuda()
    y = torch.empty_like(x)
    ispa.ispa_selftest_exp2_poly(x, y)
    torch.cuda.synchronize()
    exact = np.exp2(x.double().cpu().numpy())
    rel = np.abs(y.double().cpu().numpy() - exact) / exact
    assert rel.max() < 1e-4, rel.max()
    rel_cuda = (y - torch.exp2(x)).abs() / torch.exp2(x)
    assert float(rel_cuda.max()) < 1e-4
