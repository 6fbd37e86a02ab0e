"""The C-ABI library: it loads, exports every symbol the header declares, and its host-only
logic (argument checks, workspace sizing, layer selection) behaves. No GPU is touched."""
import ctypes
import json
import math
import os
import re

import pytest

from streaming_video_attention_b200 import ispa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(ispa_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = ispa.lib()
    declared = _declared_symbols()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(ispa.EXPORTS)
    assert b"sm_100a" in L.ispa_version()


def test_invalid_arguments_are_rejected_before_any_launch():
    L = ispa.lib()
    assert L.ispa_attn_split(None, None, None, None, None, None, None, None, None, None, None, None, 0,
                             None) == ispa.ISPA_ERR_INVALID_ARG
    assert b"desc" in L.ispa_last_error()
    d = ispa.make_desc(128, 64, 2, 96)
    assert L.ispa_attn_split(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, None, 0,
                             None) == ispa.ISPA_ERR_UNSUPPORTED
    d = ispa.make_desc(128, 64, 2, 64, sink=(0, 40), chunk=(30, 64))
    assert L.ispa_attn_split(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, None, 0,
                             None) == ispa.ISPA_ERR_INVALID_ARG
    assert b"overlap" in L.ispa_last_error()
    d = ispa.make_desc(128, 64, 2, 64, sink=(0, 70), chunk=(0, 0))
    assert L.ispa_attn_split(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, None, 0,
                             None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_select_layers(None, 3, 1, None, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_selftest_bounded_wait(0, None) == ispa.ISPA_ERR_INVALID_ARG


def test_project_arguments_are_checked_before_any_launch():
    L = ispa.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails its checks first
    assert L.ispa_project(fake, -1, 128, fake, 128, fake, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project(fake, 4, 0, fake, 128, fake, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project(fake, 4, 128, fake, 128, fake, 7, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project(None, 4, 128, fake, 128, fake, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project(ctypes.c_void_p((1 << 20) + 2), 4, 128, fake, 128, fake, ispa.ISPA_BF16,
                          None) == ispa.ISPA_ERR_INVALID_ARG
    assert b"aligned" in L.ispa_last_error()
    assert L.ispa_project(None, 0, 128, None, 128, None, ispa.ISPA_BF16, None) == ispa.ISPA_OK


def test_workspace_sizes():
    d = ispa.make_desc(4680, 37440, 12, 128, dtype=ispa.ISPA_BF16)
    # fused statistics need the A_loc and R operands: 2 * n_q * D bf16
    assert ispa.workspace_bytes(d, 0, 0) >= 2 * 4680 * 1536 * 2
    # the solve needs three D x D float32 matrices per layer in a batch
    assert ispa.workspace_bytes(None, 30, 1536) >= 30 * 3 * 1536 * 1536 * 4


def test_select_layers_golden():
    with open(os.path.join(ROOT, "tests", "golden", "selection_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        eps = [math.nan if e == "nan" else e for e in c["eps"]]
        idx, flags = ispa.ispa_select_layers(eps, c["K"])
        assert idx == c["idx"], c
        assert flags == c["is_local"], c


def test_select_layers_matches_oracle_on_random_errors():
    import numpy as np
    import oracle
    rng = np.random.default_rng(5)
    for trial in range(50):
        L = int(rng.integers(1, 60))
        eps = rng.choice([0.1, 0.2, 0.3], size=L) if trial % 2 else rng.random(L)
        eps = eps.astype(np.float32).tolist()
        K = int(rng.integers(0, L + 2))
        assert ispa.ispa_select_layers(eps, K) == oracle.select_layers(eps, K)


def test_set_attn_kernel_choice_round_trips():
    prev = ispa.ispa_set_attn_kernel(ispa.ISPA_ATTN_PAIR)
    try:
        assert ispa.ispa_set_attn_kernel(ispa.ISPA_ATTN_SINGLE) == ispa.ISPA_ATTN_PAIR
        with pytest.raises(ispa.IspaError):
            ispa.ispa_set_attn_kernel(7)
        assert ispa.ispa_set_attn_kernel(ispa.ISPA_ATTN_TWO_GROUP) == ispa.ISPA_ATTN_SINGLE
        assert ispa.ispa_set_attn_kernel(ispa.ISPA_ATTN_AUTO) == ispa.ISPA_ATTN_TWO_GROUP
    finally:
        ispa.ispa_set_attn_kernel(prev)


def test_w8a8_arguments_are_checked_before_any_launch():
    L = ispa.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails its checks first
    assert L.ispa_quantize_w8(None, ispa.ISPA_BF16, 128, 128, fake, fake, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_quantize_w8(fake, ispa.ISPA_BF16, 96, 128, fake, fake, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_quantize_w8(fake, 7, 128, 128, fake, fake, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project_w8a8(fake, 10, 128, fake, fake, 200, fake, None, 0, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_project_w8a8(fake, 10, 128, fake, fake, 128, fake, None, 0, None) == ispa.ISPA_ERR_WORKSPACE
    assert L.ispa_project_w8a8(None, 10, 128, fake, fake, 128, fake, None, 0, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_project_w8a8(fake, 0, 128, fake, fake, 128, fake, None, 0, None) == ispa.ISPA_OK
    # the workspace covers the row codes and scales
    assert ispa.workspace_bytes(None, 4680, 1536) >= 4680 * 1536 + 4 * 4680


def test_k_blocks_count_matches_oracle():
    import oracle
    for n_kv, sink, chunk in [(1000, (0, 64), (900, 1000)), (300, (0, 0), (200, 300)), (640, (0, 130), (130, 640)),
                              (5, (0, 1), (1, 3)), (37440, (0, 1560), (32760, 37440)), (0, (0, 0), (0, 0))]:
        desc = ispa.make_desc(10, n_kv, 2, 128, sink, chunk)
        assert ispa.ispa_k_blocks(desc) == len(oracle.kv_blocks(n_kv, sink, chunk)), (n_kv, sink, chunk)


def test_i8_arguments_are_checked_before_any_launch():
    L = ispa.lib()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails its checks first
    d64 = ispa.make_desc(10, 100, 2, 64, (0, 10), (50, 100))
    dfp32 = ispa.make_desc(10, 100, 2, 128, (0, 10), (50, 100), dtype=ispa.ISPA_FP32)
    d128 = ispa.make_desc(10, 100, 2, 128, (0, 10), (50, 100))
    assert L.ispa_quantize_q_i8(fake, 10, 2, 64, fake, fake, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_quantize_q_i8(fake, 10, 2, 128, None, fake, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_quantize_k_i8(ctypes.byref(d64), fake, fake, fake, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_quantize_k_i8(ctypes.byref(d128), fake, fake, None, None) == ispa.ISPA_ERR_INVALID_ARG
    args = (fake, fake, fake, fake, fake, fake, fake, None, None, None, None, None, None, 0, None)
    assert L.ispa_attn_split_i8(ctypes.byref(dfp32), *args) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_attn_split_i8(ctypes.byref(d64), *args) == ispa.ISPA_ERR_UNSUPPORTED
    no_qs = (fake, None) + args[2:]
    assert L.ispa_attn_split_i8(ctypes.byref(d128), *no_qs) == ispa.ISPA_ERR_INVALID_ARG


def test_split_ops_and_accum_ops_arguments_are_checked_before_any_launch():
    L = ispa.lib()
    fake = ctypes.c_void_p(1 << 20)
    d = ispa.make_desc(10, 100, 2, 128, (0, 10), (50, 100))
    assert L.ispa_attn_split_ops(ctypes.byref(d), fake, fake, fake, fake, fake, None, None, None, None, None, fake,
                                 None) == ispa.ISPA_ERR_INVALID_ARG              # a_ops missing
    assert L.ispa_accum_ops(None, 1, fake, fake, 10, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_accum_ops(None, 0, None, None, 0, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG
    st = (ispa.CStats * 2)(ispa.CStats(256, 1 << 20, 1 << 20, 1 << 20, 1 << 20),
                           ispa.CStats(128, 1 << 20, 1 << 20, 1 << 20, 1 << 20))
    assert L.ispa_accum_ops(st, 2, fake, fake, 10, ispa.ISPA_BF16, None) == ispa.ISPA_ERR_INVALID_ARG   # D differs
    assert L.ispa_accum_ops(st, 0, None, None, 10, ispa.ISPA_BF16, None) == ispa.ISPA_OK                 # no layers
