"""Host logic of the streaming session that needs no GPU: the re-warmup trigger rule (the
library's ispa_rewarm_check, a host-only call), against the oracle's statement of the same rule on
hand cases and random live-error histories."""
import types

import numpy as np

import oracle
from streaming_video_attention_b200.session import IspaSession


def _session_rule(history):
    layers = 1 + max((l for d in history for l in d), default=0)
    fake = types.SimpleNamespace(live_history=history, layers=layers, RATIO=IspaSession.RATIO,
                                 MIN_RISE=IspaSession.MIN_RISE)
    return IspaSession.rewarm_layers(fake)


def test_rule_needs_a_reference_chunk():
    assert _session_rule([]) == []
    assert _session_rule([{0: 3.0}]) == []


def test_rule_hand_cases():
    hist = [{1: 0.01, 2: 2.0}, {1: 0.012, 2: 2.4}]
    assert _session_rule(hist + [{1: 0.3, 2: 2.2}]) == [1]
    assert _session_rule(hist + [{1: 0.011, 2: 8.5}]) == [2]
    assert _session_rule(hist + [{1: 0.029, 2: 2.0}]) == []
    assert _session_rule([{3: 1e-4}, {3: 9e-3}]) == []


def test_rewarm_check_abi():
    from streaming_video_attention_b200 import ispa
    nan = float("nan")
    # layer 0 rises 30x; layer 1 is not monitored in the latest chunk; layer 2 has no earlier value;
    # layer 3 rises 5x but by less than min_rise
    hist = [[0.01, 0.5, nan, 0.001], [0.012, 0.4, nan, 0.002], [0.3, nan, 9.0, 0.005]]
    assert ispa.ispa_rewarm_check(hist, 4.0, 0.02) == [1, 0, 0, 0]
    assert ispa.ispa_rewarm_check(hist, 4.0, 0.0) == [1, 0, 0, 1]
    assert ispa.ispa_rewarm_check(hist[:1], 4.0, 0.02) == [0, 0, 0, 0]
    L = ispa.lib()
    assert L.ispa_rewarm_check(None, 2, 3, 4.0, 0.02, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_rewarm_check(None, -1, 0, 4.0, 0.02, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_rewarm_check(None, 0, 0, 4.0, 0.02, None) == 0


def test_rule_matches_oracle_on_random_histories():
    rng = np.random.default_rng(3)
    for _ in range(300):
        n_chunks = int(rng.integers(2, 7))
        layers = list(range(int(rng.integers(1, 6))))
        hist = []
        for _ in range(n_chunks):
            present = [l for l in layers if rng.random() < 0.9]
            # live errors come from float32 device buffers
            hist.append({l: float(np.float32(np.exp(rng.normal(-3.0, 2.0)))) for l in present})
        want = oracle.rewarm_trigger(hist[:-1], hist[-1])
        assert _session_rule(hist) == want, hist


def test_kv_cache_accounting():
    from streaming_video_attention_b200.session import kv_cache_bytes
    # one frame of K and V at the 1.3B shape: 2 x 1560 tokens x 1536 x 2 bytes
    frame = 2 * 1560 * 1536 * 2
    assert kv_cache_bytes([0], 20, 3, 1, 1560, 1536) == 24 * frame          # sink + 20 history + chunk
    assert kv_cache_bytes([1], 20, 3, 1, 1560, 1536) == 4 * frame           # sink + chunk
    before = kv_cache_bytes([0] * 30, 20, 3, 1, 1560, 1536)
    after = kv_cache_bytes([1] * 15 + [0] * 15, 20, 3, 1, 1560, 1536)
    assert after == 15 * 24 * frame + 15 * 4 * frame
    assert abs((before - after) / before - 20 / 48) < 1e-12               # half the layers: 41.7 % removed
    # with a long history the removed share approaches the absorbed share of layers
    long_b = kv_cache_bytes([0] * 30, 119, 3, 1, 1560, 1536)
    long_a = kv_cache_bytes([1] * 15 + [0] * 15, 119, 3, 1, 1560, 1536)
    assert 0.48 < (long_b - long_a) / long_b < 0.5


def test_flush_stats_groups_consecutive_layers_with_equal_rows(monkeypatch):
    """Warmup calls only write operands; flush_stats() accumulates each run of consecutive
    layers in one call on contiguous operands; a call with another row count, or a second call
    for a pending layer, flushes first; transition() flushes before solving."""
    import torch
    from streaming_video_attention_b200 import ispa

    calls = []
    monkeypatch.setattr(ispa, "ispa_attn_split_ops", lambda desc, q, k, v, o, lse, a, r, *args, **kw:
                        calls.append(("ops", desc.n_q, a.shape, a.data_ptr())))
    monkeypatch.setattr(ispa, "ispa_accum_ops", lambda stats, a, r, n, code, stream=None:
                        calls.append(("accum", [id(s) for s in stats], tuple(a.shape), a.is_contiguous(), n)))
    monkeypatch.setattr(ispa, "alloc_workspace", lambda nbytes, device="cuda": None)   # no solve here
    monkeypatch.setattr(ispa, "ispa_stats_reset", lambda st, stream=None: None)
    sess = IspaSession(5, 2, 128, 1e-2, 2, "bf16", device="cpu")
    ids = [id(s) for s in sess.stats]

    def call(layer, n_q):
        q = torch.zeros((n_q, 2, 128), dtype=torch.bfloat16)
        kv = torch.zeros((300, 2, 128), dtype=torch.bfloat16)
        sess.full_attention(layer, q, kv, kv, (0, 50), (200, 300), None, None, collect=True)

    for layer, n in ((0, 10), (1, 10), (2, 10), (3, 8), (4, 10)):
        call(layer, n)
    assert [c[0] for c in calls] == ["ops", "ops", "ops", "accum", "ops", "accum", "ops"]
    assert calls[3][1:] == (ids[0:3], (3, 10, 256), True, 10)
    assert calls[5][1:] == (ids[3:4], (1, 8, 256), True, 8)
    # slots of one row count are packed: layer l at l * n * D elements
    base = calls[0][3]
    assert [c[3] - base for c in calls[:3]] == [0, 10 * 256 * 2, 2 * 10 * 256 * 2]
    calls.clear()
    sess.flush_stats()
    assert calls == [("accum", ids[4:5], (1, 10, 256), True, 10)]
    calls.clear()
    sess.flush_stats()                                   # nothing pending: no call
    assert calls == []
    call(2, 10)
    call(2, 10)                                          # the same layer again: flush in between
    assert [c[0] for c in calls] == ["ops", "accum", "ops"]
    assert calls[1][1] == ids[2:3]
    sess.rewarm()                                        # pending operands are dropped
    calls.clear()
    sess.flush_stats()
    assert calls == []
