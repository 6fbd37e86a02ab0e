"""Streaming ISPA driver: the per-layer state machine around the C-ABI calls.

[ISPA §3.1 Overall Framework] Dual-stream warmup (every layer is an F-layer and collects
statistics) -> Layer Absorb at the end of the warmup (solve, error, selection of the K
layers with the lowest error, W_new = W + dW) -> memory-efficient inference (L-layers
attend to the sink + chunk rows only and project with W_new; F-layers keep full
attention). [ISPA §3.1 last paragraph, §3.3 last paragraph] On a scene change the same
procedure is re-entered: rewarm() restores every layer to an F-layer with its original
weights and zeroes the statistics; the next transition replaces the old dW.

The session owns the statistics buffers, dW, the error vector and the updated weights; the
caller owns the KV cache (evicting the history of an L-layer is the caller freeing it).

Statistics of a warmup chunk: each layer's full_attention(collect=True) writes its operands
(A_loc, R) into the layer's slot of one buffer of layers x n_q x D elements (slots packed for
the chunk's row count, so a run of layers is one contiguous operand), and flush_stats() (called by
the caller after the chunk's last layer, and by transition()) accumulates every pending layer
in one launch -- the same sums, bit for bit, as accumulating layer by layer, without a short
final wave per layer. batch_stats=False accumulates inside each call instead.

Re-warmup trigger (the pages leave it open; reading): after a transition the F-layers still
see their history, so full_attention(..., monitor=True) accumulates one chunk's statistics
and live_errors() evaluates the error of the dW solved at the transition on them
(ispa_absorb_error). rewarm_layers() names the monitored layers whose live error rose above
both RATIO x and MIN_RISE + the lowest live error they showed since the transition -- a
scene change that the absorbed projection no longer reconstructs. The reference is the live
minimum rather than the selection's eps, which is in-sample: where the residual is not
predictable (i.i.d. layers) dW overfits the warmup and every fresh chunk sits far above it.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import ispa


def kv_cache_bytes(is_local: Sequence[int], history_frames: int, chunk_frames: int, sink_frames: int,
                   tokens_per_frame: int, D: int, elem_bytes: int = 2) -> int:
    """Bytes of K and V held across the layers [ISPA §3.1 step 3: an L-layer keeps only the sink
    and the current chunk, its history is evicted; an F-layer keeps the sink, its recent history
    frames and the chunk]. history_frames counts the frames an F-layer holds besides the sink and
    the chunk."""
    per_frame = 2 * tokens_per_frame * D * elem_bytes
    total = 0
    for loc in is_local:
        frames = sink_frames + chunk_frames + (0 if loc else history_frames)
        total += frames * per_frame
    return total


class IspaSession:
    RATIO = 4.0        # live error above RATIO x its minimum since the transition ...
    MIN_RISE = 0.02    # ... and above that minimum + MIN_RISE

    def __init__(self, layers: int, heads: int, head_dim: int, lam: float, K: int, dtype: str = "bf16",
                 device: str = "cuda", w8a8: bool = False, batch_stats: bool = True):
        self.layers, self.heads, self.head_dim = layers, heads, head_dim
        self.D = heads * head_dim
        self.lam, self.K = float(lam), int(K)
        self.dtype = dtype
        self.code = ispa.ISPA_BF16 if dtype == "bf16" else ispa.ISPA_FP32
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.device = device
        self.stats = [ispa.Stats(self.D, device) for _ in range(layers)]
        self.W0: List[Optional[torch.Tensor]] = [None] * layers
        self.W_new = [torch.empty(self.D, self.D, dtype=self.tdtype, device=device) for _ in range(layers)]
        self.dW = torch.empty(layers, self.D, self.D, dtype=torch.float32, device=device)
        self.eps = torch.empty(layers, dtype=torch.float32, device=device)
        self.err_terms = torch.empty(layers, 2, dtype=torch.float64, device=device)
        self.status = torch.zeros(layers, dtype=torch.int32, device=device)
        self.ws_solve = ispa.alloc_workspace(ispa.workspace_bytes(None, layers, self.D), device)
        self._ws_attn: Optional[torch.Tensor] = None
        self.is_local = [0] * layers
        self.idx: List[int] = []
        self.eps_host: List[float] = []
        self.transitions = 0
        # W8A8 projection of the L-layers (int8 codes of W_new, transposed, and column scales)
        self.w8a8 = bool(w8a8) and dtype == "bf16"
        self.wq: List[Optional[torch.Tensor]] = [None] * layers
        self.wq_scale: List[Optional[torch.Tensor]] = [None] * layers
        self.monitor: List[Optional[ispa.Stats]] = [None] * layers
        self.live_history: List[Dict[int, float]] = []
        self._eps_live = torch.empty(layers, dtype=torch.float32, device=device)
        # warmup statistics operands awaiting flush_stats(): layer -> rows
        self.batch_stats = bool(batch_stats)
        self._ops: Optional[Tuple[torch.Tensor, torch.Tensor]] = None
        self._pending: Dict[int, int] = {}

    # ---------------------------------------------------------------- state
    def set_weights(self, W: Sequence[torch.Tensor]) -> None:
        """Original output projections, [D_in, D_out] device tensors of the session dtype."""
        assert len(W) == self.layers
        self.W0 = list(W)

    def rewarm(self, stream=None) -> None:
        """Enter (or re-enter) the dual-stream warmup: every layer F, statistics zeroed."""
        self._pending = {}
        for st in self.stats:
            ispa.ispa_stats_reset(st, stream)
        self.is_local = [0] * self.layers
        self.idx = []
        self._reset_monitor(stream)

    def _reset_monitor(self, stream=None) -> None:
        for st in self.monitor:
            if st is not None:
                ispa.ispa_stats_reset(st, stream)
        self.live_history = []

    def weight(self, layer: int) -> torch.Tensor:
        return self.W_new[layer] if self.is_local[layer] else self.W0[layer]

    def _attn_ws(self, desc) -> torch.Tensor:
        need = ispa.workspace_bytes(desc, 0, 0)
        if self._ws_attn is None or self._ws_attn.numel() < need:
            self._ws_attn = ispa.alloc_workspace(need, self.device)
        return self._ws_attn

    def reserve(self, max_n_q: int) -> None:
        """Size the attention workspace and the statistics operand buffer up front (no
        allocation inside a timed loop)."""
        d = ispa.make_desc(max_n_q, 1, self.heads, self.head_dim, dtype=self.code)
        self._attn_ws(d)
        if self.batch_stats:
            self._ops_buffers(max_n_q)

    def _ops_buffers(self, n_q: int) -> Tuple[torch.Tensor, torch.Tensor]:
        """Flat operand buffers for layers x n_q rows: layer l of a chunk with n rows per layer
        sits at [l * n * D, (l + 1) * n * D), so consecutive layers are contiguous for any n."""
        need = self.layers * n_q * self.D
        if self._ops is None or self._ops[0].numel() < need:
            self._ops = (torch.empty(need, dtype=self.tdtype, device=self.device),
                         torch.empty(need, dtype=self.tdtype, device=self.device))
        return self._ops

    def _ops_slot(self, layer: int, n: int) -> Tuple[torch.Tensor, torch.Tensor]:
        a_all, r_all = self._ops_buffers(n)
        lo, hi = layer * n * self.D, (layer + 1) * n * self.D
        return a_all[lo:hi].view(n, self.D), r_all[lo:hi].view(n, self.D)

    def flush_stats(self, stream=None) -> None:
        """Accumulate the pending warmup operands: one launch per run of consecutive layers (all
        pending layers share one row count)."""
        if not self._pending:
            return
        a_all, r_all = self._ops
        layers = sorted(self._pending)
        n = self._pending[layers[0]]
        start = 0
        while start < len(layers):
            end = start + 1
            while end < len(layers) and layers[end] == layers[end - 1] + 1:
                end += 1
            l0, l1 = layers[start], layers[end - 1] + 1
            lo, hi = l0 * n * self.D, l1 * n * self.D
            ispa.ispa_accum_ops(self.stats[l0:l1], a_all[lo:hi].view(l1 - l0, n, self.D),
                                r_all[lo:hi].view(l1 - l0, n, self.D), n, self.code, stream)
            start = end
        self._pending = {}

    # ---------------------------------------------------------------- per-layer calls
    def full_attention(self, layer: int, q, k, v, sink: Tuple[int, int], chunk: Tuple[int, int], o, lse,
                       collect: bool, o_loc=None, lse_loc=None, o_hist=None, lse_hist=None, stream=None,
                       monitor: bool = False) -> None:
        """An F-layer call; with collect=True (warmup) the call's statistics operands are kept for
        flush_stats() (batch_stats=True) or accumulated at once (batch_stats=False); with
        monitor=True (after a transition) this chunk's statistics go to the layer's monitor."""
        n_q, n_kv = q.shape[0], k.shape[0]
        desc = ispa.make_desc(n_q, n_kv, self.heads, self.head_dim, sink, chunk, dtype=self.code)
        st = None
        if collect:
            st = self.stats[layer]
        elif monitor:
            if self.monitor[layer] is None:
                self.monitor[layer] = ispa.Stats(self.D, self.device)
            st = self.monitor[layer]
        if collect and self.batch_stats:
            if layer in self._pending or (self._pending and next(iter(self._pending.values())) != n_q):
                self.flush_stats(stream)   # a second call for the layer, or another row count, before a flush
            a_op, r_op = self._ops_slot(layer, n_q)
            ispa.ispa_attn_split_ops(desc, q, k, v, o, lse, a_op, r_op, o_loc, lse_loc, o_hist,
                                     lse_hist, stream=stream)
            self._pending[layer] = n_q
            return
        ws = self._attn_ws(desc) if st is not None else None
        ispa.ispa_attn_split(desc, q, k, v, o, lse, o_loc, lse_loc, o_hist, lse_hist, stats=st, ws=ws, stream=stream)

    def local_attention(self, layer: int, q, k_loc, v_loc, o, lse=None, y=None, stream=None) -> None:
        """An L-layer call: sink + chunk rows only; y = O W_new when y is given (through the
        int8 W8A8 path when the session was created with w8a8=True)."""
        n_q, n_kv = q.shape[0], k_loc.shape[0]
        desc = ispa.make_desc(n_q, n_kv, self.heads, self.head_dim, dtype=self.code)
        quant = self.w8a8 and y is not None
        w = self.W_new[layer] if (y is not None and not quant) else None
        ws = self._attn_ws(desc) if (lse is None or quant) else None
        ispa.ispa_local_attn(desc, q, k_loc, v_loc, o, lse, w, None if quant else y, ws=ws, stream=stream)
        if quant:
            ispa.ispa_project_w8a8(o, self.wq[layer], self.wq_scale[layer], y, ws=ws, stream=stream)

    # ---------------------------------------------------------------- the switch
    def transition(self, K: Optional[int] = None, stream=None) -> List[int]:
        """Layer Absorb + Dynamic Layer Selection. Synchronises `stream` to read the errors."""
        K = self.K if K is None else K
        self.flush_stats(stream)
        ispa.ispa_solve_absorb(self.stats, self.W0, self.code, self.lam, self.dW, self.eps, self.err_terms,
                               self.W_new, self.status, self.ws_solve, stream)
        eps = self.eps.to("cpu", non_blocking=False).tolist()
        status = self.status.to("cpu").tolist()
        self.eps_host = eps
        self.idx, flags = ispa.ispa_select_layers(eps, K)
        self.is_local = [int(f) for f in flags]
        self.transitions += 1
        self._reset_monitor(stream)
        if self.w8a8:
            for l in self.idx:
                if self.wq[l] is None:
                    self.wq[l] = torch.empty(self.D, self.D, dtype=torch.int8, device=self.device)
                    self.wq_scale[l] = torch.empty(self.D, dtype=torch.float32, device=self.device)
                ispa.ispa_quantize_w8(self.W_new[l], self.code, self.wq[l], self.wq_scale[l], stream)
        if any(s != ispa.ISPA_OK for s in status):
            bad = [l for l, s in enumerate(status) if s != ispa.ISPA_OK]
            raise ispa.IspaError(ispa.ISPA_ERR_NOT_SPD, "transition", f"G + lambda I not SPD in layers {bad}")
        return list(self.idx)

    # ---------------------------------------------------------------- re-warmup trigger
    def live_errors(self, stream=None) -> Dict[int, float]:
        """Error of the transition's dW on the statistics each monitored F-layer gathered since
        the last call; resets those statistics and records the result. Synchronises `stream`."""
        layers = [l for l in range(self.layers) if self.monitor[l] is not None and not self.is_local[l]]
        if not layers or self.transitions == 0:
            return {}
        ispa.ispa_absorb_error([self.monitor[l] for l in layers], [self.W0[l] for l in layers], self.code,
                               [self.dW[l] for l in layers], self._eps_live, ws=self.ws_solve, stream=stream)
        vals = self._eps_live[:len(layers)].to("cpu").tolist()
        for l in layers:
            ispa.ispa_stats_reset(self.monitor[l], stream)
        live = dict(zip(layers, vals))
        self.live_history.append(live)
        return live

    def rewarm_layers(self) -> List[int]:
        """Monitored layers whose latest live error left the range seen since the transition
        (the library's ispa_rewarm_check on the recorded live errors)."""
        if len(self.live_history) < 2:
            return []
        nan = float("nan")
        hist = [[d.get(l, nan) for l in range(self.layers)] for d in self.live_history]
        fired = ispa.ispa_rewarm_check(hist, self.RATIO, self.MIN_RISE)
        return [l for l in range(self.layers) if fired[l]]

    def selection_margin(self) -> Optional[float]:
        """(eps_(K+1) - eps_(K)) / eps_(K) of the last transition: how decisive the cut was."""
        if not self.eps_host or self.K <= 0 or self.K >= self.layers:
            return None
        s = sorted(self.eps_host)
        a, b = s[self.K - 1], s[self.K]
        return (b - a) / a if a > 0 else None
