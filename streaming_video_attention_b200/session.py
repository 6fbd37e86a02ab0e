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
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import ispa


class IspaSession:
    def __init__(self, layers: int, heads: int, head_dim: int, lam: float, K: int, dtype: str = "bf16",
                 device: str = "cuda"):
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

    # ---------------------------------------------------------------- state
    def set_weights(self, W: Sequence[torch.Tensor]) -> None:
        """Original output projections, [D_in, D_out] device tensors of the session dtype."""
        assert len(W) == self.layers
        self.W0 = list(W)

    def rewarm(self, stream=None) -> None:
        """Enter (or re-enter) the dual-stream warmup: every layer F, statistics zeroed."""
        for st in self.stats:
            ispa.ispa_stats_reset(st, stream)
        self.is_local = [0] * self.layers
        self.idx = []

    def weight(self, layer: int) -> torch.Tensor:
        return self.W_new[layer] if self.is_local[layer] else self.W0[layer]

    def _attn_ws(self, desc) -> torch.Tensor:
        need = ispa.workspace_bytes(desc, 0, 0)
        if self._ws_attn is None or self._ws_attn.numel() < need:
            self._ws_attn = ispa.alloc_workspace(need, self.device)
        return self._ws_attn

    def reserve(self, max_n_q: int) -> None:
        """Size the attention workspace up front (no allocation inside a timed loop)."""
        d = ispa.make_desc(max_n_q, 1, self.heads, self.head_dim, dtype=self.code)
        self._attn_ws(d)

    # ---------------------------------------------------------------- per-layer calls
    def full_attention(self, layer: int, q, k, v, sink: Tuple[int, int], chunk: Tuple[int, int], o, lse,
                       collect: bool, o_loc=None, lse_loc=None, o_hist=None, lse_hist=None, stream=None) -> None:
        """An F-layer call; with collect=True (warmup) the ridge statistics accumulate too."""
        n_q, n_kv = q.shape[0], k.shape[0]
        desc = ispa.make_desc(n_q, n_kv, self.heads, self.head_dim, sink, chunk, dtype=self.code)
        ws = self._attn_ws(desc) if collect else None
        ispa.ispa_attn_split(desc, q, k, v, o, lse, o_loc, lse_loc, o_hist, lse_hist,
                             stats=self.stats[layer] if collect else None, ws=ws, stream=stream)

    def local_attention(self, layer: int, q, k_loc, v_loc, o, lse=None, y=None, stream=None) -> None:
        """An L-layer call: sink + chunk rows only; y = O W_new when y is given."""
        n_q, n_kv = q.shape[0], k_loc.shape[0]
        desc = ispa.make_desc(n_q, n_kv, self.heads, self.head_dim, dtype=self.code)
        w = self.W_new[layer] if y is not None else None
        ws = self._attn_ws(desc) if lse is None else None
        ispa.ispa_local_attn(desc, q, k_loc, v_loc, o, lse, w, y, ws=ws, stream=stream)

    # ---------------------------------------------------------------- the switch
    def transition(self, K: Optional[int] = None, stream=None) -> List[int]:
        """Layer Absorb + Dynamic Layer Selection. Synchronises `stream` to read the errors."""
        K = self.K if K is None else K
        ispa.ispa_solve_absorb(self.stats, self.W0, self.code, self.lam, self.dW, self.eps, self.err_terms,
                               self.W_new, self.status, self.ws_solve, stream)
        eps = self.eps.to("cpu", non_blocking=False).tolist()
        status = self.status.to("cpu").tolist()
        self.eps_host = eps
        self.idx, flags = ispa.ispa_select_layers(eps, K)
        self.is_local = [int(f) for f in flags]
        self.transitions += 1
        if any(s != ispa.ISPA_OK for s in status):
            bad = [l for l, s in enumerate(status) if s != ispa.ISPA_OK]
            raise ispa.IspaError(ispa.ISPA_ERR_NOT_SPD, "transition", f"G + lambda I not SPD in layers {bad}")
        return list(self.idx)

    def selection_margin(self) -> Optional[float]:
        """(eps_(K+1) - eps_(K)) / eps_(K) of the last transition: how decisive the cut was."""
        if not self.eps_host or self.K <= 0 or self.K >= self.layers:
            return None
        s = sorted(self.eps_host)
        a, b = s[self.K - 1], s[self.K]
        return (b - a) / a if a > 0 else None
