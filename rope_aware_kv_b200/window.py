"""Windowed streaming driver: keep a KV cache pruned while tokens are generated.

Generated tokens are appended to the cache in windows; whenever the cache
reaches B + window rows per unit it is pruned back to the B best-scored rows
(hyper.ai summary of TriAttention, Method section: the cache is pruned every
128 generated tokens, all units of all layers in one batched step).  Kept rows
stay in temporal order (jaedaily.cn tutorial, eviction step).

The driver only sequences library calls: ``tri_append`` for each window, then
``tri_prune`` into the other of two cache buffers (ping-pong) or
``tri_prune_inplace`` on the single buffer.  Every unit of the batch holds the
same number of rows at all times (each append adds the same number of rows to
every unit, each prune keeps min(B, rows)), so that count is tracked on the
host and no device value is read back between steps.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (HEAD_DIM, TriConfig, config, tri_append, tri_prune, tri_prune_inplace,
               tri_prune_workspace_bytes, workspace)


class WindowDriver:
    """Cache buffers, counts and workspace of one streaming batch.

    Units are ordered ``(seq * n_layers + layer) * n_kvheads + kvhead``, as in
    every library call; ``stats`` are the calibration statistics
    ``[n_layers][n_kvheads * G][64][4]``.  ``cap = B + window`` rows per unit.
    """

    def __init__(self, n_seq: int, n_layers: int, n_kvheads: int, G: int, B: int,
                 stats: torch.Tensor, window: int = 128, dtype=torch.bfloat16,
                 device=None, cfg: Optional[TriConfig] = None, inplace: bool = False,
                 values: bool = True):
        if B < 1 or window < 1:
            raise ValueError("B and window must be positive")
        device = torch.device(device) if device is not None else stats.device
        self.n_seq, self.n_layers, self.n_kvheads, self.G = n_seq, n_layers, n_kvheads, G
        self.B, self.window, self.cap = B, window, B + window
        self.U = n_seq * n_layers * n_kvheads
        self.stats = stats
        self.cfg = cfg if cfg is not None else config()
        self.inplace = inplace
        n_buf = 1 if inplace else 2
        shape = (self.U, self.cap, HEAD_DIM)
        self.k = [torch.zeros(shape, dtype=dtype, device=device) for _ in range(n_buf)]
        self.v = [torch.zeros(shape, dtype=dtype, device=device) if values else None
                  for _ in range(n_buf)]
        self.pos = [torch.full((self.U, self.cap), -1, dtype=torch.int32, device=device)
                    for _ in range(n_buf)]
        # Two count arrays: a prune reads one and writes the other.
        self.nv = [torch.zeros((self.U,), dtype=torch.int32, device=device) for _ in range(2)]
        self.p_cur = torch.zeros((n_seq,), dtype=torch.int64, device=device)
        self.kept = torch.empty((self.U, B), dtype=torch.int32, device=device)
        self.ws = workspace(tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, self.cap, B),
                            device)
        self.buf = 0       # cache buffer holding the current rows
        self.cnt = 0       # count array holding n_valid
        self.rows = 0      # rows per unit (host copy of n_valid)
        self.tokens = 0    # tokens appended so far
        self.prunes = 0

    def reset(self):
        """Empty the cache (counts and current positions back to zero)."""
        for t in self.nv:
            t.zero_()
        self.p_cur.zero_()
        self.buf = self.cnt = self.rows = self.tokens = self.prunes = 0

    # -- current cache -----------------------------------------------------
    @property
    def k_cache(self) -> torch.Tensor:
        return self.k[self.buf]

    @property
    def v_cache(self) -> Optional[torch.Tensor]:
        return self.v[self.buf]

    @property
    def pos_cache(self) -> torch.Tensor:
        return self.pos[self.buf]

    @property
    def n_valid(self) -> torch.Tensor:
        return self.nv[self.cnt]

    @property
    def full(self) -> bool:
        """The cache holds B + window rows: the next step is a prune."""
        return self.rows >= self.cap

    # -- steps -------------------------------------------------------------
    def append(self, k_new: torch.Tensor, v_new: Optional[torch.Tensor],
               pos_new: torch.Tensor, auto_prune: bool = True, stream=None) -> bool:
        """Append n new rows per unit ([U][n][128] keys and values, [U][n]
        positions); prune once the cache is full.  Returns whether it pruned."""
        n = k_new.shape[1]
        if self.rows + n > self.cap:
            raise ValueError(f"{n} new rows overflow the cache ({self.rows} of {self.cap} held)")
        tri_append(self.k_cache, self.v_cache, self.pos_cache, self.n_seq, self.n_valid, k_new,
                   v_new if self.v_cache is not None else None, pos_new, p_cur=self.p_cur,
                   ws=self.ws, stream=stream)
        self.rows += n
        self.tokens += n
        if auto_prune and self.full:
            self.prune(stream=stream)
            return True
        return False

    def prune(self, final: Optional[torch.Tensor] = None, stream=None):
        """Prune every unit back to min(B, rows) rows (the kept indices are
        left in ``self.kept``, the final scores in ``final`` if given)."""
        src_cnt, dst_cnt = self.cnt, 1 - self.cnt
        if self.inplace:
            tri_prune_inplace(self.cfg, self.k[0], self.v[0], self.pos[0], self.n_seq,
                              self.n_layers, self.n_kvheads, self.G, self.p_cur, self.stats,
                              self.B, self.nv[dst_cnt], n_valid=self.nv[src_cnt],
                              kept=self.kept, ws=self.ws, stream=stream, final=final)
        else:
            a, b = self.buf, 1 - self.buf
            tri_prune(self.cfg, self.k[a], self.v[a], self.pos[a], self.n_seq, self.n_layers,
                      self.n_kvheads, self.G, self.p_cur, self.stats, self.B, self.k[b], self.v[b],
                      self.pos[b], self.nv[dst_cnt], n_valid=self.nv[src_cnt], kept=self.kept,
                      ws=self.ws, stream=stream, final=final)
            self.buf = b
        self.cnt = dst_cnt
        self.rows = min(self.B, self.rows)
        self.prunes += 1
