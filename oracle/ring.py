"""Integer model of the checkpoint + input-buffer bookkeeping -- TEST INFRASTRUCTURE.

The ReplaySSM reports represent a layer's state as a checkpoint plus a buffer of
the recent inputs; outputs are computed from both without writing state, and
the checkpoint is rewritten only when the buffer is full ("Tenir le journal
plutot que le solde", blog.thibaultmonteiro.fr; "Reshenie ReplaySSM",
aikraft.ru: the checkpoint is stored once per window).  Speculative drafts are
appended to the buffer and a rejection only moves the buffer pointer, never
touching the checkpoint ("Un retour en arriere qui devient trivial",
irisproject.cloud).

Readings of what the pages leave open:
* counters per sequence: ``seq_pos`` = committed tokens, ``ckpt_pos`` = tokens
  folded into the checkpoint, ``len = seq_pos - ckpt_pos`` in [0, W];
* lazy flush: before appending n tokens, fold the committed entries if
  len + n > W (so plain decode folds exactly W entries at steps W, 2W, ...);
  ``flush`` folds whatever is committed (if len > 0);
* ring of R = W + max(max_draft, 1) slots, token n lives in slot n mod R; the
  extra slots keep the entries being folded apart from the ones being appended
  in the same call;
* verify(K): optional flush, then drafts seq_pos .. seq_pos+K-1 are appended
  uncommitted and ``pending = K``; commit(a): 0 <= a <= pending moves
  ``seq_pos += a`` and clears ``pending``; an out-of-range a is recorded as an
  error, treated as a = 0 (nothing accepted) and still clears ``pending``;
* eager mode keeps no buffer: the state is always current (ckpt_pos = seq_pos)
  and flush_count stays 0.
"""
from __future__ import annotations

import numpy as np


class MisuseError(Exception):
    """Host-detectable misuse (the C-ABI returns RSSM_ESTATE / RSSM_EINVAL for it)."""


class RingModel:
    def __init__(self, batch: int, window: int, max_draft: int = 1, mode: str = "replay"):
        if window < 1 or max_draft < 0 or batch < 1:
            raise MisuseError("bad sizes")
        self.batch, self.W, self.max_draft, self.mode = batch, window, max_draft, mode
        self.R = window + max(max_draft, 1)
        self.seq_pos = np.zeros(batch, np.int64)
        self.ckpt_pos = np.zeros(batch, np.int64)
        self.pending = np.zeros(batch, np.int32)
        self.flush_count = np.zeros(batch, np.int32)
        self.host_pending = 0
        self.log = []  # (op, flushed mask, slots written [B, n])

    def slot(self, n):
        return np.asarray(n) % self.R

    @property
    def length(self) -> np.ndarray:
        return self.seq_pos - self.ckpt_pos

    def _flush_mask(self, n_new: int) -> np.ndarray:
        if self.mode != "replay":
            return np.zeros(self.batch, bool)
        return self.length + n_new > self.W

    def _fold(self, mask: np.ndarray):
        self.ckpt_pos[mask] = self.seq_pos[mask]
        self.flush_count[mask] += 1

    def decode(self):
        if self.host_pending:
            raise MisuseError("decode while a verify is pending")
        mask = self._flush_mask(1)
        self._fold(mask)
        slots = self.slot(self.seq_pos)[:, None]
        self.seq_pos += 1
        if self.mode != "replay":
            self.ckpt_pos[:] = self.seq_pos
        self.log.append(("decode", mask.copy(), slots))
        return mask, slots

    def verify(self, K: int):
        if self.host_pending:
            raise MisuseError("verify while a verify is pending")
        if not (1 <= K <= self.max_draft and K <= self.W):
            raise MisuseError("K out of range")
        mask = self._flush_mask(K)
        self._fold(mask)
        slots = self.slot(self.seq_pos[:, None] + np.arange(K)[None, :])
        self.pending[:] = K
        self.host_pending = K
        self.log.append(("verify", mask.copy(), slots))
        return mask, slots

    def commit(self, accept) -> np.ndarray:
        if not self.host_pending:
            raise MisuseError("commit with nothing pending")
        a = np.asarray(accept, np.int64)
        bad = (a < 0) | (a > self.pending)
        a = np.where(bad, 0, a)
        self.seq_pos += a
        if self.mode != "replay":
            self.ckpt_pos[:] = self.seq_pos
        self.pending[:] = 0
        self.host_pending = 0
        self.log.append(("commit", bad.copy(), None))
        return bad

    def flush(self):
        if self.host_pending:
            raise MisuseError("flush while a verify is pending")
        mask = (self.length > 0) if self.mode == "replay" else np.zeros(self.batch, bool)
        self._fold(mask)
        self.log.append(("flush", mask.copy(), None))
        return mask

    def live_entries(self, b: int):
        """Absolute token indices whose inputs must be in the buffer of sequence b:
        committed-but-unfolded ones and pending drafts."""
        return list(range(int(self.ckpt_pos[b]), int(self.seq_pos[b] + self.pending[b])))
