"""Float64 CPU oracle of decode-time KV compression with a state cache.

TEST INFRASTRUCTURE, like ``csa_oracle``: only the tests may import or run it; the
product never calls it and shares no code with it.

Sources (cited by page title and section):
  [P1] 【论文解读】DeepSeek-V4 (wkq9411.github.io):
       二、基础设施 (六) 推理框架 -- two kinds of KV cache: a state cache for the sliding
         window and for the uncompressed tail tokens of CSA/HCA that do not yet fill a
         compression block, and a classical cache of finished compressed entries whose
         blocks cover a multiple of lcm(m, m') raw tokens;
       一、模型架构 (三) 1(1) and 2(1) -- the compression of one block (overlapped for CSA,
         plain for HCA); 3(1), 3(2) -- RMSNorm and RoPE of each finished entry;
         3(3) -- the n_win most recent uncompressed tokens.
  [P4] DeepseekV4论文解析 (blog.chaseai.de), 2. Hybrid Attention：CSA + HCA, 从注意力公式到
       可部署系统 -- the five kinds of per-request state, the fixed-size state cache for
       the window and the unfinished tail, paged cache for finished entries, and
       lcm(4, 128) = 128 raw tokens = 32 CSA entries = 1 HCA entry per logical block.

Readings where the pages leave the mechanics open:
  S1  A CSA entry i needs the a-rows of block i and the b-rows of block i-1, so the
      state holds the current block's incoming (C^a, Z^a, C^b, Z^b) rows and the last
      finished block's (C^b, Z^b) rows. Entry i is compressed, normalised and rotated at
      position m*i the moment token m*(i+1)-1 arrives (the same arithmetic as a whole
      prefill), and the finished block's b-rows replace the held ones.
  S2  HCA holds the current block's (C, Z) rows; entry i is made when token
      m'*(i+1)-1 arrives.
  S3  The window is a ring of n_win rows: the row of position p lives in slot p mod n_win
      and is given in its final (normed, rotated) form.
  S4  Finished entries live in pages of one logical block (128 raw tokens): 32 CSA entries
      or 1 HCA entry. A request takes a page from a shared pool when its first entry of
      a new block is written, and a page table maps its logical pages to physical ones.
  S5  The compressed indexer keys are extended the same way, without RMSNorm / RoPE (the
      pages attach those to the attention's queries and KV entries only): finalize=False.
"""
from __future__ import annotations

import math
from typing import List, Optional

import numpy as np

from . import csa_oracle as O


class PagePool:
    """Physical pages of finished entries shared by all requests of one layer: ``rows``
    entries of ``c`` values each. Free pages are handed out in the order of ``order``
    (any permutation), so that logical and physical order differ."""

    def __init__(self, n_pages: int, rows: int, c: int, order=None):
        self.data = np.full((n_pages, rows, c), np.nan)
        self.free: List[int] = list(order) if order is not None else list(range(n_pages))
        assert sorted(self.free) == list(range(n_pages))
        self.rows = rows

    def take(self) -> int:
        if not self.free:
            raise MemoryError("page pool exhausted")
        return self.free.pop(0)

    def give_back(self, pages) -> None:
        self.free.extend(pages)


class _Request:
    """Page table, window ring and token count common to both layer kinds."""

    def __init__(self, pool: PagePool, m: int, c: int, n_win: int, block_tokens: int):
        assert block_tokens % m == 0 and block_tokens // m == pool.rows
        self.pool, self.m, self.c, self.n_win = pool, m, c, n_win
        self.block_tokens = block_tokens
        self.page_table: List[int] = []
        self.n_tok = 0
        self.n_entries = 0
        self.ring = np.full((max(n_win, 1), c), np.nan)

    # window ring (S3)
    def _push_window(self, row, pos: int) -> None:
        if self.n_win > 0:
            self.ring[pos % self.n_win] = np.asarray(row, np.float64)

    def window_rows(self, t: int) -> np.ndarray:
        """Rows of positions max(t-n_win+1, 0) .. t, oldest first; t must be the last
        appended position."""
        assert t == self.n_tok - 1
        pos = O.window_positions(t, self.n_win, max(t - self.n_win + 1, 0), self.n_win)
        return self.ring[pos % self.n_win]

    # paged entries (S4)
    def _write_entry(self, row) -> None:
        i = self.n_entries
        page, slot = divmod(i, self.pool.rows)
        if page == len(self.page_table):
            self.page_table.append(self.pool.take())
        self.pool.data[self.page_table[page], slot] = row
        self.n_entries += 1

    def entries(self) -> np.ndarray:
        """Finished entries in logical order, read through the page table."""
        out = np.empty((self.n_entries, self.c))
        for i in range(self.n_entries):
            page, slot = divmod(i, self.pool.rows)
            out[i] = self.pool.data[self.page_table[page], slot]
        return out

    def release(self) -> None:
        self.pool.give_back(self.page_table)
        self.page_table = []


class CsaState(_Request):
    """One request's CSA state cache (S1) and its pages of finished entries."""

    def __init__(self, pool: PagePool, *, m: int, c: int, bias, n_win: int, r: int,
                 base: float, eps: float, gamma=None, block_tokens: int = 128,
                 finalize: bool = True):
        super().__init__(pool, m, c, n_win, block_tokens)
        bias = np.asarray(bias, np.float64)
        self.Ba, self.Bb = bias[:m], bias[m:2 * m]
        self.r, self.base, self.eps, self.gamma = r, base, eps, gamma
        self.finalize = finalize
        self.cur = {k: [] for k in ("Ca", "Za", "Cb", "Zb")}  # rows of the open block
        self.prev_Cb: Optional[np.ndarray] = None  # b-rows of the last finished block
        self.prev_Zb: Optional[np.ndarray] = None

    def held_rows(self) -> int:
        """Raw token rows the state cache holds for compression (the open block's four
        tensors count once per token, the last finished block's b-rows once each)."""
        return len(self.cur["Ca"]) + (0 if self.prev_Cb is None else self.m)

    def append(self, ca, cb, za, zb, win_row) -> Optional[int]:
        """Token at position n_tok arrives; returns the index of the entry it finishes."""
        t = self.n_tok
        for k, v in (("Ca", ca), ("Za", za), ("Cb", cb), ("Zb", zb)):
            self.cur[k].append(np.asarray(v, np.float64))
        self._push_window(win_row, t)
        self.n_tok += 1
        if self.n_tok % self.m:
            return None
        i = t // self.m
        self._write_entry(self._finish_block(i))
        self.prev_Cb, self.prev_Zb = np.stack(self.cur["Cb"]), np.stack(self.cur["Zb"])
        self.cur = {k: [] for k in self.cur}
        return i

    def _b_branch(self):
        """(b-logits, b-values) of the open block: the last finished block's b-rows, or
        -inf logits and zero values at a sequence start [P1 1(1)]."""
        if self.prev_Zb is None:
            return np.full((self.m, self.c), -np.inf), np.zeros((self.m, self.c))
        return self.prev_Zb + self.Bb, self.prev_Cb

    def _finish_block(self, i: int) -> np.ndarray:
        """Entry i from the open block's a-rows and the b-branch, then RMSNorm and RoPE at
        its position (S1)."""
        ca_blk = np.stack(self.cur["Ca"])
        za_l = np.stack(self.cur["Za"]) + self.Ba
        zb_l, cb_blk = self._b_branch()
        S = O._softmax_rows(np.concatenate([za_l, zb_l], axis=0))
        entry = (S[:self.m] * ca_blk).sum(axis=0) + (S[self.m:] * cb_blk).sum(axis=0)
        return self._finalize(entry, i)

    def _finalize(self, entry, i: int) -> np.ndarray:
        if not self.finalize:  # indexer keys (S5)
            return entry
        return O.finalize_entries(entry[None], i, self.m, self.r, self.base, self.eps,
                                  self.gamma)[0]

    def resume(self, Ca, Cb, Za, Zb, entries, win_rows) -> None:
        """Take over a request after a prefill of n0 = len(Ca) tokens that wrote
        ``entries`` (its floor(n0/m) finished entries) through the whole-chunk path: the
        entries go to pages, the open block's rows and the last finished block's b-rows
        to the state, and the last min(n0, n_win) window rows to the ring."""
        assert self.n_tok == 0 and self.n_entries == 0
        Ca, Cb, Za, Zb = (np.asarray(x, np.float64) for x in (Ca, Cb, Za, Zb))
        n0 = Ca.shape[0]
        nb = n0 // self.m
        assert len(entries) == nb
        for row in entries:
            self._write_entry(np.asarray(row, np.float64))
        if nb > 0:
            lo = self.m * (nb - 1)
            self.prev_Cb, self.prev_Zb = Cb[lo:lo + self.m].copy(), Zb[lo:lo + self.m].copy()
        tail = slice(self.m * nb, n0)
        self.cur = {"Ca": list(Ca[tail]), "Za": list(Za[tail]), "Cb": list(Cb[tail]),
                    "Zb": list(Zb[tail])}
        win_rows = np.asarray(win_rows, np.float64)
        for p in range(max(n0 - self.n_win, 0), n0):
            self._push_window(win_rows[p], p)
        self.n_tok = n0


class HcaState(_Request):
    """One request's HCA state cache (S2) and its pages of finished entries."""

    def __init__(self, pool: PagePool, *, m: int, c: int, bias, n_win: int, r: int,
                 base: float, eps: float, gamma=None, block_tokens: int = 128,
                 finalize: bool = True):
        super().__init__(pool, m, c, n_win, block_tokens)
        self.B = np.asarray(bias, np.float64)
        self.r, self.base, self.eps, self.gamma = r, base, eps, gamma
        self.finalize = finalize
        self.cur_C: List[np.ndarray] = []
        self.cur_Z: List[np.ndarray] = []

    def held_rows(self) -> int:
        return len(self.cur_C)

    def append(self, cv, zv, win_row) -> Optional[int]:
        """Token at position n_tok arrives; returns the index of the entry it finishes."""
        t = self.n_tok
        self.cur_C.append(np.asarray(cv, np.float64))
        self.cur_Z.append(np.asarray(zv, np.float64))
        self._push_window(win_row, t)
        self.n_tok += 1
        if self.n_tok % self.m:
            return None
        i = t // self.m
        S = O._softmax_rows(np.stack(self.cur_Z) + self.B)
        entry = (S * np.stack(self.cur_C)).sum(axis=0)
        if self.finalize:
            entry = O.finalize_entries(entry[None], i, self.m, self.r, self.base, self.eps,
                                       self.gamma)[0]
        self._write_entry(entry)
        self.cur_C, self.cur_Z = [], []
        return i


def _hca_resume(self, C, Z, entries, win_rows) -> None:
    """Take over a request after a prefill of n0 = len(C) tokens that wrote ``entries``
    (its floor(n0/m') finished entries): entries to pages, the open block's rows to the
    state, the last min(n0, n_win) window rows to the ring."""
    assert self.n_tok == 0 and self.n_entries == 0
    C, Z = np.asarray(C, np.float64), np.asarray(Z, np.float64)
    n0 = C.shape[0]
    nb = n0 // self.m
    assert len(entries) == nb
    for row in entries:
        self._write_entry(np.asarray(row, np.float64))
    self.cur_C, self.cur_Z = list(C[self.m * nb:n0]), list(Z[self.m * nb:n0])
    win_rows = np.asarray(win_rows, np.float64)
    for p in range(max(n0 - self.n_win, 0), n0):
        self._push_window(win_rows[p], p)
    self.n_tok = n0


HcaState.resume = _hca_resume


def block_tokens(m_csa: int, m_hca: int) -> int:
    """Raw tokens covered by one logical cache block: lcm(m, m') [P1 二(六)]."""
    return math.lcm(m_csa, m_hca)
