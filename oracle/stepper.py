"""Oracle composition of the LSA decode step, tau cadence included.

TEST INFRASTRUCTURE, NOT THE PRODUCT (see the package docstring).

"FlashMemory-DeepSeek-V4 ... Lookahead Sparse Attention", gist.science technical
summary, section 2.1: every tau steps (Periodic Triggering, tau = 64) the memory
indexer scores every preceding compressed entry (Scoring Mechanism), every entry
with I >= 0.5 is fetched from the cold pool (Dynamic Fetching), and a
fine-grained top-k inside the fetched subset feeds core attention (Tiered
Selection).  Between refreshes the kept set stays fixed; each step re-ranks it
with that step's indexer query (the reading used for "fine-grained Top-k
selection within this restricted boundary").
"""
from __future__ import annotations

import numpy as np

from . import TAU, gather, index_score, index_score_list, local_to_global, select, sparse_attn, topk


class OracleDecoder:
    """Plain sequential driver over the oracle stages; holds the kept set between refreshes."""

    def __init__(self, wl, tau: int = TAU):
        self.wl = wl
        self.tau = tau
        self.kept_idx = None
        self.kept_off = None
        self.slot_of = None

    def refresh(self, q, w):
        wl = self.wl
        z, I = index_score(q, wl.q_dtype, w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off, wl.H, wl.d)
        kept_idx, kept_off, mask = select(z, wl.seq_off)
        self.kept_idx, self.kept_off = kept_idx, kept_off
        return z, I, mask

    def step(self, t, q, w, Q, with_gather=False):
        """One decode step; returns a dict of every stage's result."""
        wl = self.wl
        res = {}
        if t % self.tau == 0 or self.kept_idx is None:
            z, I, mask = self.refresh(q, w)
            res.update(z=z, I=I, mask=mask)
            b_of = np.repeat(np.arange(wl.B), np.diff(self.kept_off))
            zk = z[wl.seq_off[:-1][b_of] + self.kept_idx] if len(self.kept_idx) else np.zeros(0)
            if with_gather:
                hot, slot_of = gather(wl.cold, wl.seq_off, self.kept_idx, self.kept_off)
                res.update(hot=hot, slot_of=slot_of)
        else:
            zk = index_score_list(q, wl.q_dtype, w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                  self.kept_idx, self.kept_off, wl.H, wl.d)
        tk, cnt = topk(zk, self.kept_idx, self.kept_off, wl.topk)
        out, lse = sparse_attn(Q, wl.attn_dtype, wl.cold, wl.attn_dtype, wl.row_stride, wl.k_off, wl.v_off,
                               local_to_global(tk, wl.seq_off), wl.scale)
        res.update(zk=zk, kept_idx=self.kept_idx, kept_off=self.kept_off, topk_idx=tk, topk_cnt=cnt,
                   out=out, lse=lse)
        return res
