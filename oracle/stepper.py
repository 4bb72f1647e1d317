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

With several indexer layers (section 2.4 "Optimal Configuration": the layers'
predictions are united at inference) each layer scores with its own keys and
query, an entry is kept when any layer keeps it, and the ranking score is the
union score max_l z_l (index_union).

Lookahead L >= 1 (blog page: critical chunks reach GPU memory "just in time";
section 2.1 "Dynamic Fetching"), the reading this build takes: the kept set of
window r >= 1 (steps r tau .. r tau + tau - 1) is predicted at step r tau - L,
after that step's own work, from that step's indexer query; steps r tau - L ..
r tau - 1 still use window r - 1's set; at step r tau the predicted set becomes
current and is re-ranked with that step's query like any listed step.  Window
0 refreshes at its first step (the first step of a run refreshes, wherever it
falls, and predicts nothing), and a window whose prediction step did not run
refreshes at its first step.  L = 0 is the plain cadence.
"""
from __future__ import annotations

import numpy as np

from . import TAU, gather, index_score, index_score_list, index_union, local_to_global, select, sparse_attn, topk


class OracleDecoder:
    """Plain sequential driver over the oracle stages; holds the kept set between refreshes."""

    def __init__(self, wl, tau: int = TAU, layers=None, lookahead: int = 0):
        """layers: [(keys, k_scale), ...] of indexer layers 1 .. L-1 (layer 0 is the workload's keys); with
        layers, step() takes q [L, B, H, d] and w [L, B, H].  lookahead: see the module docstring."""
        assert 0 <= lookahead < tau
        self.wl = wl
        self.tau = tau
        self.lookahead = lookahead
        self.layers = [(wl.keys, wl.k_scale)] + list(layers or [])
        self.kept_idx = None
        self.kept_off = None
        self.kept_z = None       # the scores the current kept set was selected on
        self.predicted = None    # (kept_idx, kept_off, z) of the next window, from its prediction step
        self.slot_of = None

    def _per_layer(self, q, w):
        if len(self.layers) == 1:
            return [(q, w, self.layers[0])]
        return [(q[l], w[l], self.layers[l]) for l in range(len(self.layers))]

    def score_all(self, q, w):
        """Scores of every entry (the union score with several layers) and their probabilities."""
        wl = self.wl
        if len(self.layers) == 1:
            return index_score(q, wl.q_dtype, w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off, wl.H, wl.d)
        zs = [index_score(ql, wl.q_dtype, wl_, keys, wl.key_dtype, ks, wl.seq_off, wl.H, wl.d, want_I=False)
              for ql, wl_, (keys, ks) in self._per_layer(q, w)]
        z = index_union(zs)[1]
        return z, 1.0 / (1.0 + np.exp(-z))   # the union's probability: that of its most confident layer

    def refresh(self, q, w):
        z, I = self.score_all(q, w)
        kept_idx, kept_off, mask = select(z, self.wl.seq_off)
        self.kept_idx, self.kept_off, self.kept_z = kept_idx, kept_off, z
        return z, I, mask

    def step(self, t, q, w, Q, with_gather=False):
        """One decode step; returns a dict of every stage's result."""
        wl = self.wl
        res = {}
        L = self.lookahead
        boundary = t % self.tau == 0
        refresh = self.kept_idx is None or (boundary and (L == 0 or self.predicted is None))
        if refresh:
            self.predicted = None
            z, I, mask = self.refresh(q, w)
            res.update(z=z, I=I, mask=mask)
            b_of = np.repeat(np.arange(wl.B), np.diff(self.kept_off))
            zk = z[wl.seq_off[:-1][b_of] + self.kept_idx] if len(self.kept_idx) else np.zeros(0)
            if with_gather:
                hot, slot_of = gather(wl.cold, wl.seq_off, self.kept_idx, self.kept_off)
                res.update(hot=hot, slot_of=slot_of)
        else:
            if boundary:   # the window's predicted set becomes current
                self.kept_idx, self.kept_off, self.kept_z = self.predicted
                self.predicted = None
            zks = [index_score_list(ql, wl.q_dtype, wl_, keys, wl.key_dtype, ks, wl.seq_off, self.kept_idx,
                                    self.kept_off, wl.H, wl.d) for ql, wl_, (keys, ks) in self._per_layer(q, w)]
            zk = zks[0] if len(zks) == 1 else index_union(zks)[1]
        tk, cnt = topk(zk, self.kept_idx, self.kept_off, wl.topk)
        out, lse = sparse_attn(Q, wl.attn_dtype, wl.cold, wl.attn_dtype, wl.row_stride, wl.k_off, wl.v_off,
                               local_to_global(tk, wl.seq_off), wl.scale)
        res.update(zk=zk, kept_idx=self.kept_idx, kept_off=self.kept_off, topk_idx=tk, topk_cnt=cnt,
                   out=out, lse=lse, z_sel=self.kept_z)
        if L > 0 and not refresh and not boundary and (t + L) % self.tau == 0:
            # the next window's kept set, from this step's query, after this step's own work (a refresh step,
            # the very first step of a run, predicts nothing)
            zp, _ = self.score_all(q, w)
            kept_idx, kept_off, _ = select(zp, wl.seq_off)
            self.predicted = (kept_idx, kept_off, zp)
            res.update(z_pred=zp, pred_kept_idx=kept_idx, pred_kept_off=kept_off)
        return res
