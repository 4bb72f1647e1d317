"""fp64 CPU oracle for the Lookahead Sparse Attention (LSA) decode hot path.

TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference leg of ``bench.py`` may
import this package.  It shares no code with the CUDA library: the arithmetic
lives in ``lsa_oracle.c`` (plain fp64 loops, OpenMP over independent outputs)
and this module only marshals numpy arrays into it.

Every function follows "FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long
Context via Lookahead Sparse Attention", gist.science technical summary,
section 2.1 (Periodic Triggering, Scoring Mechanism, Dynamic Fetching, Tiered
Selection), with the score fixed as I = sigmoid(sum_j w_j ReLU(q_j . k_s)).

Parity pins: see ``tests/test_oracle_pins.py``.  The pages print no worked
numeric example, so every pin is a closed form, an invariant, a library
routine on a special case or brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsa_oracle.c")
_LIB = os.path.join(_HERE, "liblsa_oracle.so")

# dtype codes of the oracle library (its own numbering)
F32, BF16, E4M3, F64 = 0, 1, 2, 3
_NP_CODE = {"f32": F32, "bf16": BF16, "e4m3": E4M3, "f64": F64}

TAU = 64  # refresh period (section 2.1 "Periodic Triggering": tau = 64)


def build(force: bool = False) -> str:
    """Compile lsa_oracle.c into liblsa_oracle.so with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.orc_bf16_to_f64.restype = dbl
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_to_f64.restype = dbl
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_decode.argtypes = [P, i32, i64, P]
        L.orc_index_score.argtypes = [P, i32, P, P, i32, P, P, i32, i32, i32, P, P]
        L.orc_index_score_list.argtypes = [P, i32, P, P, i32, P, P, P, P, i32, i32, i32, P, P]
        L.orc_select.restype = i64
        L.orc_select.argtypes = [P, P, i32, P, P, P]
        L.orc_topk.argtypes = [P, P, P, i32, i32, P, P]
        L.orc_index_union.argtypes = [P, i32, i64, P, P]
        L.orc_query_encode.argtypes = [P, i32, i32, i32, P, P, P, i32, i32, i32, i32, P, P, P]
        L.orc_gather.argtypes = [P, i64, P, P, P, i32, P, P]
        L.orc_sparse_attn.argtypes = [P, i32, P, i32, i64, i64, i64, P, i32, i32, i32, i32, dbl, P, P]
        L.orc_num_threads.restype = i32
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def decode(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Decode raw element bits (f32 / bf16 as uint16 / e4m3 as uint8) to fp64."""
    raw = np.ascontiguousarray(raw)
    out = np.empty(raw.shape, np.float64)
    lib().orc_decode(_p(raw), _NP_CODE[dtype], raw.size, _p(out))
    return out


def index_score(q, q_dtype, w, k, k_dtype, k_scale, seq_off, H, d, want_I=True):
    """z[s] = sum_j w[b,j] ReLU(q[b,j,:] . k[s,:]) and I[s] = sigmoid(z[s]) for every entry.

    q: raw [B,H,d]; w: f32 [B,H]; k: raw [sum N, d]; k_scale: f32 [sum N, ceil(d/128)] or None.
    """
    seq_off = _c(seq_off, np.int64)
    B = len(seq_off) - 1
    n = int(seq_off[-1])
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    w = _c(w, np.float32)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    z = np.empty(n, np.float64)
    I = np.empty(n, np.float64) if want_I else None
    lib().orc_index_score(_p(q), _NP_CODE[q_dtype], _p(w), _p(k), _NP_CODE[k_dtype], _p(ks),
                          _p(seq_off), B, H, d, _p(z), _p(I))
    return (z, I) if want_I else z


def index_score_list(q, q_dtype, w, k, k_dtype, k_scale, seq_off, idx, idx_off, H, d):
    """Scores of the listed entries idx[idx_off[b]:idx_off[b+1]] (local indices) only."""
    seq_off = _c(seq_off, np.int64)
    idx = _c(idx, np.int32)
    idx_off = _c(idx_off, np.int64)
    B = len(seq_off) - 1
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    w = _c(w, np.float32)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    z = np.empty(int(idx_off[-1]), np.float64)
    lib().orc_index_score_list(_p(q), _NP_CODE[q_dtype], _p(w), _p(k), _NP_CODE[k_dtype], _p(ks),
                               _p(seq_off), _p(idx), _p(idx_off), B, H, d, _p(z), None)
    return z


def select(z, seq_off):
    """Kept entries (z >= 0, i.e. I >= 0.5) per sequence: (kept_idx, kept_off, mask)."""
    z = _c(z, np.float64)
    seq_off = _c(seq_off, np.int64)
    B = len(seq_off) - 1
    kept_idx = np.empty(max(int(seq_off[-1]), 1), np.int32)
    kept_off = np.empty(B + 1, np.int64)
    mask = np.empty(int(seq_off[-1]), np.uint8)
    n = lib().orc_select(_p(z), _p(seq_off), B, _p(kept_idx), _p(kept_off), _p(mask))
    return kept_idx[:n].copy(), kept_off, mask.astype(bool)


def index_union(z_layers):
    """OR-mode union of indexer layers: (keep, score); keep[s] = any layer has z >= 0, score = the largest
    non-NaN z of the layers (NaN when every layer's is NaN)."""
    zs = [_c(z, np.float64) for z in z_layers]
    n = len(zs[0])
    arr = (ctypes.c_void_p * len(zs))(*[z.ctypes.data for z in zs])
    keep = np.empty(max(n, 1), np.uint8)
    score = np.empty(max(n, 1), np.float64)
    lib().orc_index_union(ctypes.cast(arr, ctypes.c_void_p), len(zs), n, _p(keep), _p(score))
    return keep[:n].astype(bool), score[:n]


def query_encode(h, h_dtype, W_dq, W_uq, W_w, w_dtype, H, d):
    """Indexer query encoder: (c, q, w) with c = W_dq h [B,rank], q = W_uq c viewed as [B,H,d] and
    w = W_w h [B,H], all fp64.  h: raw [B,hidden]; W_dq raw [rank,hidden]; W_uq raw [H*d,rank];
    W_w raw [H,hidden]."""
    h = np.ascontiguousarray(h)
    W_dq, W_uq, W_w = (np.ascontiguousarray(a) for a in (W_dq, W_uq, W_w))
    B, hidden = h.shape
    rank = W_dq.shape[0]
    assert W_dq.shape == (rank, hidden) and W_uq.shape == (H * d, rank) and W_w.shape == (H, hidden)
    c = np.empty((B, rank), np.float64)
    q = np.empty((B, H, d), np.float64)
    w = np.empty((B, H), np.float64)
    lib().orc_query_encode(_p(h), _NP_CODE[h_dtype], B, hidden, _p(W_dq), _p(W_uq), _p(W_w), _NP_CODE[w_dtype],
                           rank, H, d, _p(c), _p(q), _p(w))
    return c, q, w


def topk(zk, kept_idx, kept_off, k):
    """Top-k by (z desc, index asc) inside each kept set; ascending indices, -1 padded."""
    zk = _c(zk, np.float64)
    kept_idx = _c(kept_idx, np.int32)
    kept_off = _c(kept_off, np.int64)
    B = len(kept_off) - 1
    out = np.empty((B, k), np.int32)
    cnt = np.empty(B, np.int32)
    lib().orc_topk(_p(zk), _p(kept_idx), _p(kept_off), B, k, _p(out), _p(cnt))
    return out, cnt


def gather(cold, seq_off, kept_idx, kept_off):
    """Hot buffer rows in kept order, plus slot_of (hot row of each entry or -1)."""
    cold = np.ascontiguousarray(cold)
    row_bytes = cold.shape[1] * cold.itemsize
    seq_off = _c(seq_off, np.int64)
    kept_idx = _c(kept_idx, np.int32)
    kept_off = _c(kept_off, np.int64)
    B = len(seq_off) - 1
    hot = np.zeros((max(int(kept_off[-1]), 1), cold.shape[1]), cold.dtype)
    slot_of = np.empty(int(seq_off[-1]), np.int32)
    lib().orc_gather(_p(cold.view(np.uint8)), row_bytes, _p(seq_off), _p(kept_idx), _p(kept_off), B,
                     _p(hot.view(np.uint8)), _p(slot_of))
    return hot[: int(kept_off[-1])], slot_of


def sparse_attn(Q, q_dtype, kv, kv_dtype, row_stride, k_off, v_off, sel_global, scale):
    """Multi-query softmax attention of Q [B,Hq,D] over the selected rows of kv.

    sel_global: int64 [B, k] global entry indices (-1 = padding).
    Returns (out [B,Hq,D] fp64, lse [B,Hq] fp64).
    """
    Q = np.ascontiguousarray(Q)
    kv = np.ascontiguousarray(kv)
    sel = _c(sel_global, np.int64)
    B, Hq, D = Q.shape
    k = sel.shape[1]
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    lib().orc_sparse_attn(_p(Q), _NP_CODE[q_dtype], _p(kv), _NP_CODE[kv_dtype], row_stride, k_off, v_off,
                          _p(sel), B, Hq, D, k, float(scale), _p(out), _p(lse))
    return out, lse


def attention_set(topk_idx, seq_off, window, hca_off=None):
    """The rows one sequence attends when the always-resident context is merged into the core attention
    (technical summary, section 2.1 "Architectural Design": all HCA chunks, 128:1 compressed, are retained
    for global awareness; section 1 "Problem Statement": the most recent 8K tokens alone answer most long
    requests).  Read as the
    set union, per sequence b, of
      * the top-k entries (topk_idx[b], local indices, -1 padded),
      * the last `window` entries of the sequence (all of them when it is shorter), and
      * every HCA row of the sequence (hca_off[b] .. hca_off[b+1]-1; none when hca_off is None),
    each row counted once.  Rows are global indices into the concatenation [entries (n_total rows); HCA
    rows], listed as: top-k entries outside the window (ascending), HCA rows (ascending), window entries
    (ascending); -1 padded to a common width.  Returns (rows int64 [B, width], count int64 [B])."""
    seq_off = np.asarray(seq_off, np.int64)
    B = len(seq_off) - 1
    n_total = int(seq_off[-1])
    lists = []
    for b in range(B):
        n_b = int(seq_off[b + 1] - seq_off[b])
        w_b = min(int(window), n_b)
        win = set(range(n_b - w_b, n_b))
        top = set(int(e) for e in np.asarray(topk_idx[b]) if e >= 0)
        hca = [] if hca_off is None else list(range(int(hca_off[b]), int(hca_off[b + 1])))
        rows = ([int(seq_off[b]) + e for e in sorted(top - win)] + [n_total + j for j in hca]
                + [int(seq_off[b]) + e for e in sorted(win)])
        assert len(rows) == len(set(rows))
        lists.append(rows)
    width = max(1, max(len(r) for r in lists))
    out = np.full((B, width), -1, np.int64)
    for b, r in enumerate(lists):
        out[b, :len(r)] = r
    return out, np.array([len(r) for r in lists], np.int64)


def local_to_global(idx, seq_off):
    """Turn a [B,k] array of per-sequence entry indices (-1 padded) into global entry indices."""
    idx = np.asarray(idx, np.int64)
    base = np.asarray(seq_off, np.int64)[:-1, None]
    return np.where(idx >= 0, idx + base, -1)
