"""Pins of the fp64 oracle to things other than itself (CPU only).

The pages ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse Attention") print no
worked numeric example, so the oracle is pinned by: a hand-worked case with
exact dyadic values (tests/golden/score_handworked.json), library routines on
special cases (torch's float8 / bfloat16 decoders, torch fp64 dense softmax
attention, numpy matrix products), closed forms (one selected entry, identical
keys, q = 0), brute force on tiny inputs (repeated argmax top-k) and the
invariants section 2.1 fixes (I >= 0.5 rule, kept set contains the top-k).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle.stepper import OracleDecoder

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- decoders

def test_e4m3_decoder_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode(codes, "e4m3")
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert nan.sum() == 2 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_bf16_decoder_matches_torch_for_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.decode(bits, "bf16")
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------------ score

def _golden():
    with open(os.path.join(GOLDEN, "score_handworked.json")) as f:
        return json.load(f)


def test_score_threshold_topk_handworked():
    g = _golden()
    q = np.array(g["q"], np.float32)[None]
    w = np.array(g["w"], np.float32)[None]
    k = np.array(g["k"], np.float32)
    seq_off = np.array([0, len(k)], np.int64)
    z, I = oracle.index_score(q, "f32", w, k, "f32", None, seq_off, g["H"], g["d"])
    assert z.tolist() == g["z"]
    np.testing.assert_allclose(I, g["I"], rtol=1e-15, atol=0)
    kept_idx, kept_off, mask = oracle.select(z, seq_off)
    assert kept_idx.tolist() == g["kept"] and kept_off.tolist() == [0, 3]
    assert mask.tolist() == [i in g["kept"] for i in range(len(k))]
    zk = z[kept_idx]
    for kk, want in g["topk"].items():
        idx, cnt = oracle.topk(zk, kept_idx, kept_off, int(kk))
        assert idx[0].tolist() == want
        assert cnt[0] == min(int(kk), 3)


def _rand_case(seed, B=3, H=5, d=7, lens=(9, 1, 14)):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, d, generator=g).numpy()
    w = torch.randn(B, H, generator=g).numpy()
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    k = torch.randn(int(seq_off[-1]), d, generator=g).numpy()
    return q, w, k, seq_off


def test_score_matches_matrix_formulation():
    """relu(K Q^T) w with numpy matmuls, per sequence: a formulation independent of the loops."""
    q, w, k, seq_off = _rand_case(1)
    z, I = oracle.index_score(q, "f32", w, k, "f32", None, seq_off, 5, 7)
    for b in range(3):
        kb = k[seq_off[b]:seq_off[b + 1]].astype(np.float64)
        ref = np.maximum(kb @ q[b].astype(np.float64).T, 0.0) @ w[b].astype(np.float64)
        np.testing.assert_allclose(z[seq_off[b]:seq_off[b + 1]], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(I, 1.0 / (1.0 + np.exp(-z)), rtol=1e-15)


def test_score_special_cases():
    q, w, k, seq_off = _rand_case(2, B=1, H=1, d=6, lens=(40,))
    # one head with unit gate: z = ReLU(q.k) >= 0 so every entry is kept
    z, I = oracle.index_score(q, "f32", np.ones((1, 1), np.float32), k, "f32", None, seq_off, 1, 6)
    np.testing.assert_allclose(z, np.maximum(k.astype(np.float64) @ q[0, 0].astype(np.float64), 0), rtol=1e-13)
    assert (I >= 0.5).all() and len(oracle.select(z, seq_off)[0]) == 40
    # q = 0: z = 0 and I = 0.5 everywhere, all kept
    z, I = oracle.index_score(np.zeros((1, 3, 6), np.float32), "f32", np.ones((1, 3), np.float32), k, "f32",
                              None, seq_off, 3, 6)
    assert (z == 0).all() and (I == 0.5).all() and len(oracle.select(z, seq_off)[0]) == 40
    # all gates negative: z <= 0; only entries whose every head is <= 0 reach z = 0
    q, w, k, seq_off = _rand_case(3, B=1, H=4, d=5, lens=(64,))
    z, _ = oracle.index_score(q, "f32", -np.abs(w), k, "f32", None, seq_off, 4, 5)
    dots = k.astype(np.float64) @ q[0].astype(np.float64).T
    assert (z <= 0).all()
    kept = oracle.select(z, seq_off)[0]
    assert kept.tolist() == np.nonzero((dots <= 0).all(axis=1))[0].tolist()


def test_score_e4m3_keys_apply_row_scale():
    g = torch.Generator().manual_seed(4)
    k32 = torch.randn(50, 16, generator=g)
    codes, scale = synth.e4m3_rows(k32)
    q = synth.bf16_bits(torch.randn(1, 3, 16, generator=g))
    w = np.array([[0.3, -1.0, 0.7]], np.float32)
    seq_off = np.array([0, 50], np.int64)
    z = oracle.index_score(q, "bf16", w, codes, "e4m3", scale, seq_off, 3, 16, want_I=False)
    kd = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * scale.astype(np.float64)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()[0]
    ref = np.maximum(kd @ qd.T, 0) @ w[0].astype(np.float64)
    np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-14)


def test_score_list_equals_full_scan_rows():
    q, w, k, seq_off = _rand_case(5)
    z = oracle.index_score(q, "f32", w, k, "f32", None, seq_off, 5, 7, want_I=False)
    idx = np.array([0, 3, 8, 0, 2, 13, 5], np.int32)
    idx_off = np.array([0, 3, 4, 7], np.int64)
    zl = oracle.index_score_list(q, "f32", w, k, "f32", None, seq_off, idx, idx_off, 5, 7)
    want = [z[seq_off[b] + idx[p]] for b in range(3) for p in range(idx_off[b], idx_off[b + 1])]
    assert zl.tolist() == want


# --------------------------------------------------------------- threshold

def test_select_is_the_half_threshold_rule():
    q, w, k, seq_off = _rand_case(6, lens=(100, 0, 57))
    z, I = oracle.index_score(q, "f32", w, k, "f32", None, seq_off, 5, 7)
    kept_idx, kept_off, mask = oracle.select(z, seq_off)
    assert np.array_equal(mask, I >= 0.5)
    assert np.array_equal(mask, z >= 0)
    assert kept_off[1] == kept_off[2]          # empty sequence keeps nothing
    for b in range(3):
        ki = kept_idx[kept_off[b]:kept_off[b + 1]]
        assert (np.diff(ki) > 0).all()
        local = np.nonzero(mask[seq_off[b]:seq_off[b + 1]])[0]
        assert ki.tolist() == local.tolist()


# ------------------------------------------------------------- layer union

def test_union_handworked():
    # three layers x six entries, chosen by hand: the union fetches what any layer fetches (z >= 0,
    # -0.0 included); a NaN is no prediction and no score
    nan = float("nan")
    z = [np.array([1.5, -1.0, nan, -0.0, -2.0, nan]),
         np.array([-2.0, -3.0, nan, -5.0, -0.5, nan]),
         np.array([-1.0, 2.25, -7.0, nan, -4.0, nan])]
    keep, score = oracle.index_union(z)
    assert keep.tolist() == [True, True, False, True, False, False]
    assert score[:5].tolist() == [1.5, 2.25, -7.0, 0.0, -0.5] and np.signbit(score[3])
    assert np.isnan(score[5])


def test_union_is_the_or_of_the_layers_selections():
    seq_off = np.array([0, 300, 300, 1000], np.int64)
    layers = []
    for l in range(3):
        q, w, k, _ = _rand_case(20 + l, lens=(300, 0, 700))
        z, _ = oracle.index_score(q, "f32", w, k, "f32", None, seq_off, 5, 7)
        layers.append(z)
    keep, score = oracle.index_union(layers)
    masks = [oracle.select(z, seq_off)[2] for z in layers]
    assert np.array_equal(keep, masks[0] | masks[1] | masks[2])
    assert np.array_equal(keep, score >= 0)                       # the score decides the same set
    stacked = np.stack(layers)
    assert np.all((stacked == score).any(axis=0))                 # the score is one of the layers' scores
    assert np.all(stacked <= score)
    # one layer: the union is that layer
    keep1, score1 = oracle.index_union([layers[1]])
    assert np.array_equal(keep1, masks[1]) and np.array_equal(score1, layers[1])
    # the union's kept set is what select keeps on the union score
    kept_idx, kept_off, mask = oracle.select(score, seq_off)
    assert np.array_equal(mask, keep)


# ------------------------------------------------------------ query encoder

def test_query_encode_handworked():
    with open(os.path.join(GOLDEN, "query_encode_handworked.json")) as f:
        g = json.load(f)
    arr = {k: np.array(g[k], np.float32) for k in ("h", "W_dq", "W_uq", "W_w")}
    c, q, w = oracle.query_encode(arr["h"], "f32", arr["W_dq"], arr["W_uq"], arr["W_w"], "f32", g["H"], g["d"])
    assert np.array_equal(c, np.array(g["c"], np.float64))
    assert np.array_equal(q, np.array(g["q"], np.float64))
    assert np.array_equal(w, np.array(g["w"], np.float64))


def test_query_encode_matches_numpy_matmul_on_bf16_operands():
    """Random bf16 operands: the oracle's loops equal numpy's fp64 matrix products of the decoded operands
    (every product of two bf16 values is exact in fp64, so only the summation order differs)."""
    g = torch.Generator().manual_seed(5)
    B, hidden, rank, H, d = 3, 40, 24, 4, 8
    h = synth.bf16_bits(torch.randn(B, hidden, generator=g))
    W_dq = synth.bf16_bits(torch.randn(rank, hidden, generator=g) / 6)
    W_uq = synth.bf16_bits(torch.randn(H * d, rank, generator=g) / 5)
    W_w = synth.bf16_bits(torch.randn(H, hidden, generator=g) / 6)
    c, q, w = oracle.query_encode(h, "bf16", W_dq, W_uq, W_w, "bf16", H, d)
    hd, Dq, Uq, Ww = (oracle.decode(a, "bf16") for a in (h, W_dq, W_uq, W_w))
    np.testing.assert_allclose(c, hd @ Dq.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(q.reshape(B, H * d), (hd @ Dq.T) @ Uq.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w, hd @ Ww.T, rtol=1e-13, atol=1e-13)
    # head j of q is the j-th block of d rows of W_uq applied to c (no transposed head/channel order)
    j = 2
    np.testing.assert_allclose(q[:, j, :], c @ Uq[j * d:(j + 1) * d].T, rtol=1e-12, atol=1e-12)


def test_query_encode_is_low_rank_in_h():
    """The map h -> q factors through the rank-r latent: over the one-hot hidden states its image has rank
    exactly r (generic weights), and q is linear in h."""
    g = torch.Generator().manual_seed(6)
    hidden, rank, H, d = 24, 5, 3, 4
    W_dq = torch.randn(rank, hidden, generator=g).numpy().astype(np.float32)
    W_uq = torch.randn(H * d, rank, generator=g).numpy().astype(np.float32)
    W_w = torch.randn(H, hidden, generator=g).numpy().astype(np.float32)
    eye = np.eye(hidden, dtype=np.float32)
    _, q, w = oracle.query_encode(eye, "f32", W_dq, W_uq, W_w, "f32", H, d)
    assert np.linalg.matrix_rank(q.reshape(hidden, H * d), tol=1e-9) == rank
    np.testing.assert_allclose(w, W_w.T.astype(np.float64), rtol=0, atol=0)   # w of e_k is column k of W_w
    h2 = torch.randn(2, hidden, generator=g).numpy().astype(np.float32)
    _, q2, _ = oracle.query_encode(h2, "f32", W_dq, W_uq, W_w, "f32", H, d)
    lin = np.tensordot(h2.astype(np.float64), q, axes=(1, 0))           # sum_k h_k q(e_k)
    np.testing.assert_allclose(q2, lin, rtol=1e-10, atol=1e-10)


# ------------------------------------------- merged attention set (window + HCA)

def test_attention_set_handworked():
    """Two sequences of 10 and 4 entries, window 3, HCA rows 2 and 1.  Sequence 0: top-k {1, 5, 8}; 8 lies in
    the window {7, 8, 9} and is counted once -> {1, 5} + HCA {0, 1} + {7, 8, 9}.  Sequence 1 (entries 10..13):
    top-k {0, 2} (local) -> 2 lies in the window {1, 2, 3} -> {0} + HCA {2} + {1, 2, 3}.  HCA rows come after
    the 14 entries in the concatenated row space (14, 15, 16)."""
    seq_off = np.array([0, 10, 14])
    topk = np.array([[1, 5, 8], [0, 2, -1]])
    rows, cnt = oracle.attention_set(topk, seq_off, 3, hca_off=np.array([0, 2, 3]))
    assert cnt.tolist() == [7, 5]
    assert rows[0].tolist() == [1, 5, 14, 15, 7, 8, 9]
    assert rows[1].tolist() == [10, 16, 11, 12, 13, -1, -1]
    # no window, no HCA: the top-k set itself
    rows0, cnt0 = oracle.attention_set(topk, seq_off, 0)
    assert cnt0.tolist() == [3, 2] and rows0[1].tolist() == [10, 12, -1]
    # a window longer than the sequence covers all of it
    rows1, cnt1 = oracle.attention_set(topk, seq_off, 50)
    assert cnt1.tolist() == [10, 4] and rows1[1].tolist() == [10, 11, 12, 13] + [-1] * 6


def _lse_merge(parts):
    """Softmax attention over a disjoint union from the parts' (out, lse): the log-sum-exp identity."""
    lses = np.stack([p[1] for p in parts])
    lse = np.logaddexp.reduce(lses, axis=0)
    out = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
    return out, lse


def test_merged_attention_is_softmax_over_the_union():
    """Attention over the merged set equals the log-sum-exp combination of attention over its three disjoint
    parts (top-k outside the window, HCA rows, window), and differs from attention that counts a top-k entry
    inside the window twice."""
    g = torch.Generator().manual_seed(17)
    B, Hq, D, stride = 2, 4, 32, 32
    seq_off = np.array([0, 300, 420])
    n_total = 420
    hca_off = np.array([0, 3, 5])
    kv = torch.randn(n_total + 5, stride, generator=g).numpy().astype(np.float32)
    Q = torch.randn(B, Hq, D, generator=g).numpy().astype(np.float32)
    topk = np.array([[3, 40, 41, 290, 299, -1], [0, 7, 100, 110, 115, 119]])
    window = 16
    rows, cnt = oracle.attention_set(topk, seq_off, window, hca_off=hca_off)
    scale = 0.2
    out, lse = oracle.sparse_attn(Q, "f32", kv, "f32", stride, 0, 0, rows, scale)
    parts = []
    for sel in ("top", "hca", "win"):
        part = np.full_like(rows, -1)
        for b in range(B):
            r = [x for x in rows[b, :cnt[b]]
                 if (sel == "hca") == (x >= n_total) and
                 (sel == "hca" or ((x - seq_off[b] >= seq_off[b + 1] - seq_off[b] - window) == (sel == "win")))]
            part[b, :len(r)] = r
        parts.append(oracle.sparse_attn(Q, "f32", kv, "f32", stride, 0, 0, part, scale))
    m_out, m_lse = _lse_merge(parts)
    np.testing.assert_allclose(out, m_out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, m_lse, rtol=1e-12, atol=1e-12)
    # counting entry 290 (in sequence 0's window) a second time changes the result
    dup = np.concatenate([rows, np.full((B, 1), -1)], axis=1)
    dup[0, cnt[0]] = 290
    out_d, _ = oracle.sparse_attn(Q, "f32", kv, "f32", stride, 0, 0, dup, scale)
    assert np.max(np.abs(out_d[0] - out[0])) > 1e-6


# ------------------------------------------------------------------- top-k

def _brute_topk(zk, idx, k):
    """k rounds of argmax; ties to the lower index; result sorted ascending."""
    left = list(range(len(zk)))
    chosen = []
    for _ in range(min(k, len(zk))):
        best = None
        for p in left:
            if best is None or zk[p] > zk[best] or (zk[p] == zk[best] and idx[p] < idx[best]):
                best = p
        chosen.append(idx[best])
        left.remove(best)
    return sorted(chosen) + [-1] * (k - len(chosen))


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    lens = [int(rng.integers(0, 60)) for _ in range(4)]
    kept_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    kept_idx = np.concatenate([np.sort(rng.choice(200, n, replace=False)) for n in lens]).astype(np.int32)
    zk = np.round(rng.normal(size=int(kept_off[-1])), 1)   # coarse values -> many exact ties
    zk[::7] = 0.0
    for k in (1, 5, 17, 64):
        idx, cnt = oracle.topk(zk, kept_idx, kept_off, k)
        for b in range(4):
            sl = slice(kept_off[b], kept_off[b + 1])
            assert idx[b].tolist() == _brute_topk(zk[sl].tolist(), kept_idx[sl].tolist(), k)
            assert cnt[b] == min(k, lens[b])


def test_topk_invariants_on_planted_case():
    wl = synth.small_ragged()
    z = oracle.index_score(wl.q, "bf16", wl.w, wl.keys, "bf16", None, wl.seq_off, wl.H, wl.d, want_I=False)
    kept_idx, kept_off, _ = oracle.select(z, wl.seq_off)
    b_of = np.repeat(np.arange(wl.B), np.diff(kept_off))
    zk = z[wl.seq_off[:-1][b_of] + kept_idx]
    idx, cnt = oracle.topk(zk, kept_idx, kept_off, wl.topk)
    for b in range(wl.B):
        ks = kept_idx[kept_off[b]:kept_off[b + 1]]
        zs = zk[kept_off[b]:kept_off[b + 1]]
        sel = idx[b][:cnt[b]]
        assert cnt[b] == min(wl.topk, len(ks))
        assert set(sel.tolist()) <= set(ks.tolist())            # kept set contains the top-k
        assert (idx[b][cnt[b]:] == -1).all()
        if len(ks) > cnt[b]:
            in_sel = np.isin(ks, sel)
            assert zs[~in_sel].max() <= zs[in_sel].min()


# --------------------------------------------------------------- attention

def _attn_case(seed, B=2, Hq=3, D=8, N=20, k=6):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, D, generator=g).numpy()
    kv = torch.randn(N, 2 * D, generator=g).numpy()
    return Q, kv


def test_attention_all_selected_equals_dense_softmax():
    Q, kv = _attn_case(7)
    N, D = kv.shape[0], Q.shape[2]
    sel = np.tile(np.arange(N, dtype=np.int64), (2, 1))
    out, lse = oracle.sparse_attn(Q, "f32", kv, "f32", 2 * D, 0, D, sel, 0.37)
    Kt = torch.from_numpy(kv[:, :D]).double()
    Vt = torch.from_numpy(kv[:, D:]).double()
    logits = torch.from_numpy(Q).double() @ Kt.T * 0.37
    ref = torch.softmax(logits, dim=-1) @ Vt
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=1e-13)


def test_attention_padding_is_ignored_and_subset_matches_dense():
    Q, kv = _attn_case(8)
    D = Q.shape[2]
    sel = np.array([[3, -1, 7, 11, -1, 19], [-1, -1, -1, 0, 2, 4]], np.int64)
    out, lse = oracle.sparse_attn(Q, "f32", kv, "f32", 2 * D, 0, D, sel, 1.0)
    for b in range(2):
        rows = sel[b][sel[b] >= 0]
        Kt = torch.from_numpy(kv[rows, :D]).double()
        Vt = torch.from_numpy(kv[rows, D:]).double()
        ref = torch.softmax(torch.from_numpy(Q[b]).double() @ Kt.T, -1) @ Vt
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    Q, kv = _attn_case(9)
    D = Q.shape[2]
    # one selected entry: output is that V row, lse is its logit
    sel = np.array([[5] + [-1] * 5, [-1] * 5 + [12]], np.int64)
    out, lse = oracle.sparse_attn(Q, "f32", kv, "f32", 2 * D, 0, D, sel, 0.5)
    np.testing.assert_array_equal(out[0], np.broadcast_to(kv[5, D:], out[0].shape))
    np.testing.assert_allclose(lse[1], 0.5 * Q[1].astype(np.float64) @ kv[12, :D].astype(np.float64), rtol=1e-13)
    # identical keys: uniform weights, output = mean of V, lse = a + log n
    kv2 = kv.copy()
    kv2[:, :D] = kv[0, :D]
    sel = np.tile(np.array([1, 4, 9, 16], np.int64), (2, 1))
    out, lse = oracle.sparse_attn(Q, "f32", kv2, "f32", 2 * D, 0, D, sel, 0.5)
    np.testing.assert_allclose(out[0, 0], kv2[[1, 4, 9, 16], D:].astype(np.float64).mean(0), rtol=1e-12)
    a = 0.5 * Q[1, 2].astype(np.float64) @ kv[0, :D].astype(np.float64)
    np.testing.assert_allclose(lse[1, 2], a + math.log(4), rtol=1e-13)
    # nothing selected: zero output, lse = -inf
    out, lse = oracle.sparse_attn(Q, "f32", kv, "f32", 2 * D, 0, D, -np.ones((2, 6), np.int64), 0.5)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_attention_latent_kv_alias_bf16():
    """K = V on one bf16 latent row (k_off = v_off = 0), checked against torch fp64."""
    g = torch.Generator().manual_seed(10)
    Q = synth.bf16_bits(torch.randn(1, 4, 32, generator=g))
    kv = synth.bf16_bits(torch.randn(30, 32, generator=g))
    sel = np.array([[2, 3, 5, 7, 11, 13, 17, 19, 23, 29]], np.int64)
    out, lse = oracle.sparse_attn(Q, "bf16", kv, "bf16", 32, 0, 0, sel, 1 / math.sqrt(32))
    Kd = oracle.decode(kv, "bf16")[sel[0]]
    Qd = oracle.decode(Q, "bf16")[0]
    ref = torch.softmax(torch.from_numpy(Qd @ Kd.T / math.sqrt(32)), -1).numpy() @ Kd
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ gather

def test_gather_copies_kept_rows_bytewise():
    rng = np.random.default_rng(11)
    cold = rng.integers(0, 65536, size=(30, 24), dtype=np.uint16)
    seq_off = np.array([0, 10, 10, 30], np.int64)
    kept_idx = np.array([1, 4, 9, 0, 7, 19], np.int32)
    kept_off = np.array([0, 3, 3, 6], np.int64)
    hot, slot_of = oracle.gather(cold, seq_off, kept_idx, kept_off)
    want_rows = [1, 4, 9, 10, 17, 29]
    assert np.array_equal(hot, cold[want_rows])
    want_slot = -np.ones(30, np.int32)
    want_slot[want_rows] = np.arange(6)
    assert np.array_equal(slot_of, want_slot)


# ---------------------------------------------------------- decode cadence

def test_decoder_tau_cadence_and_kept_superset():
    wl = synth.small_ragged(lengths=(300, 700), topk=64, Hq=4, D=64)
    dec = OracleDecoder(wl, tau=4)
    r0 = dec.step(0, *wl.step_inputs(0), with_gather=True)
    kept0 = r0["kept_idx"].copy()
    r1 = dec.step(1, *wl.step_inputs(1))
    assert np.array_equal(r1["kept_idx"], kept0)           # no refresh between tau boundaries
    assert "z" in r0 and "z" not in r1
    for r in (r0, r1):
        for b in range(wl.B):
            sel = r["topk_idx"][b][: r["topk_cnt"][b]]
            assert set(sel.tolist()) <= set(r["kept_idx"][r["kept_off"][b]:r["kept_off"][b + 1]].tolist())
    r4 = dec.step(4, *wl.step_inputs(4))
    assert "z" in r4                                       # refresh again at t = tau


def test_decoder_lookahead_cadence():
    """Lookahead L = 2, tau = 4: steps 0-3 run exactly the plain cadence's window 0 (steps 2 and 3 still use
    its kept set); step 2 predicts window 1's set, which equals a plain refresh given step 2's query; step 4
    makes it current without a refresh and ranks it by the listed scores of step 4's query; a run that skips
    the prediction step (6) refreshes at 8 like the plain cadence; a run whose first step is a prediction step
    only refreshes there."""
    wl = synth.small_ragged(lengths=(300, 700), topk=64, Hq=4, D=64)
    tau, L = 4, 2
    la = OracleDecoder(wl, tau=tau, lookahead=L)
    plain = OracleDecoder(wl, tau=tau)
    res = {t: la.step(t, *wl.step_inputs(t)) for t in (0, 1, 2, 3, 4, 5, 8)}   # step 6 skipped
    for t in range(4):
        r = plain.step(t, *wl.step_inputs(t))
        for key in ("kept_idx", "kept_off", "topk_idx", "topk_cnt", "out", "lse"):
            assert np.array_equal(res[t][key], r[key]), (t, key)
    assert "z_pred" in res[2] and all("z_pred" not in res[t] for t in (0, 1, 3, 4, 5, 8))
    q2, w2, _ = wl.step_inputs(2)
    q4, w4, Q4 = wl.step_inputs(4)
    ref = OracleDecoder(wl, tau=tau).step(0, q2, w2, Q4)          # a refresh from step 2's query
    assert np.array_equal(res[4]["kept_idx"], ref["kept_idx"])
    assert np.array_equal(res[4]["kept_off"], ref["kept_off"])
    assert "z" not in res[4] and np.array_equal(res[4]["z_sel"], res[2]["z_pred"])
    zk4 = oracle.index_score_list(q4, wl.q_dtype, w4, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                  ref["kept_idx"], ref["kept_off"], wl.H, wl.d)
    tk4, _ = oracle.topk(zk4, ref["kept_idx"], ref["kept_off"], wl.topk)
    assert np.array_equal(res[4]["topk_idx"], tk4)
    assert np.array_equal(res[5]["kept_idx"], res[4]["kept_idx"])   # the window keeps its set
    r8 = OracleDecoder(wl, tau=tau).step(8, *wl.step_inputs(8))     # no prediction ran: a refresh at 8
    assert "z" in res[8] and np.array_equal(res[8]["kept_idx"], r8["kept_idx"])
    first = OracleDecoder(wl, tau=tau, lookahead=L).step(2, *wl.step_inputs(2))
    assert "z" in first and "z_pred" not in first


def test_layered_decoder_reduces_to_one_layer_and_keeps_the_or():
    """Three copies of one indexer layer give exactly the one-layer decode (the union of equal scores is
    that score); with three different layers every layer's own kept set lies inside the union's, and the
    union's top-k ranks by the largest layer score."""
    wl = synth.small_ragged(lengths=(300, 700), topk=64, Hq=4, D=64)
    one = OracleDecoder(wl, tau=4)
    three = OracleDecoder(wl, tau=4, layers=[(wl.keys, wl.k_scale)] * 2)
    for t in (0, 1, 4):
        q, w, Q = wl.step_inputs(t)
        a = one.step(t, q, w, Q)
        b = three.step(t, np.stack([q] * 3), np.stack([w] * 3), Q)
        for key in ("kept_idx", "kept_off", "topk_idx", "topk_cnt", "out", "lse", "zk"):
            assert np.array_equal(a[key], b[key]), (t, key)
    others = [synth.small_ragged(seed=5 + 10 * l, lengths=(300, 700), topk=64, Hq=4, D=64) for l in (1, 2)]
    mixed = OracleDecoder(wl, tau=4, layers=[(o.keys, o.k_scale) for o in others])
    ins = [wl.step_inputs(0)] + [o.step_inputs(0) for o in others]
    r = mixed.step(0, np.stack([i[0] for i in ins]), np.stack([i[1] for i in ins]), ins[0][2])
    kept = set(zip(np.repeat(np.arange(wl.B), np.diff(r["kept_off"])).tolist(), r["kept_idx"].tolist()))
    zs = []
    for l, src in enumerate([wl] + others):
        z_l = oracle.index_score(ins[l][0], wl.q_dtype, ins[l][1], src.keys, src.key_dtype, src.k_scale,
                                 wl.seq_off, wl.H, wl.d, want_I=False)
        zs.append(z_l)
        idx, off, _ = oracle.select(z_l, wl.seq_off)
        own = set(zip(np.repeat(np.arange(wl.B), np.diff(off)).tolist(), idx.tolist()))
        assert own <= kept
    assert np.array_equal(r["z"], np.max(np.stack(zs), axis=0))


# ----------------------------------------------------- synthetic workloads

def test_gate_calibration_reproduces_background_leakage():
    from oracle.calibrate_gate import TARGET, pass_rate

    H, d = 64, 128
    g = torch.Generator().manual_seed(12345 + 131 * H + d)
    u = synth.unit(g, d)
    q = synth.bf16_bits(synth.indexer_queries(g, H, d, u)[None])
    keys = synth.bf16_bits(synth.background_keys(g, 65536, d))
    rate = pass_rate(synth.GATE_GAMMA[(H, d)], q, keys, H, d)
    assert abs(rate - TARGET) < 2e-4


def test_planted_workload_kept_fraction():
    wl = synth.ctx128k(with_cold=False)
    z = oracle.index_score(wl.q, "bf16", wl.w, wl.keys, "bf16", None, wl.seq_off, wl.H, wl.d, want_I=False)
    keep = z >= 0
    assert 0.115 <= wl.planted.mean() <= 0.125
    assert keep[wl.planted].mean() > 0.99
    assert 0.003 < keep[~wl.planted].mean() < 0.02
    assert 0.12 < keep.mean() < 0.14


def test_e4m3_quantization_recipe():
    g = torch.Generator().manual_seed(13)
    x = torch.randn(64, 128, generator=g) * torch.rand(64, 1, generator=g) * 5
    codes, scale = synth.e4m3_rows(x)
    dec = oracle.decode(codes, "e4m3") * scale
    assert not np.isnan(dec).any()
    assert np.allclose(np.abs(oracle.decode(codes, "e4m3")).max(axis=1), 448.0)
    rel = np.abs(dec - x.numpy()) / np.maximum(np.abs(x.numpy()), scale * 2 ** -6)
    assert rel.max() <= 2 ** -4 + 1e-6
