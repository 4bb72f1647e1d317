"""Parity of every CUDA stage with the fp64 oracle, called through the C ABI.

Sizes span several tiles with ragged tails; the full-size workloads (128K and
500K-token contexts, the ragged serving batch) run the decode steps in the same
launch configuration the benchmark times.  Tolerances: see tests/gpu_cases.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import (ATTN_TOL, I_TOL, Z_TOL, gpu_full_scores, gpu_select, in_mask_band, lsa_mod,
                       rel_err_per_head, run_decode_and_check)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


SCORE_CASES = {
    "tiny": lambda: synth.tiny(),
    "ragged_bf16": lambda: synth.small_ragged(key_dtype="bf16"),
    "ragged_e4m3": lambda: synth.small_ragged(key_dtype="e4m3"),
    "ragged_e4m3_d64_h16": lambda: synth.small_ragged(key_dtype="e4m3", H=16, d=64, lengths=(777, 129, 3000)),
    "ragged_bf16_d64_h32": lambda: synth.small_ragged(key_dtype="bf16", H=32, d=64, lengths=(2048, 1, 999)),
    "ragged_bf16_h16": lambda: synth.small_ragged(key_dtype="bf16", H=16, d=128, lengths=(1, 127, 128, 129, 4000)),
    "ragged_e4m3_h32": lambda: synth.small_ragged(key_dtype="e4m3", H=32, d=128, lengths=(5000, 300, 0, 129)),
}


# ------------------------------------------------------------------ score

@pytest.mark.parametrize("tc", [False, True], ids=["cuda_core", "tcgen05"])
@pytest.mark.parametrize("name", sorted(SCORE_CASES))
def test_index_score_full_matches_oracle(lsa, name, tc):
    wl = SCORE_CASES[name]()
    dev = synth.to_torch(wl, pin_cold=False)
    z, I = gpu_full_scores(wl, dev, lsa, tc=tc)
    if tc and wl.q_dtype == "bf16":   # every bf16-query case here has a shape the tensor cores run
        assert lsa.last_kernel() == f"scan_tc {wl.key_dtype} d{wl.d}"
    elif not tc:
        assert lsa.last_kernel() == "score_cuda_core"
    z_ref, I_ref = oracle.index_score(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                      wl.H, wl.d)
    assert np.abs(z - z_ref).max() <= Z_TOL
    assert np.abs(I - I_ref).max() <= I_TOL
    # the arithmetic is fp32 accumulation of exactly representable products: far inside the tolerance
    assert np.abs(z - z_ref).max() <= 1e-4 * max(1.0, np.abs(z_ref).max())


@pytest.mark.parametrize("tc", [False, True], ids=["cuda_core", "tcgen05"])
@pytest.mark.parametrize("name", ["tiny", "ragged_e4m3", "ragged_bf16", "ragged_bf16_d64_h32", "ragged_e4m3_h32"])
def test_index_score_listed_matches_oracle(lsa, name, tc):
    wl = SCORE_CASES[name]()
    dev = synth.to_torch(wl, pin_cold=False)
    rng = np.random.default_rng(3)
    lists = [np.sort(rng.choice(int(n), size=int(rng.integers(0, n + 1)), replace=False))
             for n in np.diff(wl.seq_off)]
    idx = np.concatenate(lists).astype(np.int32)
    idx_off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int64)
    cap = int(idx_off[-1]) + 5
    z = torch.full((cap,), 123.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx_d = torch.from_numpy(np.concatenate([idx, np.zeros(5, np.int32)])).cuda()   # list buffer of `cap` slots
    lsa.index_score(dev["q"], wl.q_dtype, dev["w"], dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"],
                    wl.n_total, wl.H, wl.d, z, None, idx=idx_d, idx_off=torch.from_numpy(idx_off).cuda(),
                    list_capacity=cap, cuda_core=not tc, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    z = z.cpu().numpy()
    z_ref = oracle.index_score_list(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off, idx,
                                    idx_off, wl.H, wl.d)
    n = int(idx_off[-1])
    assert np.abs(z[:n] - z_ref).max() <= Z_TOL
    assert (z[n:] == 123.0).all()          # nothing written past the list


def test_index_score_listed_e4m3_stage_reuse(lsa):
    """Listed e4m3 scan with enough rows that every CTA reuses its stages (about 4 tiles of 256 rows per
    CTA): 40K listed entries per sequence of the 500K-context workload.  The listed scores equal the full
    scan's scores of the same entries (same arithmetic), a sample matches the oracle, and no bounded wait
    gives up (a stage-free wait that misread a barrier two phases ahead used to time out here)."""
    wl = synth.ctx500k(with_cold=False)
    dev = synth.to_torch(wl, pin_cold=False)
    z_full, _ = gpu_full_scores(wl, dev, lsa, want_I=False, tc=True)
    rng = np.random.default_rng(9)
    lists = [np.sort(rng.choice(int(n), size=40000, replace=False)) for n in np.diff(wl.seq_off)]
    idx = np.concatenate(lists).astype(np.int32)
    idx_off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int64)
    cap = int(idx_off[-1])
    z = torch.full((cap,), 123.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        lsa.index_score(dev["q"], wl.q_dtype, dev["w"], dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"],
                        wl.n_total, wl.H, wl.d, z, None, idx=torch.from_numpy(idx).cuda(),
                        idx_off=torch.from_numpy(idx_off).cuda(), list_capacity=cap, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    z = z.cpu().numpy()
    b_of = np.repeat(np.arange(wl.B), np.diff(idx_off))
    glob = wl.seq_off[:-1][b_of] + idx
    assert np.abs(z - z_full[glob]).max() <= 1e-6 * max(1.0, np.abs(z_full).max())
    pick = np.sort(rng.choice(cap, size=3000, replace=False))
    sub = [idx[pick][b_of[pick] == b] for b in range(wl.B)]
    sub_off = np.concatenate([[0], np.cumsum([len(x) for x in sub])]).astype(np.int64)
    z_ref = oracle.index_score_list(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                    np.concatenate(sub).astype(np.int32), sub_off, wl.H, wl.d)
    assert np.abs(z[pick] - z_ref).max() <= Z_TOL


# --------------------------------------------------------------- select

@pytest.mark.parametrize("name", ["tiny", "ragged_bf16", "ragged_e4m3"])
def test_select_stage_exact_and_vs_fp64(lsa, name):
    wl = SCORE_CASES[name]()
    dev = synth.to_torch(wl, pin_cold=False)
    z, _ = gpu_full_scores(wl, dev, lsa, want_I=False, tc=True)
    kept, ko, mask, err = gpu_select(z, wl.seq_off, lsa)
    assert err == 0
    # stage-exact: the oracle's selection on the GPU's own fp32 scores
    k_ref, ko_ref, m_ref = oracle.select(z.astype(np.float64), wl.seq_off)
    assert np.array_equal(kept, k_ref) and np.array_equal(ko, ko_ref) and np.array_equal(mask, m_ref)
    # against the fp64 scores: equal outside the 1e-5 band around I = 0.5
    z64 = oracle.index_score(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off, wl.H, wl.d,
                             want_I=False)
    m64 = z64 >= 0
    band = in_mask_band(z64)
    assert np.array_equal(mask[~band], m64[~band])


SELECT_LENGTHS = [0, 1, 31, 32, 33, 1023, 1024, 1025, 0, 5000, 0]


@pytest.mark.parametrize("pattern", ["random", "all", "none", "signed_zero"])
def test_select_edge_cases(lsa, pattern):
    seq_off = np.concatenate([[0], np.cumsum(SELECT_LENGTHS)]).astype(np.int64)
    n = int(seq_off[-1])
    rng = np.random.default_rng(7)
    z = rng.normal(size=n).astype(np.float32)
    if pattern == "all":
        z = np.abs(z)
    elif pattern == "none":
        z = -np.abs(z) - 1e-3
    elif pattern == "signed_zero":
        z[::3] = -0.0
        z[1::3] = 0.0
        z[2::3] = -1e-30
    kept, ko, mask, err = gpu_select(z, seq_off, lsa)
    k_ref, ko_ref, m_ref = oracle.select(z.astype(np.float64), seq_off)
    assert err == 0
    assert np.array_equal(kept, k_ref) and np.array_equal(ko, ko_ref) and np.array_equal(mask, m_ref)


def test_select_capacity_overflow(lsa):
    seq_off = np.array([0, 3000, 3100, 9000], np.int64)
    z = np.random.default_rng(8).normal(size=9000).astype(np.float32)
    k_ref, ko_ref, _ = oracle.select(z.astype(np.float64), seq_off)
    cap = len(k_ref) // 2
    kept, ko, _, err = gpu_select(z, seq_off, lsa, capacity=cap)
    assert err == 3                                       # LSA_ERR_CAPACITY
    assert np.array_equal(ko, ko_ref)                     # true offsets even past capacity
    assert np.array_equal(kept, k_ref[:cap])


# ------------------------------------------------- scan + select, fused

def _score_select_gpu(lsa, wl, dev, capacity=None):
    n = wl.n_total
    B = len(wl.seq_off) - 1
    cap = n if capacity is None else capacity
    z = torch.full((max(n, 1) + 64,), 77.0, dtype=torch.float32, device="cuda")
    kept_idx = torch.full((max(cap, 1) + 16,), -7, dtype=torch.int32, device="cuda")
    kept_off = torch.full((B + 1,), -7, dtype=torch.int64, device="cuda")
    ws = torch.full((lsa.index_score_select_workspace_size(n, B),), 0xA5, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.index_score_select(dev["q"], wl.q_dtype, dev["w"], dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"],
                           n, wl.H, wl.d, z, kept_idx, cap, kept_off, ws, err=err)
    torch.cuda.synchronize()
    kernel = lsa.last_kernel()
    kept = kept_idx.cpu().numpy()
    assert (kept[cap:] == -7).all(), "selection wrote past the capacity"
    assert (z[n:].cpu().numpy() == 77.0).all(), "scan wrote past the entry axis"
    return z[:n].cpu().numpy(), kept, kept_off.cpu().numpy(), int(err.item()), kernel


@pytest.mark.parametrize("name", ["tiny", "ragged_bf16", "ragged_e4m3", "ragged_e4m3_d64_h16", "ragged_bf16_d64_h32",
                                  "ragged_bf16_h16", "ragged_e4m3_h32"])
def test_index_score_select_fused_matches_stages(lsa, name):
    """The fused scan + select gives the full scan's z bit for bit and, on those scores, the oracle's kept lists
    (sequences of every length modulo the tile: empty, 1, one tile, a ragged tail)."""
    wl = SCORE_CASES[name]()
    dev = synth.to_torch(wl, pin_cold=False)
    z, kept, ko, err, kernel = _score_select_gpu(lsa, wl, dev)
    assert err == 0
    if wl.q_dtype == "bf16":   # the tensor-core shapes: the selection comes from the scan's ballots
        assert kernel == "select_tiles_scatter"
    z_sep, _ = gpu_full_scores(wl, dev, lsa, want_I=False, tc=True)
    assert np.array_equal(z.view(np.uint32), z_sep.view(np.uint32))
    k_ref, ko_ref, _ = oracle.select(z.astype(np.float64), wl.seq_off)
    assert np.array_equal(ko, ko_ref)
    assert np.array_equal(kept[:len(k_ref)], k_ref)


def test_index_score_select_fused_capacity_overflow(lsa):
    wl = synth.small_ragged(key_dtype="e4m3", lengths=(5000, 300, 0, 129))
    dev = synth.to_torch(wl, pin_cold=False)
    z, kept_full, ko_full, err, _ = _score_select_gpu(lsa, wl, dev)
    assert err == 0
    total = int(ko_full[-1])
    cap = total // 2
    z2, kept, ko, err, _ = _score_select_gpu(lsa, wl, dev, capacity=cap)
    assert err == 3                                       # LSA_ERR_CAPACITY
    assert np.array_equal(ko, ko_full)                    # true offsets even past capacity
    assert np.array_equal(kept[:cap], kept_full[:cap])


def test_index_score_select_fused_full_size_500k(lsa):
    """The 500K-token batch (4 x 131072 e4m3 entries): the fused kept lists against the oracle's selection of the
    same scores, and equal to lsa_select's."""
    wl = synth.ctx500k(with_cold=False)
    dev = synth.to_torch(wl, pin_cold=False)
    z, kept, ko, err, kernel = _score_select_gpu(lsa, wl, dev)
    assert err == 0 and kernel == "select_tiles_scatter"
    k_ref, ko_ref, _ = oracle.select(z.astype(np.float64), wl.seq_off)
    assert np.array_equal(ko, ko_ref)
    assert np.array_equal(kept[:len(k_ref)], k_ref)
    kept2, ko2, _, err2 = gpu_select(z, wl.seq_off, lsa)
    assert err2 == 0 and np.array_equal(ko2, ko) and np.array_equal(kept2[:len(k_ref)], k_ref)


# ----------------------------------------------------------------- top-k

def _topk_gpu(lsa, z, z_by_entry, seq_off, kept, ko, k, cap=None):
    B = len(ko) - 1
    cap = len(kept) if cap is None else cap
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dt)).cuda()
    idx = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    pos = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    cnt = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    lsa.topk(t(z, np.float32), z_by_entry, t(seq_off, np.int64), t(kept if len(kept) else [0], np.int32),
             t(ko, np.int64), cap, k, idx, pos, cnt)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), pos.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("k", [1, 7, 32, 300, 2048])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_stage_exact(lsa, k, ties):
    rng = np.random.default_rng(k + 1000 * ties)
    # the last two keep ~40K and ~144K entries: keys re-read from global memory, runs longer than 64
    lens = [0, 5, 40, 999, 4096, 20000, 2048, 2049, 50000, 180000]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(seq_off[-1])
    z = rng.normal(size=n).astype(np.float32)
    if ties:
        z = np.round(z * 4) / 4          # few distinct values: ties everywhere
        z[::5] = -0.0
        z[1::5] = 0.0
    z = np.abs(z) * np.where(rng.random(n) < 0.8, 1, -1).astype(np.float32)   # ~80% kept
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    b_of = np.repeat(np.arange(len(lens)), np.diff(ko))
    zk = z[seq_off[:-1][b_of] + kept].astype(np.float64)
    ref_idx, ref_cnt = oracle.topk(zk, kept, ko, k)
    # by entry (refresh step) and by kept position (listed step)
    for by_entry, zin in ((1, z), (0, zk.astype(np.float32))):
        idx, pos, cnt = _topk_gpu(lsa, zin, by_entry, seq_off, kept, ko, k)
        assert np.array_equal(cnt, ref_cnt)
        assert np.array_equal(idx, ref_idx)
        for b in range(len(lens)):
            c = cnt[b]
            assert (pos[b][c:] == -1).all()
            assert np.array_equal(kept[pos[b][:c]], idx[b][:c])
            assert ((pos[b][:c] >= ko[b]) & (pos[b][:c] < ko[b + 1])).all()


@pytest.mark.parametrize("k", [64, 2048, 4096])
def test_topk_clustered_scores_stage_exact(lsa, k):
    """Scores shaped like a kept set of the 500K context: ~14K kept per sequence, chunk-correlated values in
    a narrow band, runs of exactly equal scores at and around the k-th, and one sequence whose scores are all
    equal: the candidate path and its fallbacks against the oracle's sorted top-k."""
    rng = np.random.default_rng(k)
    lens = [14400, 14000, 15000, 30000, 9000]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(seq_off[-1])
    chunk_mean = np.repeat(rng.uniform(0.05, 0.3, size=(n + 63) // 64), 64)[:n]
    z = (chunk_mean + 0.01 * rng.normal(size=n)).astype(np.float32)
    z[rng.random(n) < 0.1] = -1.0                                    # ~10% not kept
    s3 = slice(seq_off[3], seq_off[4])
    z[s3] = np.round(z[s3] * 64) / 64                                # many exact ties
    z[seq_off[4]:] = 0.125                                           # all equal
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    b_of = np.repeat(np.arange(len(lens)), np.diff(ko))
    zk = z[seq_off[:-1][b_of] + kept].astype(np.float64)
    ref_idx, ref_cnt = oracle.topk(zk, kept, ko, k)
    for by_entry, zin in ((1, z), (0, zk.astype(np.float32))):
        idx, pos, cnt = _topk_gpu(lsa, zin, by_entry, seq_off, kept, ko, k)
        assert np.array_equal(cnt, ref_cnt)
        assert np.array_equal(idx, ref_idx)


@pytest.mark.parametrize("sampled", ["low", "high"])
def test_topk_unrepresentative_sample_falls_back_exactly(lsa, sampled):
    """The scores at the evenly spaced positions the kernel samples are made the smallest (or largest) of their
    sequence, so the pivots drawn from them miss the k-th largest (too many keys above the upper pivot, too few
    from the lower one up, or too many between them) and the exact full-range select must run."""
    k = 2048
    lens = [12800, 6400, 25600]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    rng = np.random.default_rng(7 if sampled == "low" else 8)
    z = rng.uniform(1.0, 2.0, size=int(seq_off[-1])).astype(np.float32)
    for b, n in enumerate(lens):
        pos = (np.arange(64) * 2 + 1) * n // 128             # the sampled kept positions (every entry is kept)
        z[seq_off[b] + pos] = 1e-3 if sampled == "low" else 50.0 + rng.random(64)
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    assert np.array_equal(np.diff(ko), lens)
    zk = z.astype(np.float64)
    ref_idx, ref_cnt = oracle.topk(zk, kept, ko, k)
    for by_entry in (1, 0):
        idx, pos, cnt = _topk_gpu(lsa, z, by_entry, seq_off, kept, ko, k)
        assert np.array_equal(cnt, ref_cnt)
        assert np.array_equal(idx, ref_idx)


def test_topk_run_of_high_scores_in_one_segment(lsa):
    """A contiguous run of 200 top scores inside one warp's segment of kept positions (far more keys above the
    upper pivot in one segment than elsewhere), with distinct top scores in one sequence and equal ones plus
    ties at the k-th score in the other."""
    k = 2048
    lens = [14400, 14400]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    rng = np.random.default_rng(11)
    z = rng.uniform(0.1, 1.0, size=int(seq_off[-1])).astype(np.float32)
    z[1000:1200] = 100.0 + rng.random(200).astype(np.float32)      # sequence 0: distinct top scores
    z[seq_off[1] + 1000:seq_off[1] + 1200] = 100.0                  # sequence 1: all equal
    z[seq_off[1]:] = np.round(z[seq_off[1]:] * 16) / 16              # ... and ties at the k-th
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    zk = z.astype(np.float64)
    ref_idx, ref_cnt = oracle.topk(zk, kept, ko, k)
    for by_entry in (1, 0):
        idx, pos, cnt = _topk_gpu(lsa, z, by_entry, seq_off, kept, ko, k)
        assert np.array_equal(cnt, ref_cnt)
        assert np.array_equal(idx, ref_idx)


def test_topk_respects_kept_capacity(lsa):
    seq_off = np.array([0, 100, 300], np.int64)
    z = np.linspace(1, 2, 300).astype(np.float32)
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    idx, pos, cnt = _topk_gpu(lsa, z, 1, seq_off, kept[:150], ko, 64, cap=150)
    assert cnt[0] == 64 and cnt[1] == 50                     # only positions < 150 are read
    assert (idx[1][:50] == np.arange(50)).all()


# ------------------------------------------------------------ layer union

def test_index_union_of_three_scanned_layers(lsa):
    # three independent indexer layers (own q, w and keys) over one ragged entry axis
    lengths = (1000, 4133, 257, 64)
    wls = [synth.small_ragged(seed=30 + l, key_dtype="e4m3", lengths=lengths) for l in range(3)]
    n = wls[0].n_total
    seq_off = wls[0].seq_off
    zs = []
    for wl in wls:
        z, _ = gpu_full_scores(wl, synth.to_torch(wl, pin_cold=False), lsa, want_I=False, tc=True)
        zs.append(z.astype(np.float32))
    zd = [torch.from_numpy(z).cuda() for z in zs]
    zu = torch.full((n + 8,), 77.0, dtype=torch.float32, device="cuda")
    lsa.index_union(zd, n, zu)
    torch.cuda.synchronize()
    keep_ref, score_ref = oracle.index_union([z.astype(np.float64) for z in zs])
    got = zu[:n].cpu().numpy()
    assert np.array_equal(got, score_ref.astype(np.float32))      # the maximum is exact
    assert (zu[n:].cpu().numpy() == 77.0).all()
    # the union's kept set: select on the union score equals the OR of the layers' predictions
    kept, ko, mask, err = gpu_select(got, seq_off, lsa)
    assert err == 0 and np.array_equal(mask, keep_ref)
    # top-k of the union ranks by the union score (stage-exact against the oracle on the same fp32 values)
    k = 256
    kept_o, ko_o, _ = oracle.select(score_ref, seq_off)
    assert np.array_equal(kept, kept_o) and np.array_equal(ko, ko_o)
    b_of = np.repeat(np.arange(len(lengths)), np.diff(ko))
    zk = got[seq_off[:-1][b_of] + kept].astype(np.float64)
    ref_idx, ref_cnt = oracle.topk(zk, kept, ko, k)
    idx, pos, cnt = _topk_gpu(lsa, got, 1, seq_off, kept, ko, k)
    assert np.array_equal(cnt, ref_cnt) and np.array_equal(idx, ref_idx)


@pytest.mark.parametrize("n,offset", [(1 << 20, 0), (1000003, 0), (4096, 1)], ids=["vec4", "ragged_n", "unaligned"])
def test_index_union_random_with_nans(lsa, n, offset):
    rng = np.random.default_rng(n)
    zs = []
    for l in range(3):
        z = rng.normal(size=n + offset).astype(np.float32)
        z[rng.random(n + offset) < 0.01] = np.nan
        z[rng.random(n + offset) < 0.01] = -0.0
        zs.append(z)
    zd = [torch.from_numpy(z).cuda()[offset:] for z in zs]      # offset 1: 4-byte aligned only (scalar path)
    zu = torch.empty(n, dtype=torch.float32, device="cuda")
    lsa.index_union(zd, n, zu)
    torch.cuda.synchronize()
    keep_ref, score_ref = oracle.index_union([z[offset:].astype(np.float64) for z in zs])
    got = zu.cpu().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(score_ref))
    fin = ~np.isnan(score_ref)
    assert np.array_equal(got[fin], score_ref[fin].astype(np.float32))
    assert np.array_equal(got >= 0, keep_ref)


# ---------------------------------------------------------------- gather

def test_gather_bytes_and_slots(lsa):
    rng = np.random.default_rng(9)
    lens = [1000, 0, 37, 4000]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(seq_off[-1])
    row_bytes = 1024
    cold = torch.from_numpy(rng.integers(0, 255, size=(n, row_bytes), dtype=np.uint8)).pin_memory()
    z = rng.normal(size=n).astype(np.float32)
    kept, ko, _ = oracle.select(z.astype(np.float64), seq_off)
    hot_ref, slot_ref = oracle.gather(cold.numpy(), seq_off, kept, ko)
    cap = len(kept) + 3
    hot = torch.zeros((cap, row_bytes), dtype=torch.uint8, device="cuda")
    slot = torch.zeros(n, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dt)).cuda()
    lsa.gather(cold, row_bytes, t(seq_off, np.int64), n, t(kept, np.int32), t(ko, np.int64), hot, cap, slot, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(hot[: len(kept)].cpu().numpy(), hot_ref)
    assert (hot[len(kept):].cpu().numpy() == 0).all()
    assert np.array_equal(slot.cpu().numpy(), slot_ref)
    # capacity overflow: the first `cap` rows, error raised
    hot2 = torch.zeros((10, row_bytes), dtype=torch.uint8, device="cuda")
    lsa.gather(cold, row_bytes, t(seq_off, np.int64), n, t(kept, np.int32), t(ko, np.int64), hot2, 10, None, err)
    torch.cuda.synchronize()
    assert err.item() == 3
    assert np.array_equal(hot2.cpu().numpy(), hot_ref[:10])


def test_gather_rejects_pageable_cold_pool(lsa):
    cold = torch.zeros((16, 64), dtype=torch.uint8)          # not page-locked
    t0 = torch.zeros(2, dtype=torch.int64, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.gather(cold, 64, t0, 16, torch.zeros(1, dtype=torch.int32, device="cuda"), t0,
                   torch.zeros((4, 64), dtype=torch.uint8, device="cuda"), 4, None, None)
    assert e.value.status == 1


# ------------------------------------------------------------- attention

ATTN_CASES = [
    # dtype, B, Hq, D, k, n_rows, separate K/V
    ("f32", 1, 8, 64, 32, 512, True),
    ("f32", 2, 5, 96, 70, 300, True),
    ("bf16", 2, 128, 512, 2048, 6000, False),
    ("bf16", 3, 16, 128, 100, 400, True),
    ("bf16", 3, 128, 512, 300, 1000, False),   # tensor-core path: partial chunk, an empty sequence
    ("bf16", 1, 128, 512, 128, 128, False),    # exactly one full chunk
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"{c[0]}-B{c[1]}-H{c[2]}-D{c[3]}-k{c[4]}")
def test_sparse_attn_matches_oracle(lsa, case):
    _attn_case(lsa, case)


def test_sparse_attn_padding_holes(lsa):
    """Padding entries (-1, and any other negative index) scattered through the row lists, so that chunks
    start with padding, hold a single selected row, or none: the tensor-core path against the oracle."""
    _attn_case(lsa, ("bf16", 3, 128, 512, 640, 5000, False), holes=True)


def _attn_case(lsa, case, holes=False):
    dt, B, Hq, D, k, n_rows, separate = case
    g = torch.Generator().manual_seed(11)
    stride = 2 * D if separate else D
    to_raw = (lambda x: synth.to_raw(x, dt))
    Q = to_raw(torch.randn(B, Hq, D, generator=g))
    kv = to_raw(torch.randn(n_rows, stride, generator=g))
    rng = np.random.default_rng(12)
    rows = np.full((B, k), -1, np.int32)
    counts = [k, k // 3, 0][:B] if B <= 3 else [k] * B
    for b in range(B):
        c = min(counts[b], n_rows)
        rows[b, :c] = np.sort(rng.choice(n_rows, size=c, replace=False))
    if holes:
        rows[0, rng.random(k) < 0.4] = -1        # sequence 0: 40% holes anywhere
        rows[0, :5] = -1                          # chunk 0 starts with padding
        rows[0, 128:256] = -1                     # chunk 1: a single selected row
        rows[0, 200] = 17
        rows[0, 256:384] = -1                     # chunk 2: nothing selected
        rows[1, 1::2] = -3                        # sequence 1: every other entry another negative value
    out = torch.empty((B, Hq, D), dtype=torch.float32 if dt == "f32" else torch.int16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(lsa.sparse_attn_workspace_size(B, Hq, D, k), dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(D)
    v_off = D if separate else 0
    lsa.sparse_attn(synth.raw_to_torch(Q), dt, synth.raw_to_torch(kv), stride, 0, v_off,
                    torch.from_numpy(rows).cuda(), B, Hq, D, k, scale, out, lse, ws)
    torch.cuda.synchronize()
    assert lsa.last_kernel().startswith("attn_combine")
    rows = np.where(rows < 0, -1, rows)   # every negative index is padding
    out_ref, lse_ref = oracle.sparse_attn(Q, dt, kv, dt, stride, 0, v_off, rows.astype(np.int64), scale)
    o = out.cpu().numpy()
    o = oracle.decode(o.view(np.uint16), "bf16") if dt == "bf16" else o.astype(np.float64)
    rel = rel_err_per_head(o, out_ref)
    assert rel <= ATTN_TOL[dt], rel
    lg = lse.cpu().numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.abs(lg[fin] - lse_ref[fin]).max() <= (1e-5 if dt == "f32" else 1e-3)
    empty = rows.max(axis=1) < 0
    assert (o[empty] == 0).all()


# ---------------------------------------------------------- decode steps

@pytest.mark.parametrize("full_fetch", [False, True], ids=["cached", "full_fetch"])
@pytest.mark.parametrize("name,steps,tau", [
    ("tiny", [0, 1, 2, 3, 4, 5], 4),
    ("ragged_bf16", [0, 1, 3, 4, 7, 8], 4),
    ("ragged_e4m3", [0, 2, 4, 5], 4),
])
def test_decode_steps_small(lsa, name, steps, tau, full_fetch):
    wl = SCORE_CASES[name]()
    reps = run_decode_and_check(wl, steps, tau, lsa, full_fetch=full_fetch)
    assert [r["t"] for r in reps] == steps


def test_hot_cache_fetches_only_new_rows(lsa):
    """A refresh that keeps the same set fetches nothing; one with a different query fetches exactly
    the kept entries that are not resident; a small hot buffer evicts rows no longer kept."""
    from gpu_cases import check_hot_cache, make_context, read_ctx

    wl = synth.small_ragged(key_dtype="bf16", lengths=(3000, 1500))
    dev = synth.to_torch(wl)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda")
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    ins = [wl.step_inputs(t) for t in (0, 5)]
    dins = [(synth.raw_to_torch(q), torch.from_numpy(np.ascontiguousarray(w)).cuda(), synth.raw_to_torch(Q))
            for q, w, Q in ins]
    q1 = synth.raw_to_torch(synth.bf16_bits(torch.randn(wl.B, wl.H, wl.d) / 8))   # an unrelated query
    z0 = oracle.index_score(ins[0][0], "bf16", ins[0][1], wl.keys, "bf16", None, wl.seq_off, wl.H, wl.d,
                            want_I=False)
    n0 = int((z0 >= 0).sum())
    for cap in (wl.n_total, n0 + 40):   # roomy, and barely larger than the first kept set
        ctx = make_context(wl, dev, lsa, kept_capacity=cap, tau=1)
        ctx.step(0, *dins[0], out, lse)
        assert ctx.fetched() == n0
        resident = set(np.nonzero(lsa.device_view(ctx.view().slot_of, wl.n_total, torch.int32).cpu().numpy() >= 0)[0])
        check_hot_cache(ctx, wl, lsa, read_ctx(ctx, wl, lsa))
        ctx.step(1, *dins[0], out, lse)               # same query: same kept set
        assert ctx.fetched() == 0
        ctx.step(2, q1, dins[0][1], dins[0][2], out, lse)
        g = read_ctx(ctx, wl, lsa)
        assert g["err"] == 0
        b_of = np.repeat(np.arange(wl.B), np.diff(g["kept_off"]))
        ent = set((wl.seq_off[:-1][b_of] + g["kept_idx"]).tolist())
        assert ctx.fetched() == len(ent - resident)
        check_hot_cache(ctx, wl, lsa, g)
        ctx.close()


@pytest.mark.parametrize("key_dtype", ["bf16", "e4m3"])
def test_decode_lookahead_matches_oracle(lsa, key_dtype):
    """Lookahead L = 3, tau = 8, every step of three windows: window 1's set predicted at step 5 and fetched
    while steps 5-7 attend window 0's set, current from step 8; the cache emptied before the prediction at
    step 13, so its fetch brings every kept row (a cold start) while steps 13-15 still read theirs."""
    wl = synth.small_ragged(key_dtype=key_dtype)
    reps = run_decode_and_check(wl, list(range(24)), 8, lsa, lookahead=3, flush_at=(13,))
    assert len(reps) == 24
    assert max(r["attn_rel"] for r in reps) <= ATTN_TOL["bf16"]


def test_decode_lookahead_skipped_prediction_refreshes(lsa):
    """A run that skips window 2's prediction step (13) refreshes at step 16, like the plain cadence."""
    wl = synth.small_ragged(key_dtype="e4m3")
    steps = [t for t in range(20) if t != 13]
    reps = run_decode_and_check(wl, steps, 8, lsa, lookahead=3)
    assert len(reps) == len(steps)


def test_decode_step_host_equals_device(lsa):
    wl = synth.small_ragged(key_dtype="e4m3")
    from gpu_cases import make_context

    dev = synth.to_torch(wl)
    ctx_a = make_context(wl, dev, lsa, tau=4)
    ctx_b = make_context(wl, dev, lsa, tau=4)
    out_a = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda")
    lse_a = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    out_b = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16).pin_memory()
    lse_b = torch.empty((wl.B, wl.Hq), dtype=torch.float32).pin_memory()
    for t in range(6):
        q_t, w_t, Q_t = wl.step_inputs(t)
        ctx_a.step(t, synth.raw_to_torch(q_t), torch.from_numpy(w_t).cuda(), synth.raw_to_torch(Q_t), out_a, lse_a)
        qh = synth.raw_to_torch(q_t, "cpu").pin_memory()
        wh = torch.from_numpy(np.ascontiguousarray(w_t)).pin_memory()
        Qh = synth.raw_to_torch(Q_t, "cpu").pin_memory()
        ctx_b.step_host(t, qh, wh, Qh, out_b, lse_b)
        torch.cuda.synchronize()
        assert torch.equal(out_a.cpu(), out_b)
        assert torch.equal(lse_a.cpu(), lse_b)
    assert ctx_a.launches() > 0
    ctx_a.close()
    ctx_b.close()


def test_decode_step_host_pipelined_equals_device(lsa):
    """Host steps issued back to back with no synchronisation in between (the input copies
    of each call overlap the previous call's kernels through the two staging slots) give the
    same bytes as device steps, for every step, across refreshes."""
    wl = synth.small_ragged(key_dtype="e4m3")
    from gpu_cases import make_context, read_ctx

    dev = synth.to_torch(wl)
    ctx_a = make_context(wl, dev, lsa, tau=4)
    ctx_b = make_context(wl, dev, lsa, tau=4)
    n = 11
    ins = [wl.step_inputs(t) for t in range(n)]
    host_in = [(synth.raw_to_torch(q, "cpu").pin_memory(), torch.from_numpy(np.ascontiguousarray(w)).pin_memory(),
                synth.raw_to_torch(Q, "cpu").pin_memory()) for q, w, Q in ins]
    # pinned outputs (written directly by the attention over the host link) and, every third step,
    # pageable ones (through the device staging buffer and a copy)
    pin = lambda x, i: x if i % 3 == 2 else x.pin_memory()
    outs_b = [pin(torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16), i) for i in range(n)]
    lses_b = [pin(torch.empty((wl.B, wl.Hq), dtype=torch.float32), i) for i in range(n)]
    torch.cuda.synchronize()
    for t in range(n):
        ctx_b.step_host(t, *host_in[t], outs_b[t], lses_b[t])
    torch.cuda.synchronize()
    out_a = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda")
    lse_a = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    for t in range(n):
        q_t, w_t, Q_t = ins[t]
        ctx_a.step(t, synth.raw_to_torch(q_t), torch.from_numpy(w_t).cuda(), synth.raw_to_torch(Q_t), out_a, lse_a)
        torch.cuda.synchronize()
        assert torch.equal(out_a.cpu(), outs_b[t]), t
        assert torch.equal(lse_a.cpu(), lses_b[t]), t
    assert int(read_ctx(ctx_b, wl, lsa)["err"]) == 0
    ctx_a.close()
    ctx_b.close()


def test_decode_graph_replay_equals_eager(lsa):
    """Steps replayed from captured CUDA graphs give the same bytes as eager steps, across
    refreshes, with the output buffers alternating (two graphs per step kind)."""
    from gpu_cases import make_context

    wl = synth.small_ragged(key_dtype="bf16")
    dev = synth.to_torch(wl)
    ctx_g = make_context(wl, dev, lsa, tau=3)
    ctx_e = make_context(wl, dev, lsa, tau=3)
    ctx_e.set_graphs(False)
    outs = [torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda") for _ in range(3)]
    lses = [torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda") for _ in range(3)]
    ins = [wl.step_inputs(t) for t in range(10)]
    dins = [(synth.raw_to_torch(q), torch.from_numpy(np.ascontiguousarray(w)).cuda(), synth.raw_to_torch(Q))
            for q, w, Q in ins]
    for t in range(10):
        o = t % 2
        ctx_g.step(t, *dins[t], outs[o], lses[o])
        ctx_e.step(t, *dins[t], outs[2], lses[2])
        torch.cuda.synchronize()
        assert torch.equal(outs[o], outs[2]), t
        assert torch.equal(lses[o], lses[2]), t
    assert ctx_g.launches() == ctx_e.launches()
    ctx_g.close()
    ctx_e.close()


@pytest.mark.parametrize("name", ["ctx128k", "ctx500k"])
def test_decode_full_size(lsa, name):
    wl = synth.WORKLOADS[name]()
    reps = run_decode_and_check(wl, [0, 1, 63], 64, lsa, kept_capacity=int(0.2 * wl.n_total))
    print(name, reps)


def test_decode_lookahead_full_size(lsa):
    """The 500K-token context with lookahead 16: window 1 predicted at step 48 and current from step 64."""
    wl = synth.ctx500k()
    reps = run_decode_and_check(wl, [0, 47, 48, 49, 63, 64, 65], 64, lsa, kept_capacity=int(0.2 * wl.n_total),
                                lookahead=16)
    assert len(reps) == 7


def test_decode_ragged_serving_batch(lsa):
    wl = synth.ragged()
    reps = run_decode_and_check(wl, [0, 1], 64, lsa)
    print("ragged", reps)
