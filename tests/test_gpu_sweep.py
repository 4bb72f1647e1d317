"""Parity of the indexer-only sweep's path (lsa_index_score + lsa_select) with
the fp64 oracle at the sweep's corners: every (H, d, key dtype) at the smallest
point (B = 1, N = 8K), the e4m3 d = 64 keys on the tensor cores for every H
(full and listed scans, asserting which kernel ran), and the largest points
(B = 32 sequences of N = 256K entries: 2 GB of bf16 keys, and e4m3 d = 64 keys
with H = 16) in the launch configuration the sweep bench times, compared on a
sample of entries the oracle scores one by one plus the stage-exact selection
over every entry.  Inputs: synth.sweep (12.5% planted chunks + ~1% leakage).
Tolerances: tests/gpu_cases.py."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import I_TOL, Z_TOL, gpu_full_scores, gpu_select, in_mask_band, lsa_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


def check_kept_fraction(wl, frac):
    """The recipe's realised kept fraction: ~13.5% with 64 heads (12.5% planted, all kept, + ~1% leakage).
    With 16 or 32 heads the gate that holds the background leakage at 1% (a larger gamma over fewer
    background heads) also pushes many planted entries below the threshold: 1-13% kept."""
    if wl.H == 64:
        assert 0.12 < frac < 0.15
    else:
        assert 0.005 < frac < 0.15


def expected_kernel(wl, listed=False):
    return ("scan_tc_listed " if listed else "scan_tc ") + f"{wl.key_dtype} d{wl.d}"


@pytest.mark.parametrize("H", [16, 32, 64])
def test_e4m3_d64_on_tensor_cores_full_and_listed(lsa, H):
    """e4m3 keys with d = 64 (64-byte rows, the 64-byte-swizzled operand layout) against the oracle, full scan
    and listed scan, ragged sequences with partial tiles and an empty one; the kernel that ran is named."""
    wl = synth.small_ragged(key_dtype="e4m3", H=H, d=64, lengths=(3000, 257, 0, 1, 4099))
    dev = synth.to_torch(wl, pin_cold=False)
    z, I = gpu_full_scores(wl, dev, lsa, tc=True)
    assert lsa.last_kernel() == expected_kernel(wl)
    z_ref, I_ref = oracle.index_score(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                      wl.H, wl.d)
    assert np.abs(z - z_ref).max() <= Z_TOL
    assert np.abs(I - I_ref).max() <= I_TOL
    assert np.abs(z - z_ref).max() <= 1e-4 * max(1.0, np.abs(z_ref).max())
    # listed: a random subset of every sequence (three tiles per CTA on the longest ones)
    rng = np.random.default_rng(H)
    lists = [np.sort(rng.choice(int(n), size=int(rng.integers(0, n + 1)), replace=False))
             for n in np.diff(wl.seq_off)]
    idx = np.concatenate(lists).astype(np.int32)
    idx_off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int64)
    cap = int(idx_off[-1]) + 3
    zl = torch.full((cap,), 55.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.index_score(dev["q"], wl.q_dtype, dev["w"], dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"],
                    wl.n_total, wl.H, wl.d, zl, None, idx=torch.from_numpy(np.concatenate([idx, [0, 0, 0]])
                                                                           .astype(np.int32)).cuda(),
                    idx_off=torch.from_numpy(idx_off).cuda(), list_capacity=cap, err=err)
    torch.cuda.synchronize()
    assert lsa.last_kernel() == expected_kernel(wl, listed=True)
    assert err.item() == 0
    zl = zl.cpu().numpy()
    n = int(idx_off[-1])
    b_of = np.repeat(np.arange(wl.B), np.diff(idx_off))
    assert np.array_equal(zl[:n], z[wl.seq_off[:-1][b_of] + idx])   # the same arithmetic as the full scan
    assert (zl[n:] == 55.0).all()


SMALL = [(1, 8192, H, d, dt) for H in synth.SWEEP_H for d in synth.SWEEP_D for dt in synth.SWEEP_DTYPES]


@pytest.mark.parametrize("B,N,H,d,dt", SMALL, ids=[f"H{p[2]}_d{p[3]}_{p[4]}" for p in SMALL])
def test_sweep_smallest_points_match_oracle(lsa, B, N, H, d, dt):
    wl = synth.sweep(B, N, H, d, dt)
    dev = synth.to_torch(wl, pin_cold=False)
    z, I = gpu_full_scores(wl, dev, lsa, tc=True)
    assert lsa.last_kernel() == expected_kernel(wl)
    z_ref, I_ref = oracle.index_score(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                      wl.H, wl.d)
    assert np.abs(z - z_ref).max() <= Z_TOL
    assert np.abs(I - I_ref).max() <= I_TOL
    kept, ko, mask, err = gpu_select(z, wl.seq_off, lsa)
    assert err == 0
    k_ref, ko_ref, m_ref = oracle.select(z.astype(np.float64), wl.seq_off)    # stage-exact
    assert np.array_equal(kept, k_ref) and np.array_equal(ko, ko_ref) and np.array_equal(mask, m_ref)
    band = in_mask_band(z_ref)
    assert np.array_equal(mask[~band], (z_ref >= 0)[~band])                    # against fp64
    check_kept_fraction(wl, ko[-1] / wl.n_total)


LARGE = [(32, 262144, 64, 128, "bf16"), (32, 262144, 16, 64, "e4m3")]


@pytest.mark.parametrize("B,N,H,d,dt", LARGE, ids=["bf16_d128_h64", "e4m3_d64_h16"])
def test_sweep_largest_points_sampled(lsa, B, N, H, d, dt):
    """8.4M entries per launch (2 GB of bf16 keys / 0.5 GB of e4m3 keys): the tensor-core scan over the whole
    axis, z of 16K sampled entries (every sequence, first and last tiles included) against the oracle, the
    selection stage-exact over every entry, and the mask against fp64 on the sample."""
    wl = synth.sweep(B, N, H, d, dt)
    dev = synth.to_torch(wl, pin_cold=False)
    z, _ = gpu_full_scores(wl, dev, lsa, want_I=False, tc=True)
    assert lsa.last_kernel() == expected_kernel(wl)
    rng = np.random.default_rng(5)
    lists = [np.unique(np.concatenate([[0, 1, N - 2, N - 1], rng.choice(N, size=508, replace=False)]))
             for _ in range(B)]
    idx = np.concatenate(lists).astype(np.int32)
    idx_off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int64)
    z_ref = oracle.index_score_list(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off, idx,
                                    idx_off, wl.H, wl.d)
    b_of = np.repeat(np.arange(B), np.diff(idx_off))
    glob = wl.seq_off[:-1][b_of] + idx
    assert np.abs(z[glob] - z_ref).max() <= Z_TOL
    I_gpu = 1.0 / (1.0 + np.exp(-z[glob].astype(np.float64)))
    assert np.abs(I_gpu - 1.0 / (1.0 + np.exp(-z_ref))).max() <= I_TOL
    kept, ko, mask, err = gpu_select(z, wl.seq_off, lsa)
    assert err == 0
    k_ref, ko_ref, m_ref = oracle.select(z.astype(np.float64), wl.seq_off)
    assert np.array_equal(ko, ko_ref) and np.array_equal(kept, k_ref) and np.array_equal(mask, m_ref)
    band = in_mask_band(z_ref)
    assert np.array_equal(mask[glob][~band], (z_ref >= 0)[~band])
    check_kept_fraction(wl, ko[-1] / wl.n_total)
