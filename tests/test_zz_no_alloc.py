"""lsa_select_noalloc, the selection for callers that cannot allocate device
memory (its scratch is a static array inside the library), against lsa_select
with a caller workspace and against the oracle's selection: identical kept
lists, offsets and masks on two calls in a row (the second call finds the first
call's scratch contents), with and without a caller mask (without one, the mask
words live in the static scratch too), a kept list longer than the output's
capacity, and sizes above the static limit rejected before any launch.
Collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from lookahead_sparse_kv_index_b200 import lsa as mod

    return mod


def _select_both(lsa, z_np, seq_off_np, capacity, want_mask=True):
    n = int(seq_off_np[-1])
    B = len(seq_off_np) - 1
    z = torch.from_numpy(z_np).cuda()
    seq_off = torch.from_numpy(seq_off_np).cuda()
    outs = []
    for use_ws in (True, False):
        kept = torch.full((capacity + 16,), -5, dtype=torch.int32, device="cuda")   # 16 guard slots
        ko = torch.full((B + 1,), -5, dtype=torch.int64, device="cuda")
        mask = torch.zeros((n + 31) // 32, dtype=torch.int32, device="cuda") if want_mask else None
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if use_ws:
            ws = torch.empty(lsa.select_workspace_size(n), dtype=torch.uint8, device="cuda")
            lsa.select(z, seq_off, n, kept, capacity, ko, mask, ws, err)
        else:
            lsa.select_noalloc(z, seq_off, n, kept, capacity, ko, mask, err)
        torch.cuda.synchronize()
        outs.append((kept.cpu().numpy(), ko.cpu().numpy(), None if mask is None else mask.cpu().numpy(),
                     int(err.item())))
    return outs


CASES = [
    (np.array([0, 70000, 70001, 300000], np.int64), 0.1),     # many tiles, a one-entry sequence
    (np.array([0, 0, 5000, 5033, 9000], np.int64), -0.3),     # empty first sequence, ragged tail
]


@pytest.mark.parametrize("want_mask", [True, False], ids=["mask", "no_mask"])
def test_select_noalloc_matches_select_and_oracle_on_consecutive_calls(lsa, want_mask):
    rng = np.random.default_rng(20)
    for seq_off, shift in CASES:                                   # two calls in a row
        n = int(seq_off[-1])
        z = (rng.normal(size=n) + shift).astype(np.float32)
        z[::7] = -0.0
        (k_ws, o_ws, m_ws, e_ws), (k_na, o_na, m_na, e_na) = _select_both(lsa, z, seq_off, n, want_mask)
        assert e_ws == e_na == 0
        assert np.array_equal(o_ws, o_na)
        total = int(o_ws[-1])
        assert np.array_equal(k_ws[:total], k_na[:total])
        k_ref, ko_ref, m_ref = oracle.select(z.astype(np.float64), seq_off)
        assert np.array_equal(o_na, ko_ref) and np.array_equal(k_na[:total], k_ref)
        if want_mask:
            assert np.array_equal(m_ws, m_na)
            words = m_na.view(np.uint32)
            bits = np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little")[:n].astype(bool)
            assert np.array_equal(bits, m_ref)


def test_select_noalloc_capacity_overflow(lsa):
    """More kept entries than the output holds: LSA_ERR_CAPACITY, the true offsets, the first `capacity`
    indices written and nothing past them, as lsa_select does."""
    seq_off = np.array([0, 3000, 3100, 9000], np.int64)
    z = np.random.default_rng(8).normal(size=9000).astype(np.float32)
    k_ref, ko_ref, _ = oracle.select(z.astype(np.float64), seq_off)
    cap = len(k_ref) // 2
    (k_ws, o_ws, _, e_ws), (k_na, o_na, _, e_na) = _select_both(lsa, z, seq_off, cap)
    assert e_ws == e_na == 3                                   # LSA_ERR_CAPACITY
    assert np.array_equal(o_na, ko_ref) and np.array_equal(o_ws, ko_ref)
    assert np.array_equal(k_na[:cap], k_ref[:cap]) and np.array_equal(k_ws[:cap], k_ref[:cap])
    assert (k_na[cap:] == -5).all() and (k_ws[cap:] == -5).all()


def test_select_noalloc_rejects_sizes_above_its_scratch(lsa):
    big = lsa.select_noalloc_max_entries() + 1
    t = torch.zeros(2, dtype=torch.int64, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.select_noalloc(torch.zeros(1, device="cuda"), t, big, torch.zeros(1, dtype=torch.int32, device="cuda"),
                           1, t, None, None)
    assert e.value.status == 1
    assert "static scratch limit" in str(e.value)
