"""lsa_select_noalloc, the selection for callers that cannot allocate device
memory (its scratch is a static array inside the library), against lsa_select
with a caller workspace: identical kept lists, offsets and masks on two calls in
a row (the second call finds the first call's scratch contents), and sizes above
the static limit rejected before any launch.  Collected last on purpose."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from lookahead_sparse_kv_index_b200 import lsa as mod

    return mod


def _select_both(lsa, z_np, seq_off_np, capacity):
    n = int(seq_off_np[-1])
    B = len(seq_off_np) - 1
    z = torch.from_numpy(z_np).cuda()
    seq_off = torch.from_numpy(seq_off_np).cuda()
    outs = []
    for use_ws in (True, False):
        kept = torch.full((capacity,), -5, dtype=torch.int32, device="cuda")
        ko = torch.full((B + 1,), -5, dtype=torch.int64, device="cuda")
        mask = torch.zeros((n + 31) // 32, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if use_ws:
            ws = torch.empty(lsa.select_workspace_size(n), dtype=torch.uint8, device="cuda")
            lsa.select(z, seq_off, n, kept, capacity, ko, mask, ws, err)
        else:
            lsa.select_noalloc(z, seq_off, n, kept, capacity, ko, mask, err)
        torch.cuda.synchronize()
        outs.append((kept.cpu().numpy(), ko.cpu().numpy(), mask.cpu().numpy(), int(err.item())))
    return outs


def test_select_noalloc_matches_select_on_consecutive_calls(lsa):
    rng = np.random.default_rng(20)
    cases = [
        (np.array([0, 70000, 70001, 300000], np.int64), 0.1),     # many tiles, a one-entry sequence
        (np.array([0, 0, 5000, 5033, 9000], np.int64), -0.3),     # empty first sequence, ragged tail
    ]
    for seq_off, shift in cases:                                   # two calls in a row
        n = int(seq_off[-1])
        z = (rng.normal(size=n) + shift).astype(np.float32)
        z[::7] = -0.0
        (k_ws, o_ws, m_ws, e_ws), (k_na, o_na, m_na, e_na) = _select_both(lsa, z, seq_off, n)
        assert e_ws == e_na == 0
        assert np.array_equal(o_ws, o_na)
        total = int(o_ws[-1])
        assert np.array_equal(k_ws[:total], k_na[:total])
        assert np.array_equal(m_ws, m_na)


def test_select_noalloc_rejects_sizes_above_its_scratch(lsa):
    big = lsa.select_noalloc_max_entries() + 1
    t = torch.zeros(2, dtype=torch.int64, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.select_noalloc(torch.zeros(1, device="cuda"), t, big, torch.zeros(1, dtype=torch.int32, device="cuda"),
                           1, t, None, None)
    assert e.value.status == 1
    assert "static scratch limit" in str(e.value)
