"""Parity of the merged attention set (top-k union recent window union HCA rows) with the oracle: the row
lists bit-exact (as entry identities), the attention over them within the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import ATTN_TOL, lsa_mod, read_ctx, rel_err_per_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


def _expected_arena_rows(topk_idx, topk_pos, seq_off, window, hca_off, win_base, hca_base, row_cap):
    """The oracle's attention set, written in arena rows (top-k entry -> its slot, window entry -> its window
    row, HCA row j -> hca_base + j), -1 padded to row_cap."""
    ref, cnt = oracle.attention_set(topk_idx, seq_off, window, hca_off)
    n_total = int(seq_off[-1])
    out = np.full((len(seq_off) - 1, row_cap), -1, np.int64)
    for b in range(len(seq_off) - 1):
        n_b = int(seq_off[b + 1] - seq_off[b])
        lo = n_b - min(window, n_b)
        slot = {int(e): int(s) for e, s in zip(topk_idx[b], topk_pos[b]) if e >= 0}
        rows = []
        for r in ref[b, :cnt[b]]:
            if r >= n_total:
                rows.append(hca_base + int(r) - n_total)
            else:
                e = int(r) - int(seq_off[b])
                rows.append(win_base + b * window + (e - lo) if e >= lo else slot[e])
        out[b, :min(len(rows), row_cap)] = rows[:row_cap]
    return out, cnt


def test_attn_set_merge_standalone_and_capacity(lsa):
    rng = np.random.default_rng(11)
    seq_off = np.array([0, 100, 100, 350, 360], np.int64)
    B, k, window = 4, 40, 30
    hca_off = np.array([0, 5, 5, 12, 13], np.int64)
    topk_idx = np.full((B, k), -1, np.int32)
    topk_pos = np.full((B, k), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    for b in range(B):
        n_b = int(seq_off[b + 1] - seq_off[b])
        c = min(n_b, [40, 0, 33, 10][b])
        sel = np.sort(rng.choice(n_b, size=c, replace=False))
        topk_idx[b, :c] = sel
        topk_pos[b, :c] = rng.choice(5000, size=c, replace=False)
        cnt[b] = c
    win_base, hca_base = 6000, 9000
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    args = [dev(topk_idx), dev(topk_pos), dev(cnt), dev(seq_off)]
    for row_cap, want_err in ((k + window + 7, 0), (50, 3)):
        rows = torch.full((B, row_cap), 123456, dtype=torch.int32, device="cuda")
        count = torch.zeros(B, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        lsa.attn_set_merge(*args, k, window, win_base, dev(hca_off), hca_base, rows, row_cap, count, err)
        torch.cuda.synchronize()
        exp, n = _expected_arena_rows(topk_idx, topk_pos, seq_off, window, hca_off, win_base, hca_base, row_cap)
        assert np.array_equal(rows.cpu().numpy(), exp)
        assert np.array_equal(count.cpu().numpy(), np.minimum(n, row_cap))
        assert err.item() == want_err
    # no HCA offsets and no window: the top-k slots themselves
    rows = torch.empty((B, k), dtype=torch.int32, device="cuda")
    lsa.attn_set_merge(*args, k, 0, win_base, None, hca_base, rows, k)
    torch.cuda.synchronize()
    assert np.array_equal(rows.cpu().numpy(), topk_pos)


@pytest.mark.parametrize("full_fetch", [False, True])
def test_merged_decode_matches_oracle(lsa, full_fetch):
    """Decode steps with a 300-entry window (longer than two of the sequences) and HCA rows (one per 128
    tokens): the context's attention rows are the oracle's attention set of the step's top-k, and the
    attention output and lse match the oracle's attention over that set."""
    from gpu_cases import make_context

    wl = synth.small_ragged(key_dtype="e4m3")
    hca, hca_off = synth.hca_rows(wl)
    dev = synth.to_torch(wl)
    window = 300
    base = make_context(wl, dev, lsa, tau=2, full_fetch=full_fetch)
    cap = base.kept_capacity
    base.close()
    hca_t = torch.from_numpy(hca.view(np.int16)).cuda()
    ctx = lsa.Context(B=wl.B, H=wl.H, d=wl.d, q_dtype=wl.q_dtype, k_dtype=wl.key_dtype, Hq=wl.Hq, D=wl.D,
                      attn_dtype=wl.attn_dtype, topk=wl.topk, seq_off_host=wl.seq_off, keys=dev["keys"],
                      k_scale=dev["k_scale"], cold_host=dev["cold"], row_bytes=wl.row_bytes,
                      kv_row_stride=wl.row_stride, k_off=wl.k_off, v_off=wl.v_off, kept_capacity=cap, tau=2,
                      scale=wl.scale, full_fetch=full_fetch, window=window, hca_rows=hca_t, hca_off_host=hca_off)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda")
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    kv = np.concatenate([wl.cold, hca])
    for t in range(3):
        q_t, w_t, Q_t = wl.step_inputs(t)
        ctx.step(t, synth.raw_to_torch(q_t), torch.from_numpy(w_t).cuda(), synth.raw_to_torch(Q_t), out, lse)
        torch.cuda.synchronize()
        g = read_ctx(ctx, wl, lsa)
        assert g["err"] == 0
        v = ctx.view()
        row_cap = int(v.attn_row_cap)
        assert row_cap == wl.topk + window + int(np.max(np.diff(hca_off)))
        rows = lsa.device_view(v.attn_rows, wl.B * row_cap, torch.int32).cpu().numpy().reshape(wl.B, row_cap)
        exp, n = _expected_arena_rows(g["topk_idx"], g["topk_pos"], wl.seq_off, window, hca_off, int(v.win_base),
                                      int(v.hca_base), row_cap)
        assert np.array_equal(rows, exp), t
        # the arena holds the rows the list names: window rows and HCA rows byte for byte
        hot = lsa.device_view(v.hot, (int(v.hca_base) + len(hca)) * wl.row_stride, torch.int16)
        hot = hot.cpu().numpy().view(np.uint16).reshape(-1, wl.row_stride)
        assert np.array_equal(hot[int(v.hca_base):], hca)
        for b in range(wl.B):
            n_b = int(wl.seq_off[b + 1] - wl.seq_off[b])
            w_b = min(window, n_b)
            w0 = int(v.win_base) + b * window
            assert np.array_equal(hot[w0:w0 + w_b], wl.cold[wl.seq_off[b + 1] - w_b:wl.seq_off[b + 1]])
        ref_rows, _ = oracle.attention_set(g["topk_idx"], wl.seq_off, window, hca_off)
        o_ref, l_ref = oracle.sparse_attn(Q_t, wl.attn_dtype, kv, wl.attn_dtype, wl.row_stride, wl.k_off, wl.v_off,
                                          ref_rows, wl.scale)
        o = oracle.decode(out.cpu().numpy().view(np.uint16), "bf16")
        rel = rel_err_per_head(o, o_ref)
        assert rel <= ATTN_TOL["bf16"], (t, rel)
        assert np.abs(lse.cpu().numpy() - l_ref).max() <= 1e-3
    ctx.close()
