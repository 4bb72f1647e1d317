"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding and compare it with the oracle under the stated tolerances.

Tolerances (CUDA path vs fp64 oracle, same seeded inputs):
  * selection mask, kept lists and top-k indices: bit-exact, except entries
    whose oracle I lies within 1e-5 of the 0.5 threshold (mask) or whose
    oracle z lies within 1e-5 * max(1, |z_k|) of the oracle's k-th largest z
    (top-k); stage-exact checks (oracle stage fed the GPU's own fp32 scores)
    allow no exception at all;
  * scores: |I - I_ref| <= 1e-3 and |z - z_ref| <= 4e-3 absolute;
  * attention: max|o - o_ref| / max|o_ref| per (sequence, head) <= 2e-2 for
    bf16 and 1e-4 for fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

I_BAND = 1e-5
Z_TOL = 4e-3
I_TOL = 1e-3
ATTN_TOL = {"bf16": 2e-2, "f32": 1e-4}


def lsa_mod():
    from lookahead_sparse_kv_index_b200 import lsa

    return lsa


def in_mask_band(z64: np.ndarray) -> np.ndarray:
    return np.abs(1.0 / (1.0 + np.exp(-z64)) - 0.5) < I_BAND


def topk_band(z_entry: float, z_k: float) -> bool:
    return abs(z_entry - z_k) <= 1e-5 * max(1.0, abs(z_k))


def unpack_mask(words: np.ndarray, n: int) -> np.ndarray:
    return np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little")[:n].astype(bool)


def gpu_full_scores(wl, dev, lsa, want_I=True, tc=False):
    """Full scan; tc=False forces the CUDA-core kernel (tc=True: tcgen05 where the shape is supported)."""
    n = wl.n_total
    z = torch.full((max(n, 1) + 64,), 77.0, dtype=torch.float32, device="cuda")
    I = torch.empty_like(z) if want_I else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.index_score(dev["q"], wl.q_dtype, dev["w"], dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"], n,
                    wl.H, wl.d, z, I, cuda_core=not tc, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0, f"device error {err.item()}"
    assert (z[n:].cpu().numpy() == 77.0).all(), "scan wrote past the entry axis"
    return z[:n].cpu().numpy(), (I[:n].cpu().numpy() if want_I else None)


def gpu_select(z_np, seq_off_np, lsa, capacity=None):
    n = int(seq_off_np[-1])
    B = len(seq_off_np) - 1
    cap = n if capacity is None else capacity
    z = torch.from_numpy(np.ascontiguousarray(z_np, np.float32)).cuda() if n else torch.zeros(1, device="cuda")
    seq_off = torch.from_numpy(seq_off_np.astype(np.int64)).cuda()
    kept_idx = torch.full((max(cap, 1),), -7, dtype=torch.int32, device="cuda")
    kept_off = torch.full((B + 1,), -7, dtype=torch.int64, device="cuda")
    mask = torch.zeros((n + 31) // 32 + 1, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(lsa.select_workspace_size(n), 16), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.select(z, seq_off, n, kept_idx, cap, kept_off, mask, ws, err)
    torch.cuda.synchronize()
    ko = kept_off.cpu().numpy()
    nk = min(int(ko[-1]), cap)
    return (kept_idx[:nk].cpu().numpy(), ko, unpack_mask(mask.cpu().numpy().view(np.uint32), n),
            int(err.item()))


def rel_err_per_head(out: np.ndarray, ref: np.ndarray) -> float:
    num = np.abs(out.astype(np.float64) - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max())


def decoded(raw: np.ndarray, dtype: str) -> np.ndarray:
    return oracle.decode(raw, dtype)


def make_context(wl, dev, lsa, kept_capacity=None, tau=64, full_fetch=False, lookahead=0):
    cap = kept_capacity or max(64, int(0.4 * wl.n_total) + 64)
    if wl.n_total <= 65536:
        cap = kept_capacity or wl.n_total + 64   # small cases may keep more than half the entries
    return lsa.Context(B=wl.B, H=wl.H, d=wl.d, q_dtype=wl.q_dtype, k_dtype=wl.key_dtype, Hq=wl.Hq, D=wl.D,
                       attn_dtype=wl.attn_dtype, topk=wl.topk, seq_off_host=wl.seq_off, keys=dev["keys"],
                       k_scale=dev["k_scale"], cold_host=dev["cold"], row_bytes=wl.row_bytes,
                       kv_row_stride=wl.row_stride, k_off=wl.k_off, v_off=wl.v_off, kept_capacity=cap, tau=tau,
                       scale=wl.scale, full_fetch=full_fetch, lookahead=lookahead)


def check_hot_cache(ctx, wl, lsa, gpu):
    """The hot buffer after a step: every kept entry's row sits in the slot its kept position names (the slot
    the attention reads), byte for byte, each in its own slot; the top-k slots are those of the chosen
    entries; slot_of and owner are inverse maps and every resident row is valid.  (After a cache flush with
    lookahead, the current set's rows stay in their slots while slot_of forgets them.)"""
    v = ctx.view()
    cap = ctx.kept_capacity
    slot_of = lsa.device_view(v.slot_of, wl.n_total, torch.int32).cpu().numpy()
    hot = lsa.device_view(v.hot, cap * ctx.row_bytes, torch.uint8).cpu().numpy().reshape(cap, ctx.row_bytes)
    cold = np.ascontiguousarray(wl.cold).view(np.uint8).reshape(wl.n_total, ctx.row_bytes)
    nk = len(gpu["kept_idx"])
    b_of = np.repeat(np.arange(wl.B), np.diff(gpu["kept_off"]))[:nk]
    ent = wl.seq_off[:-1][b_of] + gpu["kept_idx"]
    if v.kept_slot:
        slots = lsa.device_view(v.kept_slot, nk, torch.int32).cpu().numpy()
    else:                                    # every kept row fetched into kept order
        slots = slot_of[ent]
    assert (slots >= 0).all()
    assert len(np.unique(slots)) == len(slots)
    assert np.array_equal(hot[slots], cold[ent])
    if v.owner:
        owner = lsa.device_view(v.owner, cap, torch.int32).cpu().numpy()
        res = np.nonzero(slot_of >= 0)[0]
        assert np.array_equal(owner[slot_of[res]], res)
        assert np.array_equal(hot[slot_of[res]], cold[res])   # rows kept resident stay valid
    for b in range(wl.B):
        c = gpu["topk_cnt"][b]
        lo, hi = gpu["kept_off"][b], min(gpu["kept_off"][b + 1], nk)
        pos = lo + np.searchsorted(gpu["kept_idx"][lo:hi], gpu["topk_idx"][b][:c])
        assert np.array_equal(gpu["kept_idx"][pos], gpu["topk_idx"][b][:c])
        assert np.array_equal(gpu["topk_pos"][b][:c], slots[pos])


def read_ctx(ctx, wl, lsa):
    v = ctx.view()
    B, k = wl.B, wl.topk
    ko = lsa.device_view(v.kept_off, B + 1, torch.int64).cpu().numpy()
    nk = min(int(ko[-1]), ctx.kept_capacity)
    return dict(
        kept_off=ko,
        kept_idx=lsa.device_view(v.kept_idx, nk, torch.int32).cpu().numpy(),
        topk_idx=lsa.device_view(v.topk_idx, B * k, torch.int32).cpu().numpy().reshape(B, k),
        topk_pos=lsa.device_view(v.topk_pos, B * k, torch.int32).cpu().numpy().reshape(B, k),
        topk_cnt=lsa.device_view(v.topk_cnt, B, torch.int32).cpu().numpy(),
        err=int(lsa.device_view(v.err, 1, torch.int32).item()),
    )


def check_decode_step(wl, t, q_t, w_t, Q_t, gpu, out_gpu, lse_gpu, z_refresh, res_o):
    """Compare one GPU decode step with the oracle's; returns a dict of measured errors."""
    B, k = wl.B, wl.topk
    report = {}
    # kept set (fixed since the last refresh): equal outside the threshold band
    for b in range(B):
        g = set(gpu["kept_idx"][gpu["kept_off"][b]:gpu["kept_off"][b + 1]].tolist())
        o = set(res_o["kept_idx"][res_o["kept_off"][b]:res_o["kept_off"][b + 1]].tolist())
        diff = np.array(sorted(g ^ o), np.int64)
        if len(diff):
            assert in_mask_band(z_refresh[wl.seq_off[b] + diff]).all(), (b, diff[:10])
    # top-k sets: equal except swaps inside the k-th-score band (or the threshold band)
    cand = []
    for b in range(B):
        gsel = gpu["topk_idx"][b][: gpu["topk_cnt"][b]]
        osel = res_o["topk_idx"][b][: res_o["topk_cnt"][b]]
        assert (gpu["topk_idx"][b][gpu["topk_cnt"][b]:] == -1).all()
        assert (np.diff(gsel) > 0).all(), "top-k must be ascending"
        cand.append(np.union1d(gsel, osel).astype(np.int32))
    idx_off = np.concatenate([[0], np.cumsum([len(c) for c in cand])]).astype(np.int64)
    z_step = oracle.index_score_list(q_t, wl.q_dtype, w_t, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                     np.concatenate(cand) if idx_off[-1] else np.zeros(1, np.int32), idx_off,
                                     wl.H, wl.d)
    n_swaps = 0
    for b in range(B):
        zb = dict(zip(cand[b].tolist(), z_step[idx_off[b]:idx_off[b + 1]].tolist()))
        gsel = set(gpu["topk_idx"][b][: gpu["topk_cnt"][b]].tolist())
        osel = set(res_o["topk_idx"][b][: res_o["topk_cnt"][b]].tolist())
        if gsel == osel:
            continue
        z_k = min(zb[e] for e in osel) if osel else 0.0
        for e in gsel ^ osel:
            ok = topk_band(zb[e], z_k) or in_mask_band(np.array([z_refresh[wl.seq_off[b] + e]]))[0]
            assert ok, (b, e, zb[e], z_k)
            n_swaps += 1
    report["topk_swaps"] = n_swaps
    # attention over the GPU's own top-k rows vs the oracle's attention on the same rows
    out_ref, lse_ref = oracle.sparse_attn(Q_t, wl.attn_dtype, wl.cold, wl.attn_dtype, wl.row_stride, wl.k_off,
                                          wl.v_off, oracle.local_to_global(gpu["topk_idx"], wl.seq_off), wl.scale)
    if wl.attn_dtype == "bf16":
        out_g = oracle.decode(out_gpu.view(np.uint16), "bf16")
    else:
        out_g = out_gpu.astype(np.float64)
    rel = rel_err_per_head(out_g, out_ref)
    report["attn_rel"] = rel
    assert rel <= ATTN_TOL[wl.attn_dtype], rel
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin)
    report["lse_abs"] = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert report["lse_abs"] <= 1e-2
    return report


def run_decode_and_check(wl, steps, tau, lsa, kept_capacity=None, full_fetch=False, lookahead=0, flush_at=()):
    """Drive the context and the oracle decoder over `steps` (plus every window's first step and, with
    lookahead, every prediction step: both sides skip the same steps); check every step in `steps`.
    flush_at: steps before which the hot-buffer cache is emptied (a cold start)."""
    from oracle.stepper import OracleDecoder

    dev = synth.to_torch(wl)
    ctx = make_context(wl, dev, lsa, kept_capacity=kept_capacity, tau=tau, full_fetch=full_fetch,
                       lookahead=lookahead)
    dec = OracleDecoder(wl, tau=tau, lookahead=lookahead)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32 if wl.attn_dtype == "f32" else torch.int16,
                      device="cuda")
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    reports = []
    z_refresh = None
    last = max(steps)
    for t in range(last + 1):
        predict = lookahead > 0 and t % tau != 0 and (t + lookahead) % tau == 0
        if t not in steps and t % tau != 0 and not predict:
            continue
        if t in flush_at:
            ctx.flush_cache()
        q_t, w_t, Q_t = wl.step_inputs(t)
        ctx.step(t, synth.raw_to_torch(q_t), torch.from_numpy(w_t).cuda(), synth.raw_to_torch(Q_t), out, lse)
        torch.cuda.synchronize()
        res_o = dec.step(t, q_t, w_t, Q_t)
        z_refresh = res_o["z_sel"]   # the scores the current kept set was selected on
        if t in steps:
            gpu = read_ctx(ctx, wl, lsa)
            assert gpu["err"] == 0
            check_hot_cache(ctx, wl, lsa, gpu)
            rep = check_decode_step(wl, t, q_t, w_t, Q_t, gpu, out.cpu().numpy(), lse.cpu().numpy(), z_refresh,
                                    res_o)
            rep["t"] = t
            reports.append(rep)
    ctx.close()
    return reports
