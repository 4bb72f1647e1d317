"""Decode with the OR-mode union of three indexer layers in the cadence, against the oracle decoder: every
refresh keeps what any layer keeps and every step ranks the kept set by the union score."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import ATTN_TOL, in_mask_band, lsa_mod, make_context, read_ctx, rel_err_per_head, topk_band

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


@pytest.mark.parametrize("key_dtype,full_fetch", [("e4m3", False), ("bf16", True)])
def test_decode_three_layer_union_matches_oracle(lsa, key_dtype, full_fetch):
    from oracle.stepper import OracleDecoder

    wls = [synth.small_ragged(seed=5 + 10 * l, key_dtype=key_dtype) for l in range(3)]
    wl = wls[0]   # layer 0 also carries the cold pool and the attention queries
    assert all(np.array_equal(x.seq_off, wl.seq_off) for x in wls)
    devs = [synth.to_torch(x, pin_cold=(l == 0)) for l, x in enumerate(wls)]
    base = make_context(wl, devs[0], lsa, tau=4)
    cap = base.kept_capacity
    base.close()
    layers = [(devs[l]["keys"], devs[l]["k_scale"]) for l in (1, 2)]
    ctx = lsa.Context(B=wl.B, H=wl.H, d=wl.d, q_dtype=wl.q_dtype, k_dtype=wl.key_dtype, Hq=wl.Hq, D=wl.D,
                      attn_dtype=wl.attn_dtype, topk=wl.topk, seq_off_host=wl.seq_off, keys=devs[0]["keys"],
                      k_scale=devs[0]["k_scale"], cold_host=devs[0]["cold"], row_bytes=wl.row_bytes,
                      kv_row_stride=wl.row_stride, k_off=wl.k_off, v_off=wl.v_off, kept_capacity=cap, tau=4,
                      scale=wl.scale, full_fetch=full_fetch, layers=layers)
    assert ctx.n_layers == 3
    dec = OracleDecoder(wl, tau=4, layers=[(wls[l].keys, wls[l].k_scale) for l in (1, 2)])
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.int16, device="cuda")
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    z_union = None
    single = []
    for t in range(6):
        ins = [x.step_inputs(t) for x in wls]
        q = np.stack([i[0] for i in ins])
        w = np.stack([np.ascontiguousarray(i[1]) for i in ins])
        Q = ins[0][2]
        ctx.step(t, synth.raw_to_torch(q), torch.from_numpy(w).cuda(), synth.raw_to_torch(Q), out, lse)
        torch.cuda.synchronize()
        res = dec.step(t, q, w, Q)
        g = read_ctx(ctx, wl, lsa)
        assert g["err"] == 0
        if "z" in res:
            z_union = res["z"]
            # the union keeps more than any single layer: each layer's own kept set is inside it
            for l in range(3):
                zl = oracle.index_score(q[l], wl.q_dtype, w[l], wls[l].keys, key_dtype, wls[l].k_scale,
                                        wl.seq_off, wl.H, wl.d, want_I=False)
                assert np.all(z_union[zl >= 0] >= 0)
                single.append(int((zl >= 0).sum()))
            assert int((z_union >= 0).sum()) >= max(single[-3:])
        # kept sets: equal outside the threshold band of the union score
        for b in range(wl.B):
            gk = set(g["kept_idx"][g["kept_off"][b]:g["kept_off"][b + 1]].tolist())
            ok = set(res["kept_idx"][res["kept_off"][b]:res["kept_off"][b + 1]].tolist())
            diff = np.array(sorted(gk ^ ok), np.int64)
            if len(diff):
                assert in_mask_band(z_union[wl.seq_off[b] + diff]).all(), (t, b, diff[:8])
        # top-k: equal except swaps inside the band of the k-th union score (oracle scores of the kept set)
        b_of = np.repeat(np.arange(wl.B), np.diff(res["kept_off"]))
        zk = {(int(b), int(e)): float(v) for b, e, v in zip(b_of, res["kept_idx"], res["zk"])}
        for b in range(wl.B):
            gsel = set(g["topk_idx"][b][:g["topk_cnt"][b]].tolist())
            osel = set(res["topk_idx"][b][:res["topk_cnt"][b]].tolist())
            if gsel == osel:
                continue
            z_k = min(zk[(b, e)] for e in osel)
            for e in gsel ^ osel:
                ze = zk.get((b, e))
                assert (ze is not None and topk_band(ze, z_k)) or in_mask_band(
                    np.array([z_union[wl.seq_off[b] + e]]))[0], (t, b, e, ze, z_k)
        # attention over the GPU's own top-k rows
        o_ref, l_ref = oracle.sparse_attn(Q, wl.attn_dtype, wl.cold, wl.attn_dtype, wl.row_stride, wl.k_off,
                                          wl.v_off, oracle.local_to_global(g["topk_idx"], wl.seq_off), wl.scale)
        o = oracle.decode(out.cpu().numpy().view(np.uint16), "bf16")
        assert rel_err_per_head(o, o_ref) <= ATTN_TOL["bf16"]
        fin = np.isfinite(l_ref)
        assert np.abs(lse.cpu().numpy()[fin] - l_ref[fin]).max() <= 1e-2   # the decode-step bound (bf16 P)
    ctx.close()
