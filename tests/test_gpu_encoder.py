"""Parity of the indexer query encoder (lsa_query_encode) with the fp64 oracle.

Tolerances follow from the arithmetic: every product of the bf16 operands is
exact in fp32, and each output is an fp32 sum of K such products whose longest
sequential chain is under 256 additions (32 lanes x 8 elements per chunk, a
5-level lane tree, at most 8 K splits), so |error| <= 2e-5 * sum_k |W_nk x_k|
per output (first-order bound n * 2^-24 with n < 330, with headroom).  q adds
the propagated error of c and, for bf16 output, the round-to-nearest-even step
(<= 2^-9 relative).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import lsa_mod

pytestmark = pytest.mark.gpu

SUM_TOL = 2e-5


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def _run(lsa, h, ew, q_dtype):
    B = h.shape[0]
    q = torch.empty((B, ew.H, ew.d), dtype=torch.int16 if q_dtype == "bf16" else torch.float32, device="cuda")
    w = torch.empty((B, ew.H), dtype=torch.float32, device="cuda")
    c = torch.empty((B, ew.rank), dtype=torch.float32, device="cuda")
    lsa.query_encode(_dev(h), _dev(ew.W_dq), _dev(ew.W_uq), _dev(ew.W_w), ew.H, ew.d, q, q_dtype, w, c)
    torch.cuda.synchronize()
    qn = q.cpu().numpy()
    if q_dtype == "bf16":
        qn = oracle.decode(qn.view(np.uint16), "bf16")
    return c.cpu().numpy().astype(np.float64), qn.astype(np.float64), w.cpu().numpy().astype(np.float64)


def _bounds(h, ew, c_ref, q_dtype):
    hd = oracle.decode(h, "bf16")
    Dq, Uq, Ww = (oracle.decode(a, "bf16") for a in (ew.W_dq, ew.W_uq, ew.W_w))
    tol_c = SUM_TOL * (np.abs(hd) @ np.abs(Dq).T) + 1e-30
    tol_w = SUM_TOL * (np.abs(hd) @ np.abs(Ww).T) + 1e-30
    # q: error of c carried through W_uq, plus the second sum's own rounding
    tol_q = tol_c @ np.abs(Uq).T + SUM_TOL * (np.abs(c_ref) @ np.abs(Uq).T)
    return tol_c, tol_q.reshape(h.shape[0], ew.H, ew.d), tol_w


def _check(lsa, B, hidden, rank, H, d, q_dtype, seed):
    ew = synth.encoder_weights(seed, H, d, hidden=hidden, rank=rank)
    h = synth.hidden_states(seed, B, hidden=hidden)
    c_ref, q_ref, w_ref = oracle.query_encode(h, "bf16", ew.W_dq, ew.W_uq, ew.W_w, "bf16", H, d)
    c, q, w = _run(lsa, h, ew, q_dtype)
    tol_c, tol_q, tol_w = _bounds(h, ew, c_ref, q_dtype)
    if q_dtype == "bf16":
        tol_q = tol_q + 2.0 ** -9 * np.abs(q_ref) * (1 + 1e-3) + 1e-30
    assert np.all(np.abs(c - c_ref) <= tol_c), np.max(np.abs(c - c_ref) / tol_c)
    assert np.all(np.abs(w - w_ref) <= tol_w), np.max(np.abs(w - w_ref) / tol_w)
    assert np.all(np.abs(q - q_ref) <= tol_q), np.max(np.abs(q - q_ref) / tol_q)
    return c, q, w


@pytest.mark.parametrize("B,hidden,rank,H,d,q_dtype", [
    (1, 1000, 72, 4, 24, "bf16"),     # ragged last chunk in both passes, one batch row
    (2, 264, 16, 3, 40, "f32"),       # K of one partial chunk; NB = 2
    (3, 2056, 520, 5, 32, "bf16"),    # batch tail inside a group of 4; rows in ragged groups
    (7, 512, 264, 8, 16, "f32"),      # two batch groups, the second partial
    (4, 4096, 256, 64, 128, "bf16"),  # the decode head shape with a short latent
])
def test_query_encode_matches_oracle(lsa, B, hidden, rank, H, d, q_dtype):
    _check(lsa, B, hidden, rank, H, d, q_dtype, seed=B * 13 + H)


def test_query_encode_full_size(lsa):
    """The default encoder shape (hidden 7168, rank 1536, 64 heads of d = 128) at batch 4, in the launch
    configuration the benchmark times; every output against the oracle."""
    _check(lsa, 4, synth.ENCODER_HIDDEN, synth.ENCODER_RANK, 64, 128, "bf16", seed=41)


def test_query_encode_deterministic_and_batch_independent(lsa):
    """Repeated calls give the same bits, and a sequence's outputs do not depend on its batch neighbours."""
    ew = synth.encoder_weights(3, 8, 32, hidden=1024, rank=128)
    h = synth.hidden_states(3, 6, hidden=1024)
    a = _run(lsa, h, ew, "f32")
    b = _run(lsa, h, ew, "f32")
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    one = _run(lsa, h[4:5], ew, "f32")
    for x, y in zip(a, one):
        assert np.array_equal(x[4:5], y)


def test_query_encode_feeds_the_scan(lsa):
    """The encoder's (q, w) go straight into lsa_index_score: the scores equal the oracle's scores of the
    oracle's own (q, w) within the scan tolerance plus the encoder's rounding carried through."""
    from gpu_cases import Z_TOL

    wl = synth.small_ragged(key_dtype="bf16")
    ew = synth.encoder_weights(9, wl.H, wl.d, hidden=2048, rank=256)
    h = synth.hidden_states(9, wl.B, hidden=2048)
    _, q_ref, w_ref = oracle.query_encode(h, "bf16", ew.W_dq, ew.W_uq, ew.W_w, "bf16", wl.H, wl.d)
    q = torch.empty((wl.B, wl.H, wl.d), dtype=torch.int16, device="cuda")
    w = torch.empty((wl.B, wl.H), dtype=torch.float32, device="cuda")
    c = torch.empty((wl.B, ew.rank), dtype=torch.float32, device="cuda")
    lsa.query_encode(_dev(h), _dev(ew.W_dq), _dev(ew.W_uq), _dev(ew.W_w), wl.H, wl.d, q, "bf16", w, c)
    dev = synth.to_torch(wl)
    n = wl.n_total
    z = torch.empty(n, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.index_score(q, "bf16", w, dev["keys"], wl.key_dtype, dev["k_scale"], dev["seq_off"], n, wl.H, wl.d, z,
                    None, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    # the oracle scores the GPU's (q, w) exactly; compare the GPU's scan of them
    q_bits = q.cpu().numpy().view(np.uint16)
    z_ref = oracle.index_score(q_bits, "bf16", w.cpu().numpy(), wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                               wl.H, wl.d, want_I=False)
    assert np.max(np.abs(z.cpu().numpy() - z_ref)) <= Z_TOL
    # and the encoder's (q, w) are the oracle's up to the bf16 rounding of q
    qd = oracle.decode(q_bits, "bf16")
    assert np.max(np.abs(qd - q_ref)) <= 2.0 ** -8 * np.max(np.abs(q_ref))
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=1e-4, atol=1e-7)
