"""The C ABI boundary, checked without a GPU: the library loads, exports every
symbol include/lsa.h declares, and rejects bad arguments on the host before
launching anything (no CUDA call is reached on these paths)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lsa():
    from lookahead_sparse_kv_index_b200 import build

    build.build()
    from lookahead_sparse_kv_index_b200 import lsa as mod

    return mod


def test_every_declared_symbol_is_exported(lsa):
    names = _declared()
    assert len(names) >= 19
    for n in names:
        assert hasattr(lsa.lib, n), n
    assert sorted(lsa.EXPORTS) == sorted(n for n in names)


def test_version_and_status_names(lsa):
    assert lsa.version() == 100
    assert lsa.lib.lsa_status_name(0) == b"LSA_OK"
    assert lsa.lib.lsa_status_name(3) == b"LSA_ERR_CAPACITY"


def test_workspace_sizes(lsa):
    assert lsa.select_workspace_size(0) == 0
    assert lsa.select_workspace_size(1) >= 16
    n = 4 * 131072
    assert lsa.select_workspace_size(n) >= (n // 1024) * 12 + n // 8
    assert lsa.sparse_attn_workspace_size(4, 128, 512, 2048) >= 4 * 32 * 128 * 514 * 4
    assert lsa.sparse_attn_workspace_size(0, 128, 512, 2048) == 0


def _score(lsa, **kw):
    a = dict(q=1 << 20, qd=1, w=1 << 20, k=1 << 20, kd=1, ks=None, so=1 << 20, n=100, idx=None, idxo=None,
             cap=0, B=1, H=64, d=128, z=1 << 20, I=None, flags=0)
    a.update(kw)
    return lsa.lib.lsa_index_score(a["q"], a["qd"], a["w"], a["k"], a["kd"], a["ks"], a["so"], a["n"], a["idx"],
                                   a["idxo"], a["cap"], a["B"], a["H"], a["d"], a["z"], a["I"], a["flags"], None,
                                   None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(z=None), 1), (dict(B=0), 1), (dict(H=65), 5), (dict(d=96), 5),
    (dict(kd=2), 1), (dict(ks=1 << 20), 1), (dict(k=(1 << 20) + 8), 1), (dict(qd=2), 5), (dict(qd=7), 1),
    (dict(idx=1 << 20), 1), (dict(n=-1), 1), (dict(flags=2), 1), (dict(flags=-1), 1),
])
def test_index_score_rejects_bad_arguments(lsa, kw, status):
    assert _score(lsa, **kw) == status
    assert lsa.lib.lsa_last_error() != b""


def test_other_entry_points_reject_bad_arguments(lsa):
    L, big = lsa.lib, 1 << 20
    assert L.lsa_select(None, big, 10, 1, big, 10, big, None, big, 1 << 20, None, None) == 1
    assert L.lsa_select(big, big, 10, 1, big, 10, big, None, big, 1, None, None) == 1          # workspace
    assert L.lsa_topk(big, 1, None, big, big, 10, 1, 32, big, None, big, None) == 1            # seq_off needed
    assert L.lsa_topk(big, 0, None, big, big, 10, 1, 5000, big, None, big, None) == 5          # k too large
    assert L.lsa_gather(big, 1000, big, 10, big, big, 1, big, 10, None, None, None) == 1       # row_bytes % 16
    assert L.lsa_sparse_attn(big, 1, big, 512, 0, 0, big, 1, 128, 48, 16, 1.0, big, None, big, 1 << 30, None, None) == 5
    assert L.lsa_sparse_attn(big, 2, big, 512, 0, 0, big, 1, 128, 512, 16, 1.0, big, None, big, 1 << 30, None, None) == 5
    assert L.lsa_sparse_attn(big, 1, big, 512, 0, 0, big, 1, 128, 512, 16, -1.0, big, None, big, 1 << 30, None, None) == 1
    assert L.lsa_sparse_attn(big, 1, big, 512, 0, 0, big, 1, 128, 512, 16, 1.0, big, None, big, 16, None, None) == 1
    assert L.lsa_selftest_bounded_wait(10, big, big, None) == 1              # limit below 1 us
    assert L.lsa_selftest_bounded_wait(1 << 40, big, big, None) == 1         # limit above 100 ms
    assert L.lsa_selftest_bounded_wait(1000000, None, big, None) == 1        # no error word
    arr = (ctypes.c_void_p * 3)(big, big, big)
    assert L.lsa_index_union(None, 3, 10, big, None) == 1                     # no layers
    assert L.lsa_index_union(arr, 0, 10, big, None) == 1                      # n_layers < 1
    assert L.lsa_index_union(arr, 9, 10, big, None) == 1                      # n_layers > 8
    assert L.lsa_index_union(arr, 3, -1, big, None) == 1                      # n_total < 0
    assert L.lsa_index_union(arr, 3, 10, None, None) == 1                     # no output
    arr[1] = None
    assert L.lsa_index_union(arr, 3, 10, big, None) == 1                      # a layer without scores


def _score_select(lsa, **kw):
    big = 1 << 20
    a = dict(q=big, qd=1, w=big, k=big, kd=1, ks=None, so=big, n=1000, B=2, H=64, d=128, z=big, kept=big, cap=1000,
             ko=big, ws=big, wsb=1 << 30)
    a.update(kw)
    return lsa.lib.lsa_index_score_select(a["q"], a["qd"], a["w"], a["k"], a["kd"], a["ks"], a["so"], a["n"], a["B"],
                                          a["H"], a["d"], a["z"], a["kept"], a["cap"], a["ko"], a["ws"], a["wsb"],
                                          None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(z=None), 1), (dict(ko=None), 1), (dict(ws=None), 1), (dict(B=0), 1),
    (dict(H=65), 5), (dict(d=96), 5), (dict(kd=2), 1), (dict(ks=1 << 20), 1), (dict(qd=2), 5),
    (dict(n=-1), 1), (dict(cap=-1), 1), (dict(kept=None), 1), (dict(wsb=16), 1), (dict(ws=(1 << 20) + 8), 1),
])
def test_index_score_select_rejects_bad_arguments(lsa, kw, status):
    assert _score_select(lsa, **kw) == status
    assert lsa.lib.lsa_last_error() != b""


def test_index_score_select_workspace_covers_both_paths(lsa):
    for n, B in [(1, 1), (1000, 3), (4 * 131072, 4), (2_200_000, 64)]:
        ws = lsa.index_score_select_workspace_size(n, B)
        assert ws >= lsa.select_workspace_size(n)          # the CUDA-core scan + lsa_select fallback
        # the fused path: per scan tile of >= 128 rows, 8 ballot words, 4 counts, base, first row, sequence
        assert ws >= ((n + 127) // 128 + B) * (32 + 16 + 8 + 8 + 4)


def test_struct_mirrors_match_the_header(lsa):
    assert lsa.lib.lsa_struct_size(0) == ctypes.sizeof(lsa.Params)
    assert lsa.lib.lsa_struct_size(1) == ctypes.sizeof(lsa.View)
    assert lsa.lib.lsa_struct_size(2) == -1


def test_encoder_and_merge_reject_bad_arguments(lsa):
    L, big = lsa.lib, 1 << 20
    ok = dict(h=big, B=4, hidden=7168, W_dq=big, rank=1536, W_uq=big, H=64, d=128, W_w=big, q=big, qdt=1, w=big,
              c=big)

    def enc(**kw):
        a = dict(ok, **kw)
        return L.lsa_query_encode(a["h"], a["B"], a["hidden"], a["W_dq"], a["rank"], a["W_uq"], a["H"], a["d"],
                                  a["W_w"], a["q"], a["qdt"], a["w"], a["c"], None)

    assert enc(h=None) == 1
    assert enc(c=None) == 1
    assert enc(B=0) == 1
    assert enc(hidden=7164) == 1          # not a multiple of 8
    assert enc(rank=4) == 1
    assert enc(H=0) == 1
    assert enc(W_uq=big + 2) == 1         # unaligned
    assert enc(qdt=2) == 5                # E4M3 queries are not produced
    # merge: topk_idx, topk_pos, topk_cnt, seq_off, B, k, window, win_base, hca_off, hca_base, rows, row_cap, ...
    assert L.lsa_attn_set_merge(None, big, big, big, 2, 32, 16, 0, None, 0, big, 64, None, None, None) == 1
    assert L.lsa_attn_set_merge(big, big, big, big, 2, 0, 16, 0, None, 0, big, 64, None, None, None) == 1
    assert L.lsa_attn_set_merge(big, big, big, big, 2, 32, -1, 0, None, 0, big, 64, None, None, None) == 1
    assert L.lsa_attn_set_merge(big, big, big, big, 2, 32, 16, 0, None, 0, big, 0, None, None, None) == 1
    assert L.lsa_attn_set_merge(big, big, big, big, 2, 32, 1 << 30, 1 << 30, None, 0, big, 64, None, None,
                                None) == 1                                              # rows overflow int32
    assert L.lsa_sparse_attn(big, 1, big, 512, 0, 0, big, 1, 128, 512, 70000, 1.0, big, None, big, 1 << 40, None,
                             None) == 5                                                 # k above 65536


def test_ctx_create_rejects_bad_params(lsa):
    import numpy as np

    so = np.array([0, 10, 5], np.int64)
    p = lsa.Params(2, 64, 128, 1, 1, 128, 512, 1, 2048, 64, 0.0, 5, so.ctypes.data, 1 << 20, None, 1 << 20,
                   1024, 512, 0, 0, 100)
    h = ctypes.c_void_p()
    assert lsa.lib.lsa_ctx_create(ctypes.byref(p), ctypes.byref(h)) == 1   # seq_off decreasing
    p.kv_row_stride = 256
    assert lsa.lib.lsa_ctx_create(ctypes.byref(p), ctypes.byref(h)) == 1   # stride * 2 != row_bytes
    so[:] = [0, 3, 5]
    p.kv_row_stride = 512
    p.window = -1
    assert lsa.lib.lsa_ctx_create(ctypes.byref(p), ctypes.byref(h)) == 1   # negative window
    p.window = 16
    p.hca_rows = 1 << 20
    assert lsa.lib.lsa_ctx_create(ctypes.byref(p), ctypes.byref(h)) == 1   # HCA rows without offsets
    p.hca_rows = None
    p.window = 0
    def rejected(why):
        return lsa.lib.lsa_ctx_create(ctypes.byref(p), ctypes.byref(h)) == 1 and why in lsa.lib.lsa_last_error().decode()

    p.n_layers = 9
    assert rejected("n_layers=9")                    # more than 8 indexer layers
    p.n_layers = 3
    assert rejected("needs k_dev_layers")            # layers without their keys
    arr = (ctypes.c_void_p * 2)(1 << 20, None)
    p.k_dev_layers = ctypes.cast(arr, ctypes.c_void_p)
    assert rejected("layer 2 has no keys")
    assert h.value is None
