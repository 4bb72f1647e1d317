"""Thin ctypes binding of liblsa.so (include/lsa.h).

Argument marshalling only: torch tensors supply device memory and streams,
every step of the path runs in the library's CUDA kernels.  There is no CPU
fallback: if liblsa.so is missing or cannot be loaded, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lookahead_sparse_kv_index_b200.build`")
_L = ctypes.CDLL(LIB_PATH)

P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

F32, BF16, E4M3 = 0, 1, 2
DTYPE = {"f32": F32, "bf16": BF16, "e4m3": E4M3}
STATUS = {0: "LSA_OK", 1: "LSA_ERR_INVALID", 2: "LSA_ERR_CUDA", 3: "LSA_ERR_CAPACITY", 4: "LSA_ERR_TIMEOUT",
          5: "LSA_ERR_UNSUPPORTED"}
(STAGE_SCORE, STAGE_SELECT, STAGE_GATHER, STAGE_TOPK, STAGE_ATTN, STAGE_RESCORE) = range(6)
STAGES = ["score", "select", "gather", "topk", "attn", "rescore"]
N_STAGES = 6

# every symbol include/lsa.h declares
EXPORTS = [
    "lsa_version", "lsa_last_error", "lsa_last_kernel", "lsa_status_name", "lsa_index_score",
    "lsa_select_workspace_size", "lsa_select_noalloc_max_entries", "lsa_select_noalloc",
    "lsa_select", "lsa_topk", "lsa_gather", "lsa_sparse_attn_workspace_size", "lsa_sparse_attn",
    "lsa_ctx_create", "lsa_ctx_destroy", "lsa_decode_step", "lsa_decode_step_host", "lsa_ctx_get_view",
    "lsa_ctx_set_graphs", "lsa_ctx_set_timing", "lsa_ctx_stage_times", "lsa_ctx_reset_counters",
    "lsa_ctx_launches", "lsa_selftest_bounded_wait", "lsa_index_union", "lsa_query_encode",
    "lsa_attn_set_merge", "lsa_struct_size", "lsa_ctx_flush_cache", "lsa_index_score_select_workspace_size",
    "lsa_index_score_select",
]


class LsaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = _L.lsa_last_error().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


class Params(ctypes.Structure):
    _fields_ = [
        ("B", i32), ("H", i32), ("d", i32), ("q_dtype", i32), ("k_dtype", i32),
        ("Hq", i32), ("D", i32), ("attn_dtype", i32), ("topk", i32), ("tau", i32), ("scale", f32),
        ("n_total", i64), ("seq_off_host", P), ("k_dev", P), ("k_scale_dev", P), ("cold_host", P),
        ("row_bytes", i64), ("kv_row_stride", i64), ("k_off", i64), ("v_off", i64), ("kept_capacity", i64),
        ("full_fetch", i32), ("window", i32), ("hca_rows", P), ("hca_off_host", P),
        ("n_layers", i32), ("k_dev_layers", P), ("k_scale_layers", P), ("lookahead", i32),
    ]


class View(ctypes.Structure):
    _fields_ = [("z", P), ("z_kept", P), ("kept_idx", P), ("kept_off", P), ("slot_of", P), ("hot", P),
                ("topk_idx", P), ("topk_pos", P), ("topk_cnt", P), ("err", P), ("kept_slot", P), ("owner", P),
                ("fetched", P), ("attn_rows", P), ("attn_row_cap", i64), ("win_base", i64), ("hca_base", i64)]


def _sig(name, res, args):
    f = getattr(_L, name)
    f.restype = res
    f.argtypes = args


_sig("lsa_version", i32, [])
_sig("lsa_struct_size", i64, [i32])
_sig("lsa_last_error", ctypes.c_char_p, [])
_sig("lsa_last_kernel", ctypes.c_char_p, [])
_sig("lsa_status_name", ctypes.c_char_p, [i32])
_sig("lsa_index_score", i32, [P, i32, P, P, i32, P, P, i64, P, P, i64, i32, i32, i32, P, P, i32, P, P])
SCORE_CUDA_CORE = 1
_sig("lsa_select_workspace_size", sz, [i64])
_sig("lsa_index_score_select_workspace_size", sz, [i64, i32])
_sig("lsa_index_score_select", i32, [P, i32, P, P, i32, P, P, i64, i32, i32, i32, P, P, i64, P, P, sz, P, P])
_sig("lsa_select", i32, [P, P, i64, i32, P, i64, P, P, P, sz, P, P])
_sig("lsa_select_noalloc_max_entries", i64, [])
_sig("lsa_select_noalloc", i32, [P, P, i64, i32, P, i64, P, P, P, P])
_sig("lsa_topk", i32, [P, i32, P, P, P, i64, i32, i32, P, P, P, P])
_sig("lsa_gather", i32, [P, i64, P, i64, P, P, i32, P, i64, P, P, P])
_sig("lsa_sparse_attn_workspace_size", sz, [i32, i32, i32, i32])
_sig("lsa_sparse_attn", i32, [P, i32, P, i64, i64, i64, P, i32, i32, i32, i32, f32, P, P, P, sz, P, P])
_sig("lsa_ctx_create", i32, [ctypes.POINTER(Params), ctypes.POINTER(P)])
_sig("lsa_ctx_destroy", i32, [P])
_sig("lsa_decode_step", i32, [P, i64, P, P, P, P, P, P])
_sig("lsa_decode_step_host", i32, [P, i64, P, P, P, P, P, P])
_sig("lsa_ctx_get_view", i32, [P, ctypes.POINTER(View)])
_sig("lsa_ctx_set_graphs", i32, [P, i32])
_sig("lsa_ctx_set_timing", i32, [P, i32])
_sig("lsa_ctx_stage_times", i32, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)])
_sig("lsa_ctx_reset_counters", i32, [P])
_sig("lsa_ctx_launches", i64, [P])
_sig("lsa_ctx_flush_cache", i32, [P, P])
_sig("lsa_selftest_bounded_wait", i32, [i64, P, P, P])
_sig("lsa_index_union", i32, [ctypes.POINTER(P), i32, i64, P, P])
_sig("lsa_query_encode", i32, [P, i32, i32, P, i32, P, i32, i32, P, P, i32, P, P, P])
_sig("lsa_attn_set_merge", i32, [P, P, P, P, i32, i32, i32, i32, P, i32, P, i32, P, P, P])

lib = _L


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status, where):
    if status != 0:
        raise LsaError(status, where)


def version() -> int:
    return int(_L.lsa_version())


def last_kernel() -> str:
    """Name of the last kernel this thread launched through the library."""
    return _L.lsa_last_kernel().decode()


# ------------------------------------------------------------------ stages

def index_score(q, q_dtype, w, k, k_dtype, k_scale, seq_off, n_total, H, d, z, I=None, idx=None, idx_off=None,
                list_capacity=0, cuda_core=False, err=None, stream=None):
    """Lookahead index score; cuda_core=True forces the CUDA-core kernel (else tcgen05 where supported)."""
    B = seq_off.numel() - 1
    _check(_L.lsa_index_score(_ptr(q), DTYPE[q_dtype], _ptr(w), _ptr(k), DTYPE[k_dtype], _ptr(k_scale),
                              _ptr(seq_off), n_total, _ptr(idx), _ptr(idx_off), list_capacity, B, H, d,
                              _ptr(z), _ptr(I), SCORE_CUDA_CORE if cuda_core else 0, _ptr(err), _stream(stream)),
           "lsa_index_score")


def select_workspace_size(n_total) -> int:
    return int(_L.lsa_select_workspace_size(n_total))


def index_score_select_workspace_size(n_total, B) -> int:
    return int(_L.lsa_index_score_select_workspace_size(n_total, B))


def index_score_select(q, q_dtype, w, k, k_dtype, k_scale, seq_off, n_total, H, d, z, kept_idx, capacity, kept_off,
                       workspace, err=None, stream=None):
    """Full index scan and threshold selection in one call (fused on the tensor-core path; see lsa.h)."""
    B = seq_off.numel() - 1
    _check(_L.lsa_index_score_select(_ptr(q), DTYPE[q_dtype], _ptr(w), _ptr(k), DTYPE[k_dtype], _ptr(k_scale),
                                     _ptr(seq_off), n_total, B, H, d, _ptr(z), _ptr(kept_idx), capacity,
                                     _ptr(kept_off), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _ptr(err), _stream(stream)), "lsa_index_score_select")


def select(z, seq_off, n_total, kept_idx, capacity, kept_off, mask, workspace, err, stream=None):
    B = seq_off.numel() - 1
    _check(_L.lsa_select(_ptr(z), _ptr(seq_off), n_total, B, _ptr(kept_idx), capacity, _ptr(kept_off), _ptr(mask),
                         _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err),
                         _stream(stream)), "lsa_select")


def select_noalloc_max_entries() -> int:
    return int(_L.lsa_select_noalloc_max_entries())


def select_noalloc(z, seq_off, n_total, kept_idx, capacity, kept_off, mask, err, stream=None):
    """lsa_select with the library's static scratch instead of a caller workspace."""
    B = seq_off.numel() - 1
    _check(_L.lsa_select_noalloc(_ptr(z), _ptr(seq_off), n_total, B, _ptr(kept_idx), capacity, _ptr(kept_off),
                                 _ptr(mask), _ptr(err), _stream(stream)), "lsa_select_noalloc")


def index_union(z_layers, n_total, z_union, stream=None):
    """OR-mode union of indexer layers: z_union = max over the layers' scores (see lsa.h)."""
    arr = (P * len(z_layers))(*[_ptr(z) for z in z_layers])
    _check(_L.lsa_index_union(arr, len(z_layers), n_total, _ptr(z_union), _stream(stream)), "lsa_index_union")


def query_encode(h, W_dq, W_uq, W_w, H, d, q_out, q_dtype, w_out, c_out, stream=None):
    """Indexer query encoder: c = W_dq h, q = W_uq c as [B,H,d], w = W_w h (see lsa.h).  h: bf16 [B,hidden];
    W_dq [rank,hidden], W_uq [H*d,rank], W_w [H,hidden] bf16 (any 2-byte tensors holding bf16 bits)."""
    B, hidden = h.shape
    rank = W_dq.shape[0]
    _check(_L.lsa_query_encode(_ptr(h), B, hidden, _ptr(W_dq), rank, _ptr(W_uq), H, d, _ptr(W_w), _ptr(q_out),
                               DTYPE[q_dtype], _ptr(w_out), _ptr(c_out), _stream(stream)), "lsa_query_encode")


def attn_set_merge(topk_idx, topk_pos, topk_cnt, seq_off, k, window, win_base, hca_off, hca_base, rows, row_cap,
                   count=None, err=None, stream=None):
    """Merged attention set: per sequence the row list top-k (outside the window) + HCA rows + window rows."""
    B = seq_off.numel() - 1
    _check(_L.lsa_attn_set_merge(_ptr(topk_idx), _ptr(topk_pos), _ptr(topk_cnt), _ptr(seq_off), B, k, window,
                                 win_base, _ptr(hca_off), hca_base, _ptr(rows), row_cap, _ptr(count), _ptr(err),
                                 _stream(stream)), "lsa_attn_set_merge")


def selftest_bounded_wait(limit_ns, err, waited_ns, stream=None):
    """Runs a bounded device wait on a barrier nothing arrives at (see lsa.h)."""
    _check(_L.lsa_selftest_bounded_wait(int(limit_ns), _ptr(err), _ptr(waited_ns), _stream(stream)),
           "lsa_selftest_bounded_wait")


def topk(z, z_by_entry, seq_off, kept_idx, kept_off, kept_capacity, k, topk_idx, topk_pos, topk_cnt, stream=None):
    B = kept_off.numel() - 1
    _check(_L.lsa_topk(_ptr(z), int(z_by_entry), _ptr(seq_off), _ptr(kept_idx), _ptr(kept_off), kept_capacity, B, k,
                       _ptr(topk_idx), _ptr(topk_pos), _ptr(topk_cnt), _stream(stream)), "lsa_topk")


def gather(cold_host, row_bytes, seq_off, n_total, kept_idx, kept_off, hot, hot_capacity, slot_of, err,
           stream=None):
    B = seq_off.numel() - 1
    _check(_L.lsa_gather(_ptr(cold_host), row_bytes, _ptr(seq_off), n_total, _ptr(kept_idx), _ptr(kept_off), B,
                         _ptr(hot), hot_capacity, _ptr(slot_of), _ptr(err), _stream(stream)), "lsa_gather")


def sparse_attn_workspace_size(B, Hq, D, k) -> int:
    return int(_L.lsa_sparse_attn_workspace_size(B, Hq, D, k))


def sparse_attn(Q, dtype, kv, kv_row_stride, k_off, v_off, rows, B, Hq, D, k, scale, out, lse, workspace,
                err=None, stream=None):
    _check(_L.lsa_sparse_attn(_ptr(Q), DTYPE[dtype], _ptr(kv), kv_row_stride, k_off, v_off, _ptr(rows), B, Hq, D,
                              k, float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(err), _stream(stream)),
           "lsa_sparse_attn")


# ----------------------------------------------------------- decode context

class Context:
    """Owns an lsa_ctx: the tau-cadence decode loop over device-resident keys and a pinned cold pool.

    The caller keeps `keys`, `k_scale` and `cold_host` alive for the context's lifetime.
    """

    def __init__(self, *, B, H, d, q_dtype, k_dtype, Hq, D, attn_dtype, topk, seq_off_host, keys, k_scale,
                 cold_host, row_bytes, kv_row_stride, k_off, v_off, kept_capacity, tau=64, scale=0.0,
                 full_fetch=False, window=0, hca_rows=None, hca_off_host=None, layers=None, lookahead=0):
        """window / hca_rows / hca_off_host: the always-resident context merged into the attention set
        (see lsa_attn_set_merge); hca_rows is a host or device tensor of HCA rows in the cold-pool row format.
        layers: [(keys, k_scale), ...] of indexer layers 1 .. L-1 (layer 0 is keys / k_scale) for the OR-mode
        union in the cadence; steps then take q [L, B, H, d] and w [L, B, H].
        lookahead: predict each window's kept set this many steps ahead and fetch it meanwhile (see lsa.h)."""
        self._seq_off = torch.as_tensor(seq_off_host, dtype=torch.int64).contiguous()
        self._hca_off = None if hca_off_host is None else torch.as_tensor(hca_off_host, dtype=torch.int64).contiguous()
        n_total = int(self._seq_off[-1])
        self.params = Params(B, H, d, DTYPE[q_dtype], DTYPE[k_dtype], Hq, D, DTYPE[attn_dtype], topk, tau,
                             float(scale), n_total, self._seq_off.data_ptr(), _ptr(keys), _ptr(k_scale),
                             _ptr(cold_host), row_bytes, kv_row_stride, k_off, v_off, kept_capacity,
                             int(bool(full_fetch)), int(window), _ptr(hca_rows),
                             None if self._hca_off is None else self._hca_off.data_ptr())
        self.params.lookahead = int(lookahead)
        self.n_layers = 1
        if layers:
            self.n_layers = 1 + len(layers)
            self._karr = (P * len(layers))(*[_ptr(k) for k, _ in layers])
            self._sarr = (P * len(layers))(*[_ptr(s) for _, s in layers])
            self.params.n_layers = self.n_layers
            self.params.k_dev_layers = ctypes.cast(self._karr, P)
            self.params.k_scale_layers = ctypes.cast(self._sarr, P) if k_scale is not None else None
        self._keep = (keys, k_scale, cold_host, layers)
        h = P()
        _check(_L.lsa_ctx_create(ctypes.byref(self.params), ctypes.byref(h)), "lsa_ctx_create")
        self.handle = h
        self.B, self.topk, self.n_total, self.kept_capacity = B, topk, n_total, kept_capacity
        self.row_bytes = row_bytes

    def close(self):
        if self.handle:
            _check(_L.lsa_ctx_destroy(self.handle), "lsa_ctx_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def step(self, t, q, w, Q, out, lse=None, stream=None):
        _check(_L.lsa_decode_step(self.handle, t, _ptr(q), _ptr(w), _ptr(Q), _ptr(out), _ptr(lse), _stream(stream)),
               "lsa_decode_step")

    def step_host(self, t, q_host, w_host, Q_host, out_host, lse_host=None, stream=None):
        _check(_L.lsa_decode_step_host(self.handle, t, _ptr(q_host), _ptr(w_host), _ptr(Q_host), _ptr(out_host),
                                       _ptr(lse_host), _stream(stream)), "lsa_decode_step_host")

    def view(self) -> View:
        v = View()
        _check(_L.lsa_ctx_get_view(self.handle, ctypes.byref(v)), "lsa_ctx_get_view")
        return v

    def set_graphs(self, on: bool):
        _check(_L.lsa_ctx_set_graphs(self.handle, int(on)), "lsa_ctx_set_graphs")

    def set_timing(self, on: bool):
        _check(_L.lsa_ctx_set_timing(self.handle, int(on)), "lsa_ctx_set_timing")

    def stage_times(self):
        ms = (ctypes.c_double * N_STAGES)()
        calls = (i64 * N_STAGES)()
        _check(_L.lsa_ctx_stage_times(self.handle, ms, calls), "lsa_ctx_stage_times")
        return {STAGES[i]: (ms[i], calls[i]) for i in range(N_STAGES)}

    def reset_counters(self):
        _check(_L.lsa_ctx_reset_counters(self.handle), "lsa_ctx_reset_counters")

    def launches(self) -> int:
        return int(_L.lsa_ctx_launches(self.handle))

    def flush_cache(self, stream=None):
        """Empty the hot-buffer cache: the next refresh or prediction fetches every kept row."""
        _check(_L.lsa_ctx_flush_cache(self.handle, _stream(stream)), "lsa_ctx_flush_cache")

    def fetched(self) -> int:
        """Rows the last refresh fetched from the cold pool (synchronises the device)."""
        return int(device_view(self.view().fetched, 1, torch.int64).item())


_cudart = None


def device_view(ptr: int, numel: int, dtype: torch.dtype) -> torch.Tensor:
    """Copy `numel` elements at a device address owned by a context into a new tensor (for inspection).

    Synchronises the device first; uses the CUDA runtime torch already loaded.
    """
    global _cudart
    if _cudart is None:
        _cudart = ctypes.CDLL("libcudart.so.12")
        _cudart.cudaMemcpy.restype = ctypes.c_int
        _cudart.cudaMemcpy.argtypes = [P, P, sz, ctypes.c_int]
    out = torch.empty(numel, dtype=dtype, device="cuda")
    if numel:
        torch.cuda.synchronize()
        rc = _cudart.cudaMemcpy(out.data_ptr(), ptr, numel * out.element_size(), 3)  # device to device
        if rc != 0:
            raise RuntimeError(f"cudaMemcpy failed with error {rc}")
    return out
