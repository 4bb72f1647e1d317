// Internal helpers shared by the CUDA translation units of liblsa.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>
#include <utility>

#include "lsa.h"

namespace lsa {

// ---------------------------------------------------------------- host side

void set_error(const char *fmt, ...);
void clear_error();

// Validation helper: returns LSA_ERR_INVALID with a message when cond fails.
#define LSA_CHECK_ARG(cond, ...)              \
    do {                                      \
        if (!(cond)) {                        \
            ::lsa::set_error(__VA_ARGS__);    \
            return LSA_ERR_INVALID;           \
        }                                     \
    } while (0)

#define LSA_CHECK_SUPPORTED(cond, ...)        \
    do {                                      \
        if (!(cond)) {                        \
            ::lsa::set_error(__VA_ARGS__);    \
            return LSA_ERR_UNSUPPORTED;       \
        }                                     \
    } while (0)

// (a failed call's error is also taken off the runtime's last-error slot, so that it is not reported
// again by the next launch check)
#define LSA_CUDA(call)                                                              \
    do {                                                                            \
        cudaError_t e_ = (call);                                                    \
        if (e_ != cudaSuccess) {                                                    \
            cudaGetLastError();                                                     \
            ::lsa::set_error("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                             __FILE__, __LINE__);                                   \
            return LSA_ERR_CUDA;                                                    \
        }                                                                           \
    } while (0)

// After a kernel launch: report launch-configuration errors.
#define LSA_LAUNCHED(name)                                                             \
    do {                                                                               \
        cudaError_t e_ = cudaGetLastError();                                           \
        if (e_ != cudaSuccess) {                                                       \
            ::lsa::set_error("launch of %s failed: %s", name, cudaGetErrorString(e_)); \
            return LSA_ERR_CUDA;                                                       \
        }                                                                              \
        ::lsa::count_launch(name);                                                     \
    } while (0)

// Per-thread kernel launch counter (read by the decode context) and the name of
// the last kernel launched (lsa_last_kernel).  `name` must be a static string.
void count_launch(const char *name);
int64_t launch_count();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t elem_size(lsa_dtype t) { return t == LSA_F32 ? 4 : t == LSA_BF16 ? 2 : 1; }
inline bool valid_dtype(int t) { return t == LSA_F32 || t == LSA_BF16 || t == LSA_E4M3; }
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Number of SMs of the current device (cached per device).
int sm_count();

// Raises a kernel's dynamic shared-memory limit on the current device to at
// least `bytes`, once: later calls are a table lookup (no CUDA call), so
// launches inside a stream capture make no attribute calls.
cudaError_t ensure_smem_raw(const void *func, size_t bytes);
template <typename F>
inline cudaError_t ensure_smem(F *func, size_t bytes) {
    return ensure_smem_raw(reinterpret_cast<const void *>(func), bytes);
}

// Internal launchers (each validates nothing; the public entry points do).
lsa_status launch_index_score(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                              lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                              int64_t n_total, const int32_t *idx, const int64_t *idx_off,
                              int64_t list_capacity, int32_t B, int32_t H, int32_t d, float *z,
                              float *I, int32_t flags, int32_t *err, cudaStream_t st);
bool index_score_tc_supported(lsa_dtype q_dtype, lsa_dtype k_dtype, int64_t n_total, int32_t B, int32_t H,
                              int32_t d);
lsa_status launch_index_score_tc(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                 const float *k_scale, const int64_t *seq_off, int64_t n_total,
                                 const int32_t *idx, const int64_t *idx_off, int64_t list_cap, int32_t B,
                                 int32_t H, int32_t d, float *z, float *I, int32_t *err, cudaStream_t st);
// Full tensor-core scan over a device-produced row axis: rows axis_off[b] .. axis_off[b+1] (clamped to
// axis_cap) of the key array k [n_rows, d] belong to sequence b; z is written per row.  Used on a compacted
// copy of the kept keys (rows in kept-list order), so z lands at the kept position.
// The full tensor-core scan that also writes the z >= 0 ballots of each scan tile (TR / 32 words) and the
// kept count of each quarter of the tile, for the fused selection; TR = index_score_tc_tile_rows.
int index_score_tc_tile_rows(lsa_dtype k_dtype);
lsa_status launch_index_score_tc_select(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                        const float *k_scale, const int64_t *seq_off, int64_t n_total, int32_t B,
                                        int32_t H, int32_t d, float *z, uint32_t *sel_bits, int32_t *sel_cnt,
                                        int32_t *err, cudaStream_t st);
// Full scan + selection: fused on the tensor-core path, else the CUDA-core scan and lsa_select's kernels.
// workspace: index_score_select_workspace(n_total, B) bytes (covers both).
size_t select_tiles_workspace(int64_t n_total, int32_t B);
size_t index_score_select_workspace(int64_t n_total, int32_t B);
lsa_status launch_index_score_select(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                                     lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                                     int64_t n_total, int32_t B, int32_t H, int32_t d, float *z, int32_t *kept_idx,
                                     int64_t capacity, int64_t *kept_off, void *workspace, int32_t *err,
                                     cudaStream_t st);
lsa_status launch_index_score_tc_axis(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                      const float *k_scale, int64_t scale_len, const int64_t *axis_off,
                                      int64_t axis_cap, int64_t n_rows, int32_t B, int32_t H, int32_t d, float *z,
                                      int32_t *err, cudaStream_t st);
// Copies the key rows (and e4m3 row scales) of the kept entries into kept-list order:
// kc[p] = k[seq_off[b] + kept_idx[p]] for p < min(kept_off[B], cap).
lsa_status launch_gather_keys(const void *k, int64_t row_bytes, const float *k_scale, const int64_t *seq_off,
                              const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int64_t cap, void *kc,
                              float *sc, cudaStream_t st);
lsa_status launch_select(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B,
                         int32_t *kept_idx, int64_t capacity, int64_t *kept_off, uint32_t *mask,
                         void *workspace, int32_t *err, cudaStream_t st);
// pos_map (nullable): topk_pos receives pos_map[p] instead of the kept position p.
lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, const int32_t *pos_map, int32_t *topk_idx, int32_t *topk_pos,
                       int32_t *topk_cnt, cudaStream_t st);
size_t fetch_workspace(int64_t cap);
lsa_status launch_fetch(const void *cold_dev, int64_t row_bytes, const int64_t *seq_off, const int32_t *kept_idx,
                        const int64_t *kept_off, int32_t B, void *hot, int64_t cap, int32_t *slot_of,
                        int32_t *owner, int32_t *kept_slot, int64_t *fetched, void *workspace, int32_t *err,
                        cudaEvent_t assigned, cudaStream_t st, const int32_t *prot_slot = nullptr,
                        const int64_t *prot_off = nullptr, int row_ctas = 0);
lsa_status launch_gather(const void *cold_dev, int64_t row_bytes, const int64_t *seq_off,
                         int64_t n_total, const int32_t *kept_idx, const int64_t *kept_off,
                         int32_t B, void *hot, int64_t hot_capacity, int32_t *slot_of,
                         int32_t *err, cudaStream_t st);
lsa_status launch_sparse_attn(const void *Q, lsa_dtype dtype, const void *kv, int64_t stride,
                              int64_t k_off, int64_t v_off, const int32_t *rows, int32_t B,
                              int32_t Hq, int32_t D, int32_t k, float scale, void *out, float *lse,
                              void *workspace, int32_t *err, cudaStream_t st);
bool sparse_attn_tc_supported(lsa_dtype dtype, int64_t k_off, int64_t v_off, int32_t Hq, int32_t D);
int sparse_attn_tc_chunk();
lsa_status launch_sparse_attn_tc(const void *Q, const void *kv, int64_t stride, int64_t k_off,
                                 const int32_t *rows, int32_t B, int32_t k, float scale, void *part_o,
                                 float *part_ml, int32_t *err, cudaStream_t st);
size_t sparse_attn_workspace(int32_t B, int32_t Hq, int32_t D, int32_t k);
constexpr int kMaxUnionLayers = 8;
lsa_status launch_union(const float *const *z_layers, int32_t n_layers, int64_t n_total, float *z_union,
                        cudaStream_t st);
lsa_status launch_merge_rows(const int32_t *topk_idx, const int32_t *topk_pos, const int32_t *topk_cnt,
                             const int64_t *seq_off, int32_t B, int32_t k, int32_t window, int32_t win_base,
                             const int64_t *hca_off, int32_t hca_base, int32_t *rows, int32_t row_cap,
                             int32_t *count, int32_t *err, cudaStream_t st);

// Launch with programmatic dependent launch: the kernel may be scheduled as
// soon as the previous kernel on the stream signals griddepcontrol.
// launch_dependents; it must execute pdl_wait() before touching anything the
// previous kernel writes (pdl_wait returns once that kernel has completed and
// its memory is visible).  Captured into CUDA graphs as programmatic edges.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ------------------------------------------------------------- device side

// Programmatic dependent launch controls (no-ops for a kernel launched without it).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// First error wins.
__device__ __forceinline__ void raise_err(int32_t *err, int32_t code) {
    if (err) atomicCAS(err, 0, code);
}

// Index of the sequence that owns position e of a CSR axis: the largest b
// with off[b] <= e (off is non-decreasing, off[0] = 0, e < off[B]).
__device__ __forceinline__ int seq_of(const int64_t *off, int B, int64_t e) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= e) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace lsa
