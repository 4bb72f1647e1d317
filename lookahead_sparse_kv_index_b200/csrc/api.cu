// Public C entry points: argument validation, error reporting, dispatch.
// Every entry point validates on the host and launches nothing on failure.
#include <cstdarg>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "lsa_internal.cuh"

namespace lsa {

static thread_local char g_msg[512] = "";
static thread_local int64_t g_launches = 0;
static thread_local const char *g_last_kernel = "";

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
}
void clear_error() { g_msg[0] = 0; }
void count_launch(const char *name) {
    ++g_launches;
    g_last_kernel = name;
}
int64_t launch_count() { return g_launches; }

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

cudaError_t ensure_smem_raw(const void *func, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    size_t &cur = done[{func, dev}];
    if (cur >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e == cudaSuccess) cur = bytes;
    return e;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

int32_t lsa_version(void) { return 100; }

int64_t lsa_struct_size(int32_t which) {
    return which == 0 ? int64_t(sizeof(lsa_params)) : which == 1 ? int64_t(sizeof(lsa_ctx_view)) : -1;
}

const char *lsa_last_error(void) { return lsa::g_msg; }

const char *lsa_last_kernel(void) { return lsa::g_last_kernel; }

const char *lsa_status_name(lsa_status s) {
    switch (s) {
    case LSA_OK: return "LSA_OK";
    case LSA_ERR_INVALID: return "LSA_ERR_INVALID";
    case LSA_ERR_CUDA: return "LSA_ERR_CUDA";
    case LSA_ERR_CAPACITY: return "LSA_ERR_CAPACITY";
    case LSA_ERR_TIMEOUT: return "LSA_ERR_TIMEOUT";
    case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED";
    }
    return "LSA_ERR_UNKNOWN";
}

lsa_status lsa_index_score(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                           lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                           int64_t n_total, const int32_t *idx, const int64_t *idx_off,
                           int64_t list_capacity, int32_t B, int32_t H, int32_t d, float *z,
                           float *I, int32_t flags, int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(q && w && k && seq_off && z, "lsa_index_score: q, w, k, seq_off and z are required");
    LSA_CHECK_ARG(B >= 1 && H >= 1 && d >= 1, "lsa_index_score: B=%d H=%d d=%d must be positive", B, H, d);
    LSA_CHECK_ARG(n_total >= 0 && n_total < (int64_t(1) << 31),
                  "lsa_index_score: n_total=%lld out of range", (long long)n_total);
    LSA_CHECK_ARG(valid_dtype(q_dtype) && valid_dtype(k_dtype), "lsa_index_score: unknown dtype");
    LSA_CHECK_SUPPORTED(q_dtype == LSA_F32 || q_dtype == LSA_BF16,
                        "lsa_index_score: q must be F32 or BF16");
    LSA_CHECK_ARG((k_dtype == LSA_E4M3) == (k_scale != nullptr),
                  "lsa_index_score: k_scale is required for E4M3 keys and only for them");
    LSA_CHECK_SUPPORTED(H <= 64, "lsa_index_score: H=%d > 64", H);
    LSA_CHECK_SUPPORTED(d == 32 || d == 64 || d == 128, "lsa_index_score: d=%d not in {32,64,128}", d);
    LSA_CHECK_ARG((d * elem_size(k_dtype)) % 16 == 0 && aligned16(k),
                  "lsa_index_score: key rows must be 16-byte aligned");
    LSA_CHECK_ARG((idx == nullptr) == (idx_off == nullptr),
                  "lsa_index_score: idx and idx_off go together");
    LSA_CHECK_ARG(idx == nullptr || (list_capacity >= 0 && list_capacity < (int64_t(1) << 31)),
                  "lsa_index_score: bad list_capacity");
    LSA_CHECK_ARG((flags & ~LSA_SCORE_CUDA_CORE) == 0, "lsa_index_score: unknown flags 0x%x", flags);
    if ((idx ? list_capacity : n_total) == 0) return LSA_OK;
    return launch_index_score(q, q_dtype, w, k, k_dtype, k_scale, seq_off, n_total, idx, idx_off,
                              list_capacity, B, H, d, z, I, flags, err, as_stream(stream));
}

size_t lsa_select_workspace_size(int64_t n_total) {
    int64_t tiles = (n_total + 1023) / 1024;
    int64_t words = (n_total + 31) / 32;
    return align_up(size_t(tiles) * 8, 256) + align_up(size_t(tiles) * 4, 256) +
           align_up(size_t(words) * 4, 256);
}

lsa_status lsa_select(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B,
                      int32_t *kept_idx, int64_t capacity, int64_t *kept_off, uint32_t *mask,
                      void *workspace, size_t ws_bytes, int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(z && seq_off && kept_off && workspace, "lsa_select: z, seq_off, kept_off, workspace required");
    LSA_CHECK_ARG(B >= 1, "lsa_select: B=%d", B);
    LSA_CHECK_ARG(n_total >= 0 && n_total < (int64_t(1) << 31), "lsa_select: n_total out of range");
    LSA_CHECK_ARG(capacity >= 0 && (kept_idx || capacity == 0), "lsa_select: bad capacity / kept_idx");
    LSA_CHECK_ARG(ws_bytes >= lsa_select_workspace_size(n_total) && aligned16(workspace),
                  "lsa_select: workspace of %zu bytes < %zu", ws_bytes, lsa_select_workspace_size(n_total));
    return launch_select(z, seq_off, n_total, B, kept_idx, capacity, kept_off, mask, workspace, err,
                         as_stream(stream));
}

size_t lsa_index_score_select_workspace_size(int64_t n_total, int32_t B) {
    return index_score_select_workspace(n_total, B < 1 ? 1 : B);
}

lsa_status lsa_index_score_select(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                                  lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                                  int64_t n_total, int32_t B, int32_t H, int32_t d, float *z, int32_t *kept_idx,
                                  int64_t capacity, int64_t *kept_off, void *workspace, size_t ws_bytes,
                                  int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(q && w && k && seq_off && z && kept_off && workspace,
                  "lsa_index_score_select: q, w, k, seq_off, z, kept_off and workspace are required");
    LSA_CHECK_ARG(B >= 1 && H >= 1 && d >= 1, "lsa_index_score_select: B=%d H=%d d=%d must be positive", B, H, d);
    LSA_CHECK_ARG(n_total >= 0 && n_total < (int64_t(1) << 31),
                  "lsa_index_score_select: n_total=%lld out of range", (long long)n_total);
    LSA_CHECK_ARG(valid_dtype(q_dtype) && valid_dtype(k_dtype), "lsa_index_score_select: unknown dtype");
    LSA_CHECK_SUPPORTED(q_dtype == LSA_F32 || q_dtype == LSA_BF16, "lsa_index_score_select: q must be F32 or BF16");
    LSA_CHECK_ARG((k_dtype == LSA_E4M3) == (k_scale != nullptr),
                  "lsa_index_score_select: k_scale is required for E4M3 keys and only for them");
    LSA_CHECK_SUPPORTED(H <= 64, "lsa_index_score_select: H=%d > 64", H);
    LSA_CHECK_SUPPORTED(d == 32 || d == 64 || d == 128, "lsa_index_score_select: d=%d not in {32,64,128}", d);
    LSA_CHECK_ARG((d * elem_size(k_dtype)) % 16 == 0 && aligned16(k),
                  "lsa_index_score_select: key rows must be 16-byte aligned");
    LSA_CHECK_ARG(capacity >= 0 && (kept_idx || capacity == 0), "lsa_index_score_select: bad capacity / kept_idx");
    LSA_CHECK_ARG(ws_bytes >= index_score_select_workspace(n_total, B) && aligned16(workspace),
                  "lsa_index_score_select: workspace of %zu bytes < %zu", ws_bytes,
                  index_score_select_workspace(n_total, B));
    cudaStream_t st = as_stream(stream);
    if (n_total == 0)
        return launch_select(z, seq_off, n_total, B, kept_idx, capacity, kept_off, nullptr, workspace, err, st);
    return launch_index_score_select(q, q_dtype, w, k, k_dtype, k_scale, seq_off, n_total, B, H, d, z, kept_idx,
                                     capacity, kept_off, workspace, err, st);
}

lsa_status lsa_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                    const int32_t *kept_idx, const int64_t *kept_off, int64_t kept_capacity,
                    int32_t B, int32_t k, int32_t *topk_idx, int32_t *topk_pos,
                    int32_t *topk_cnt, void *stream) {
    clear_error();
    LSA_CHECK_ARG(z && kept_idx && kept_off && topk_idx && topk_cnt,
                  "lsa_topk: z, kept_idx, kept_off, topk_idx, topk_cnt required");
    LSA_CHECK_ARG(!z_by_entry || seq_off, "lsa_topk: z_by_entry needs seq_off");
    LSA_CHECK_ARG(B >= 1, "lsa_topk: B=%d", B);
    LSA_CHECK_SUPPORTED(k >= 1 && k <= 4096, "lsa_topk: k=%d not in [1, 4096]", k);
    LSA_CHECK_ARG(kept_capacity >= 0, "lsa_topk: kept_capacity < 0");
    return launch_topk(z, z_by_entry, seq_off, kept_idx, kept_off, B, k, kept_capacity, nullptr, topk_idx,
                       topk_pos, topk_cnt, as_stream(stream));
}

lsa_status lsa_gather(const void *cold_host, int64_t row_bytes, const int64_t *seq_off,
                      int64_t n_total, const int32_t *kept_idx, const int64_t *kept_off, int32_t B,
                      void *hot, int64_t hot_capacity, int32_t *slot_of, int32_t *err,
                      void *stream) {
    clear_error();
    LSA_CHECK_ARG(cold_host && seq_off && kept_idx && kept_off && hot,
                  "lsa_gather: cold_host, seq_off, kept_idx, kept_off, hot required");
    LSA_CHECK_ARG(row_bytes > 0 && row_bytes % 16 == 0, "lsa_gather: row_bytes=%lld must be a positive multiple of 16",
                  (long long)row_bytes);
    LSA_CHECK_ARG(B >= 1 && n_total >= 0 && hot_capacity >= 0, "lsa_gather: bad sizes");
    LSA_CHECK_ARG(aligned16(cold_host) && aligned16(hot), "lsa_gather: cold and hot must be 16-byte aligned");
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, cold_host);
    if (e != cudaSuccess) cudaGetLastError();
    LSA_CHECK_ARG(e == cudaSuccess && attr.type == cudaMemoryTypeHost && attr.devicePointer,
                  "lsa_gather: cold_host is not page-locked host memory mapped for the device");
    const void *cold_dev = attr.devicePointer;
    return launch_gather(cold_dev, row_bytes, seq_off, n_total, kept_idx, kept_off, B, hot,
                         hot_capacity, slot_of, err, as_stream(stream));
}

size_t lsa_sparse_attn_workspace_size(int32_t B, int32_t Hq, int32_t D, int32_t k) {
    if (B < 1 || Hq < 1 || D < 1 || k < 1) return 0;
    return sparse_attn_workspace(B, Hq, D, k);
}

lsa_status lsa_sparse_attn(const void *Q, lsa_dtype dtype, const void *kv, int64_t kv_row_stride,
                           int64_t k_off, int64_t v_off, const int32_t *rows, int32_t B,
                           int32_t Hq, int32_t D, int32_t k, float scale, void *out, float *lse,
                           void *workspace, size_t ws_bytes, int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(Q && kv && rows && out && workspace, "lsa_sparse_attn: Q, kv, rows, out, workspace required");
    LSA_CHECK_SUPPORTED(dtype == LSA_F32 || dtype == LSA_BF16, "lsa_sparse_attn: dtype must be F32 or BF16");
    LSA_CHECK_ARG(B >= 1, "lsa_sparse_attn: B=%d", B);
    LSA_CHECK_SUPPORTED(D % 32 == 0 && D >= 32 && D <= 512, "lsa_sparse_attn: D=%d", D);
    LSA_CHECK_SUPPORTED(Hq >= 1 && Hq <= 256, "lsa_sparse_attn: Hq=%d", Hq);
    LSA_CHECK_SUPPORTED(k >= 1 && k <= 65536, "lsa_sparse_attn: k=%d not in [1, 65536]", k);
    LSA_CHECK_ARG(kv_row_stride >= D && k_off >= 0 && v_off >= 0 && k_off + D <= kv_row_stride &&
                      v_off + D <= kv_row_stride,
                  "lsa_sparse_attn: K/V must lie inside a row");
    LSA_CHECK_ARG((kv_row_stride * elem_size(dtype)) % 16 == 0 && (k_off * elem_size(dtype)) % 16 == 0 &&
                      (v_off * elem_size(dtype)) % 16 == 0 && aligned16(kv) && aligned16(Q) && aligned16(out),
                  "lsa_sparse_attn: rows, K and V must be 16-byte aligned");
    LSA_CHECK_ARG(scale > 0.0f && scale < 1e30f, "lsa_sparse_attn: scale must be positive and finite");
    LSA_CHECK_ARG(ws_bytes >= sparse_attn_workspace(B, Hq, D, k) && aligned16(workspace),
                  "lsa_sparse_attn: workspace of %zu bytes < %zu", ws_bytes, sparse_attn_workspace(B, Hq, D, k));
    return launch_sparse_attn(Q, dtype, kv, kv_row_stride, k_off, v_off, rows, B, Hq, D, k, scale, out,
                              lse, workspace, err, as_stream(stream));
}

}  // extern "C"
