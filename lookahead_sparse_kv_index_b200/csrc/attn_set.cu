// Merged attention set ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse
// Attention", gist.science technical summary, section 2.1 "Architectural
// Design": every Heavily Compressed Attention chunk, 128:1, stays resident for
// global awareness; section 1 "Problem Statement": the most recent 8K tokens
// alone answer most long requests).  Per sequence the core attention runs over
// the set union of its top-k entries, its last `window` entries and all of its
// HCA rows, each row once: a top-k entry inside the window is attended through
// the window's copy.
//
// One CTA per sequence writes its row list: the top-k slots of entries below
// the window (stable, so ascending entry order), then the HCA rows, then the
// window rows, then -1 padding up to row_cap.  The lists index one KV arena
// (hot buffer, window rows, HCA rows), so the attention kernels read them like
// any other row list.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 1024;

// Exclusive prefix of `flag` over the CTA (warp ballots, then the warp totals).
__device__ __forceinline__ int block_rank(bool flag, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        const int v = lane < (kThreads >> 5) ? s_warp[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        s_warp[lane] = incl - v;
        if (lane == 31) *total = incl;
    }
    __syncthreads();
    const int r = s_warp[warp] + in_warp;
    __syncthreads();   // s_warp is reused by the next call
    return r;
}

__global__ void __launch_bounds__(kThreads) merge_rows(const int32_t *__restrict__ topk_idx,
                                                       const int32_t *__restrict__ topk_pos,
                                                       const int32_t *__restrict__ topk_cnt,
                                                       const int64_t *__restrict__ seq_off, int k, int window,
                                                       int win_base, const int64_t *__restrict__ hca_off,
                                                       int hca_base, int32_t *__restrict__ rows, int row_cap,
                                                       int32_t *__restrict__ count, int32_t *err) {
    __shared__ int s_warp[32];
    __shared__ int s_total;
    pdl_launch_dependents();
    pdl_wait();   // the top-k comes from the preceding kernel
    const int b = blockIdx.x;
    const int64_t n_b = seq_off[b + 1] - seq_off[b];
    const int w_b = int(n_b < window ? n_b : window);
    const int64_t lo = n_b - w_b;   // the window holds entries lo .. n_b-1
    const int cnt = min(max(topk_cnt[b], 0), k);
    int32_t *out = rows + int64_t(b) * row_cap;

    int n_top = 0;
    for (int p0 = 0; p0 < cnt; p0 += kThreads) {
        const int p = p0 + threadIdx.x;
        int32_t e = -1;
        if (p < cnt) e = topk_idx[int64_t(b) * k + p];
        const bool keep = e >= 0 && e < lo;
        const int r = block_rank(keep, s_warp, &s_total);
        if (keep && n_top + r < row_cap) out[n_top + r] = topk_pos[int64_t(b) * k + p];
        n_top += s_total;
        __syncthreads();
    }
    const int64_t h0 = hca_off ? hca_off[b] : 0;
    const int n_hca = hca_off ? int(hca_off[b + 1] - h0) : 0;
    const int64_t total = int64_t(n_top) + n_hca + w_b;
    if (total > row_cap && threadIdx.x == 0) raise_err(err, LSA_ERR_CAPACITY);
    for (int j = threadIdx.x; j < row_cap; j += kThreads) {
        if (j < n_top) continue;   // written above
        int32_t v = -1;
        if (j < n_top + n_hca)
            v = hca_base + int32_t(h0 + (j - n_top));
        else if (j < total)
            v = win_base + b * window + (j - n_top - n_hca);
        out[j] = v;
    }
    if (count && threadIdx.x == 0) count[b] = int32_t(total < row_cap ? total : row_cap);
}

}  // namespace

lsa_status launch_merge_rows(const int32_t *topk_idx, const int32_t *topk_pos, const int32_t *topk_cnt,
                             const int64_t *seq_off, int32_t B, int32_t k, int32_t window, int32_t win_base,
                             const int64_t *hca_off, int32_t hca_base, int32_t *rows, int32_t row_cap,
                             int32_t *count, int32_t *err, cudaStream_t st) {
    LSA_CUDA(launch_pdl(merge_rows, dim3(B), dim3(kThreads), 0, st, topk_idx, topk_pos, topk_cnt, seq_off, int(k),
                        int(window), int(win_base), hca_off, int(hca_base), rows, int(row_cap), count, err));
    LSA_LAUNCHED("merge_rows");
    return LSA_OK;
}

}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_attn_set_merge(const int32_t *topk_idx, const int32_t *topk_pos, const int32_t *topk_cnt,
                                         const int64_t *seq_off, int32_t B, int32_t k, int32_t window,
                                         int32_t win_base, const int64_t *hca_off, int32_t hca_base, int32_t *rows,
                                         int32_t row_cap, int32_t *count, int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(topk_idx && topk_pos && topk_cnt && seq_off && rows,
                  "lsa_attn_set_merge: topk_idx, topk_pos, topk_cnt, seq_off and rows are required");
    LSA_CHECK_ARG(B >= 1 && B <= 65535, "lsa_attn_set_merge: B=%d out of range", B);
    LSA_CHECK_ARG(k >= 1, "lsa_attn_set_merge: k=%d < 1", k);
    LSA_CHECK_ARG(window >= 0 && win_base >= 0 && hca_base >= 0,
                  "lsa_attn_set_merge: window, win_base and hca_base must be >= 0");
    LSA_CHECK_ARG(row_cap >= 1, "lsa_attn_set_merge: row_cap=%d < 1", row_cap);
    LSA_CHECK_ARG(int64_t(win_base) + int64_t(B) * window < (int64_t(1) << 31),
                  "lsa_attn_set_merge: window rows overflow int32 row indices");
    return launch_merge_rows(topk_idx, topk_pos, topk_cnt, seq_off, B, k, window, win_base, hca_off, hca_base, rows,
                             row_cap, count, err, as_stream(stream));
}
