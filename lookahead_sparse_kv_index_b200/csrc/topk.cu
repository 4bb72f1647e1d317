// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One CTA of 1024 threads per sequence.  Scores map to an order-preserving
// 32-bit key (larger z -> larger key, -0.0 folded onto +0.0).  A most-
// significant-digit radix select (passes of 11 bits, below the bits every key
// shares) finds the digits of the k-th largest key and how many entries sharing
// them must be taken; an ordered pass then takes every key above and the
// lowest-index entries at the threshold, and compacts them in kept-list order,
// which is ascending entry order.  A few tens of thousands of kept entries per
// sequence fit in shared memory, so every pass works there and the only
// synchronisation is the CTA's own barrier (a cluster of CTAs spent most of its
// time in cluster-wide barriers at this size).
#include "lsa_internal.cuh"

namespace lsa {
namespace {

__device__ __forceinline__ uint32_t order_key(float z) {
    uint32_t b = __float_as_uint(z);
    if (b == 0x80000000u) b = 0u;                      // -0.0 ranks as +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kStageKeys = 40960;   // keys staged in shared memory (160 KB)
constexpr int kMaxK = 4096;          // the largest k (the entry points check it); positions of the chosen in smem
constexpr int kDigit = 11;
constexpr int kBins = 1 << kDigit;   // 2048: two bins per thread

// Exclusive block-wide prefix sum of v (kThreads threads); *total receives the sum.
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        s_warp[lane] = s;
    }
    __syncthreads();
    const int res = (warp ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kWarps - 1];
    return res;   // s_warp is rewritten only after the caller's next barrier
}

// Exclusive block-wide prefix sum of a 64-bit value (two counters packed as hi:lo 32-bit halves).
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t *s_warp64) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp64[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint64_t t = s_warp64[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        s_warp64[lane] = t;
    }
    __syncthreads();
    return (warp ? s_warp64[warp - 1] : 0) + x - v;
}

__global__ void __launch_bounds__(kThreads, 1)
topk_select(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
            const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
            const int32_t *__restrict__ pos_map, int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos,
            int32_t *__restrict__ topk_cnt) {
    extern __shared__ uint32_t s_keys[];   // [kStageKeys] keys, then [kMaxK] positions of the chosen
    int *s_pos = reinterpret_cast<int *>(s_keys + kStageKeys);
    __shared__ int s_hist[kBins];
    __shared__ int s_warp[kWarps];
    __shared__ uint64_t s_warp64[kWarps];
    __shared__ uint32_t s_red[2][kWarps];
    __shared__ uint32_t s_want;
    __shared__ int s_kr, s_done;

    pdl_launch_dependents();   // attention may stage its queries meanwhile
    pdl_wait();                // scores come from the preceding scan
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t p0 = kept_off[b];
    int64_t n64 = kept_off[b + 1] - p0;
    if (p0 >= kept_cap) n64 = 0;
    else if (p0 + n64 > kept_cap) n64 = kept_cap - p0;
    if (n64 < 0) n64 = 0;
    const int n = int(n64);
    int32_t *out_idx = topk_idx + int64_t(b) * k;
    int32_t *out_pos = topk_pos ? topk_pos + int64_t(b) * k : nullptr;

    if (n <= k) {   // everything kept is chosen
        for (int i = threadIdx.x; i < k; i += kThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? (pos_map ? pos_map[p0 + i] : int32_t(p0 + i)) : -1;
        }
        if (threadIdx.x == 0) topk_cnt[b] = n;
        return;
    }
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    const bool staged = n <= kStageKeys;
    auto load_key = [&](int i) -> uint32_t {   // i: position in the sequence's kept list
        const int64_t p = p0 + i;
        return order_key(z_by_entry ? z[sbase + kept_idx[p]] : z[p]);
    };
    // each thread owns the contiguous run [lo, hi) of positions (the ordered take needs runs)
    const int per = (n + kThreads - 1) / kThreads;
    const int lo = min(n, int(threadIdx.x) * per), hi = min(n, lo + per);

    // stage the keys (coalesced: consecutive threads, consecutive positions), min / max on the way
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i0 = int(threadIdx.x); i0 < n; i0 += 8 * kThreads) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kThreads;
            v[u] = i < n ? load_key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kThreads;
            if (i < n) {
                if (staged) s_keys[i] = v[u];
                kmin = min(kmin, v[u]);
                kmax = max(kmax, v[u]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) { s_red[0][warp] = kmin; s_red[1][warp] = kmax; }
    __syncthreads();   // also publishes the staged keys
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
#pragma unroll 4
    for (int w = 0; w < kWarps; ++w) { gmin = min(gmin, s_red[0][w]); gmax = max(gmax, s_red[1][w]); }
    auto key = [&](int i) -> uint32_t { return staged ? s_keys[i] : load_key(i); };

    const uint32_t diff = gmin ^ gmax;
    int top = diff ? 31 - __clz(diff) : -1;   // bits above `top` are shared by every key
    uint32_t hmask = top >= 31 ? 0u : (top >= 0 ? ~((2u << top) - 1u) : 0xFFFFFFFFu);
    uint32_t want = gmin & hmask;
    int kr = k;
    s_hist[threadIdx.x] = 0;   // each pass's reader zeroes its bins for the next pass
    s_hist[threadIdx.x + kThreads] = 0;
    __syncthreads();
    while (top >= 0) {
        const int width = top + 1 < kDigit ? top + 1 : kDigit;
        const int shift = top + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key(i);
            if ((u & hmask) == want) atomicAdd(&s_hist[(u >> shift) & dmask], 1);
        }
        __syncthreads();
        {   // thread t owns bins 2047 - 2t and 2046 - 2t (descending key order); suffix counts by a block scan
            const int bh = kBins - 1 - 2 * int(threadIdx.x);
            const int h0 = s_hist[bh], h1 = s_hist[bh - 1];
            s_hist[bh] = 0;   // only this thread reads these two bins
            s_hist[bh - 1] = 0;
            int tot;
            int above = block_excl_scan(h0 + h1, s_warp, &tot);   // entries in bins above bh
            if (above < kr && above + h0 >= kr) {
                s_want = want | (uint32_t(bh) << shift);
                s_kr = kr - above;
                s_done = (above + h0 == kr);
            } else if (above + h0 < kr && above + h0 + h1 >= kr) {
                s_want = want | (uint32_t(bh - 1) << shift);
                s_kr = kr - above - h0;
                s_done = (above + h0 + h1 == kr);
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= dmask << shift;
        top = shift - 1;
        if (s_done) break;   // uniform: read after the barrier, rewritten only after the next barrier
    }
    // ordered take: keys whose resolved bits exceed `want`, then the first kr equal to it (in kept-list
    // order).  One scan of the packed counts (equal : above) gives both this thread's rank among the
    // equal keys and the number of keys above before it.
    int n_eq = 0, n_above = 0;
    for (int i = lo; i < hi; ++i) {
        const uint32_t u = key(i) & hmask;
        n_eq += u == want;
        n_above += u > want;
    }
    const uint64_t pre = block_excl_scan64((uint64_t(n_eq) << 32) | uint32_t(n_above), s_warp64);
    const int eq_rank = int(pre >> 32);
    int out = int(uint32_t(pre)) + min(eq_rank, kr);
    // the take records the position of each output slot; the entry indices are then fetched with
    // independent loads, two slots per thread (a dependent load per taken key serialised the tail)
    int r = eq_rank;
    for (int i = lo; i < hi; ++i) {
        const uint32_t u = key(i) & hmask;
        bool t = u > want;
        if (u == want) { t = r < kr; ++r; }
        if (t) {
            if (out < k) s_pos[out] = i;
            ++out;
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < k; j += kThreads) {
        const int64_t p = p0 + s_pos[j];
        out_idx[j] = kept_idx[p];
        if (out_pos) out_pos[j] = pos_map ? pos_map[p] : int32_t(p);
    }
    if (threadIdx.x == 0) topk_cnt[b] = k;
}

}  // namespace

lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, const int32_t *pos_map, int32_t *topk_idx, int32_t *topk_pos,
                       int32_t *topk_cnt, cudaStream_t st) {
    const size_t smem = size_t(kStageKeys) * 4 + size_t(kMaxK) * 4;
    LSA_CUDA(ensure_smem(topk_select, smem));
    LSA_CUDA(launch_pdl(topk_select, dim3(B), dim3(kThreads), smem, st, z, z_by_entry, seq_off, kept_idx, kept_off,
                        kept_cap, k, pos_map, topk_idx, topk_pos, topk_cnt));
    LSA_LAUNCHED("topk_select");
    return LSA_OK;
}

}  // namespace lsa
