// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One 1024-thread block per sequence.  Scores map to an order-preserving
// 32-bit key (larger z -> larger key, -0.0 folded onto +0.0).  A most-
// significant-digit radix select (4 passes of 8 bits, shared-memory
// histograms) finds the key T of the k-th largest entry and how many entries
// equal to T must be taken; a final ordered pass takes every key > T and the
// lowest-index entries with key == T, and compacts them in kept-list order,
// which is ascending entry order.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float z) {
    uint32_t b = __float_as_uint(z);
    if (b == 0x80000000u) b = 0u;                      // -0.0 ranks as +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide prefix sum of one int per thread (1024 threads);
// returns the exclusive prefix, writes the block total to *total.
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        s_warp[lane] = s;
    }
    __syncthreads();
    const int res = (warp ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[31];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_radix(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
           const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off,
           int64_t kept_cap, int k, int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos,
           int32_t *__restrict__ topk_cnt) {
    __shared__ int hist[256];
    __shared__ int s_warp[32];
    __shared__ uint32_t s_want;
    __shared__ int s_kr;

    const int b = blockIdx.x;
    const int64_t p0 = kept_off[b];
    int64_t n = kept_off[b + 1] - p0;
    if (p0 >= kept_cap) n = 0;
    else if (p0 + n > kept_cap) n = kept_cap - p0;
    if (n < 0) n = 0;
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    int32_t *out_idx = topk_idx + int64_t(b) * k;
    int32_t *out_pos = topk_pos ? topk_pos + int64_t(b) * k : nullptr;

    auto key_at = [&](int64_t i) -> uint32_t {
        const int64_t p = p0 + i;
        return order_key(z_by_entry ? z[sbase + kept_idx[p]] : z[p]);
    };

    if (n <= k) {
        for (int64_t i = threadIdx.x; i < k; i += kTopkThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? int32_t(p0 + i) : -1;
        }
        if (threadIdx.x == 0) topk_cnt[b] = int32_t(n);
        return;
    }

    uint32_t want = 0, hmask = 0;
    int kr = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (threadIdx.x < 256) hist[threadIdx.x] = 0;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < n; i += kTopkThreads) {
            const uint32_t u = key_at(i);
            if ((u & hmask) == want) atomicAdd(&hist[(u >> shift) & 0xFFu], 1);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int local = 0;
#pragma unroll
            for (int x = 0; x < 8; ++x) local += hist[8 * lane + x];
            int suf = local;   // inclusive suffix sum over lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            int above = suf - local;  // entries in higher lanes' bins
#pragma unroll
            for (int x = 7; x >= 0; --x) {
                const int h = hist[8 * lane + x];
                if (above < kr && above + h >= kr) {
                    s_want = want | (uint32_t(8 * lane + x) << shift);
                    s_kr = kr - above;
                }
                above += h;
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= 0xFFu << shift;
        __syncthreads();
    }
    // want is the exact key of the k-th largest; take kr of the entries equal to it.
    int tie_carry = 0, out_carry = 0;
    for (int64_t c0 = 0; c0 < n; c0 += kTopkThreads) {
        const int64_t i = c0 + threadIdx.x;
        uint32_t u = 0;
        const bool valid = i < n;
        if (valid) u = key_at(i);
        const bool gt = valid && u > want;
        const bool eq = valid && u == want;
        int tot;
        const int eq_rank = block_excl_scan(eq ? 1 : 0, s_warp, &tot) + tie_carry;
        tie_carry += tot;
        const bool take = gt || (eq && eq_rank < kr);
        const int r = block_excl_scan(take ? 1 : 0, s_warp, &tot) + out_carry;
        out_carry += tot;
        if (take && r < k) {
            out_idx[r] = kept_idx[p0 + i];
            if (out_pos) out_pos[r] = int32_t(p0 + i);
        }
    }
    if (threadIdx.x == 0) topk_cnt[b] = k;
}

}  // namespace

lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, int32_t *topk_idx, int32_t *topk_pos, int32_t *topk_cnt,
                       cudaStream_t st) {
    topk_radix<<<B, kTopkThreads, 0, st>>>(z, z_by_entry, seq_off, kept_idx, kept_off, kept_cap, k,
                                           topk_idx, topk_pos, topk_cnt);
    LSA_LAUNCHED("topk_radix");
    return LSA_OK;
}

}  // namespace lsa
