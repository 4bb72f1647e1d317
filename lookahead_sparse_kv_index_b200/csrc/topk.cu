// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One 512-thread block per sequence.  Scores map to an order-preserving 32-bit
// key (larger z -> larger key, -0.0 folded onto +0.0).  A most-significant-
// digit radix select (up to 4 passes of 8 bits) finds the digits of the k-th
// largest key and how many entries sharing them must be taken; an ordered pass
// then takes every key above and the lowest-index entries at the threshold,
// and compacts them in kept-list order, which is ascending entry order.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

__device__ __forceinline__ uint32_t order_key(float z) {
    uint32_t b = __float_as_uint(z);
    if (b == 0x80000000u) b = 0u;                      // -0.0 ranks as +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Kept sets of up to kRegThreads * kKpt entries live in registers: thread t owns the contiguous positions [t*kKpt, (t+1)*kKpt) and loads their
// scores and entry indices in one unrolled batch (independent loads in flight
// instead of a chain of dependent ones); the radix passes count from
// registers into per-warp histograms; the ordered take needs two block scans
// and writes each thread's run in order.  Lanes of a warp that hit the same
// histogram bin are merged with __match_any_sync before one shared atomic
// (kept scores cluster in a few leading-digit bins, so unmerged atomics would
// serialise), and the select stops as soon as the threshold bin holds exactly
// the entries still needed.  Larger kept sets run the same select reading the
// keys from global memory (topk_large).
constexpr int kRegThreads = 512;
constexpr int kKpt = 48;
constexpr int kRegWarps = kRegThreads / 32;

__device__ __forceinline__ int block_excl_scan512(int v, int *s_warp, int *total) {
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
        int s = lane < kRegWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kRegWarps) s_warp[lane] = s;
    }
    __syncthreads();
    const int res = (warp ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kRegWarps - 1];
    __syncthreads();
    return res;
}

// Kept sets too large for the registers: the same radix select, reading the
// keys from global memory in every pass.
__device__ void topk_large(const float *__restrict__ z, int z_by_entry, int64_t sbase,
                           const int32_t *__restrict__ kept_idx, int64_t p0, int n, int k,
                           int32_t *__restrict__ out_idx, int32_t *__restrict__ out_pos,
                           int (*s_hist)[256], int *s_warp, uint32_t *s_want, int *s_kr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto key_at = [&](int i) -> uint32_t {
        return order_key(z_by_entry ? z[sbase + kept_idx[p0 + i]] : z[p0 + i]);
    };
    uint32_t want = 0, hmask = 0;
    int kr = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) s_hist[warp][i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += kRegThreads) {
            const int i = i0 + int(threadIdx.x);
            const uint32_t u = i < n ? key_at(i) : 0u;
            const bool in = i < n && (u & hmask) == want;
            const int digit = in ? int((u >> shift) & 0xFFu) : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (in && (__ffs(peers) - 1) == lane) atomicAdd(&s_hist[warp][digit], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            int sum = 0;
            for (int w = 0; w < kRegWarps; ++w) sum += s_hist[w][threadIdx.x];
            s_hist[0][threadIdx.x] = sum;
        }
        __syncthreads();
        if (warp == 0) {
            int local = 0;
            for (int x = 0; x < 8; ++x) local += s_hist[0][8 * lane + x];
            int suf = local;
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            int above = suf - local;
            for (int x = 7; x >= 0; --x) {
                const int h = s_hist[0][8 * lane + x];
                if (above < kr && above + h >= kr) {
                    *s_want = want | (uint32_t(8 * lane + x) << shift);
                    *s_kr = kr - above;
                }
                above += h;
            }
        }
        __syncthreads();
        want = *s_want;
        kr = *s_kr;
        hmask |= 0xFFu << shift;
        __syncthreads();
    }
    const int per = (n + kRegThreads - 1) / kRegThreads;
    const int lo = min(n, int(threadIdx.x) * per), hi = min(n, lo + per);
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += key_at(i) == want;
    int tot;
    const int eq_rank = block_excl_scan512(n_eq, s_warp, &tot);
    int n_take = 0;
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key_at(i);
            if (u > want) ++n_take;
            else if (u == want) { n_take += r < kr; ++r; }
        }
    }
    int out = block_excl_scan512(n_take, s_warp, &tot);
    int r = eq_rank;
    for (int i = lo; i < hi; ++i) {
        const uint32_t u = key_at(i);
        bool take = u > want;
        if (u == want) { take = r < kr; ++r; }
        if (take && out < k) {
            out_idx[out] = kept_idx[p0 + i];
            if (out_pos) out_pos[out] = int32_t(p0 + i);
            ++out;
        }
    }
}

__global__ void __launch_bounds__(kRegThreads)
topk_reg(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
         const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
         int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos, int32_t *__restrict__ topk_cnt) {
    __shared__ int s_hist[kRegWarps][256];
    __shared__ int s_warp[32];
    __shared__ uint32_t s_want;
    __shared__ int s_kr;

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

    if (n <= k) {
        for (int i = threadIdx.x; i < k; i += kRegThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? int32_t(p0 + i) : -1;
        }
        if (threadIdx.x == 0) topk_cnt[b] = n;
        return;
    }
    if (n > kRegThreads * kKpt) {
        topk_large(z, z_by_entry, z_by_entry ? seq_off[b] : 0, kept_idx, p0, n, k, out_idx, out_pos, s_hist, s_warp,
                   &s_want, &s_kr);
        if (threadIdx.x == 0) topk_cnt[b] = k;
        return;
    }
    const int lo = threadIdx.x * kKpt;
    int32_t ids[kKpt];
    uint32_t key[kKpt];
#pragma unroll
    for (int j = 0; j < kKpt; ++j) ids[j] = lo + j < n ? kept_idx[p0 + lo + j] : 0;
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
#pragma unroll
    for (int j = 0; j < kKpt; ++j)
        key[j] = lo + j < n ? order_key(z_by_entry ? z[sbase + ids[j]] : z[p0 + lo + j]) : 0u;

    uint32_t want = 0, hmask = 0;
    int kr = k;
    __shared__ int s_done;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) s_hist[warp][i] = 0;
        __syncthreads();
        // kept scores cluster in a few bins of the leading digits: lanes that hit the same bin are
        // merged first, so a warp issues one shared atomic per distinct bin
#pragma unroll
        for (int j = 0; j < kKpt; ++j) {
            const bool in = lo + j < n && (key[j] & hmask) == want;
            const int digit = in ? int((key[j] >> shift) & 0xFFu) : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (in && (__ffs(peers) - 1) == lane) atomicAdd(&s_hist[warp][digit], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            int sum = 0;
#pragma unroll
            for (int w = 0; w < kRegWarps; ++w) sum += s_hist[w][threadIdx.x];
            s_hist[0][threadIdx.x] = sum;
        }
        __syncthreads();
        if (warp == 0) {
            int local = 0;
#pragma unroll
            for (int x = 0; x < 8; ++x) local += s_hist[0][8 * lane + x];
            int suf = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            int above = suf - local;
#pragma unroll
            for (int x = 7; x >= 0; --x) {
                const int h = s_hist[0][8 * lane + x];
                if (above < kr && above + h >= kr) {
                    s_want = want | (uint32_t(8 * lane + x) << shift);
                    s_kr = kr - above;
                    s_done = (above + h == kr);   // the whole bin is taken: no finer digit needed
                }
                above += h;
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= 0xFFu << shift;
        if (s_done) break;
        __syncthreads();
    }
    // take every key whose resolved digits exceed `want`, and the first kr whose digits equal it
    int n_eq = 0;
#pragma unroll
    for (int j = 0; j < kKpt; ++j) n_eq += (lo + j < n && (key[j] & hmask) == want);
    int tot;
    const int eq_rank = block_excl_scan512(n_eq, s_warp, &tot);
    uint64_t take = 0;   // per-position take flags (kKpt <= 64)
    int n_take = 0;
    {
        int r = eq_rank;
#pragma unroll
        for (int j = 0; j < kKpt; ++j) {
            bool t = false;
            if (lo + j < n) {
                const uint32_t kk = key[j] & hmask;
                if (kk > want) t = true;
                else if (kk == want) { t = r < kr; ++r; }
            }
            if (t) {
                ++n_take;
                take |= uint64_t(1) << j;
            }
        }
    }
    int out = block_excl_scan512(n_take, s_warp, &tot);
#pragma unroll
    for (int j = 0; j < kKpt; ++j) {
        if ((take >> j) & 1u) {
            if (out < k) {
                out_idx[out] = ids[j];
                if (out_pos) out_pos[out] = int32_t(p0 + lo + j);
            }
            ++out;
        }
    }
    if (threadIdx.x == 0) topk_cnt[b] = k;
}

}  // namespace

lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, int32_t *topk_idx, int32_t *topk_pos, int32_t *topk_cnt,
                       cudaStream_t st) {
    // sequences whose kept set fits in registers (all of them at the decode step's shapes unless a
    // sequence keeps more than 24576 entries) are done by topk_reg; the shared-memory kernel runs only
    // when the kept capacity allows a larger set, and then only for such sequences.
    LSA_CUDA(launch_pdl(topk_reg, dim3(B), dim3(kRegThreads), 0, st, z, z_by_entry, seq_off, kept_idx, kept_off,
                        kept_cap, k, topk_idx, topk_pos, topk_cnt));
    LSA_LAUNCHED("topk_reg");
    return LSA_OK;
}

}  // namespace lsa
