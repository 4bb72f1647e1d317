// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One 1024-thread block per sequence.  Scores map to an order-preserving
// 32-bit key (larger z -> larger key, -0.0 folded onto +0.0).  A most-
// significant-digit radix select (4 passes of 8 bits) finds the key T of the
// k-th largest entry and how many entries equal to T must be taken; a final
// ordered pass takes every key > T and the lowest-index entries with key == T,
// and compacts them in kept-list order, which is ascending entry order.
//
// Kept sets of up to kSmemKeys entries are staged once in shared memory; every warp keeps its own 256-bin histogram and lanes that hit the
// same bin are merged with __match_any_sync before one atomic (the kept
// entries' keys share their top byte, so a single histogram would serialise);
// the final pass gives each thread a contiguous run of positions, so it needs
// only two block scans.  Larger kept sets re-read the scores from global
// memory in every pass instead of staging them.
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

constexpr int kSmemKeys = 32768;   // keys staged in shared memory (128 KB)
constexpr int kWarps = kTopkThreads / 32;

__global__ void __launch_bounds__(kTopkThreads)
topk_smem(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
          const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
          int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos, int32_t *__restrict__ topk_cnt,
          int min_n) {
    extern __shared__ uint32_t s_keys[];                 // [n]
    __shared__ int s_hist[kWarps][256];
    __shared__ int s_warp[32];
    __shared__ uint32_t s_want;
    __shared__ int s_kr;

    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t p0 = kept_off[b];
    int64_t n64 = kept_off[b + 1] - p0;
    if (p0 >= kept_cap) n64 = 0;
    else if (p0 + n64 > kept_cap) n64 = kept_cap - p0;
    if (n64 < 0) n64 = 0;
    const int n = int(n64);
    if (n < min_n) return;   // handled by topk_reg
    int32_t *out_idx = topk_idx + int64_t(b) * k;
    int32_t *out_pos = topk_pos ? topk_pos + int64_t(b) * k : nullptr;

    if (n <= k) {   // everything kept is chosen
        for (int i = threadIdx.x; i < k; i += kTopkThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? int32_t(p0 + i) : -1;
        }
        if (threadIdx.x == 0) topk_cnt[b] = n;
        return;
    }
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    const bool staged = n <= kSmemKeys;
    auto key = [&](int i) -> uint32_t {
        return staged ? s_keys[i] : order_key(z_by_entry ? z[sbase + kept_idx[p0 + i]] : z[p0 + i]);
    };
    if (staged)
        for (int i = threadIdx.x; i < n; i += kTopkThreads)
            s_keys[i] = order_key(z_by_entry ? z[sbase + kept_idx[p0 + i]] : z[p0 + i]);

    uint32_t want = 0, hmask = 0;
    int kr = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) s_hist[warp][i] = 0;
        __syncthreads();
        for (int i0 = warp * 32; i0 < n; i0 += kTopkThreads) {
            const int i = i0 + lane;
            const uint32_t u = i < n ? key(i) : 0u;
            const bool in = i < n && (u & hmask) == want;
            const int digit = in ? int((u >> shift) & 0xFFu) : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (in && (__ffs(peers) - 1) == lane) atomicAdd(&s_hist[warp][digit], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 256) {   // fold the warp histograms into warp 0's row
            int sum = 0;
#pragma unroll 8
            for (int w = 0; w < kWarps; ++w) sum += s_hist[w][threadIdx.x];
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
                }
                above += h;
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= 0xFFu << shift;
    }
    // ordered take: thread t owns positions [t*per, (t+1)*per)
    const int per = (n + kTopkThreads - 1) / kTopkThreads;
    const int lo = min(n, threadIdx.x * per), hi = min(n, lo + per);
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += key(i) == want;
    int tot;
    int eq_rank = block_excl_scan(n_eq, s_warp, &tot);
    int n_take = 0;
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key(i);
            if (u > want) ++n_take;
            else if (u == want) { n_take += r < kr; ++r; }
        }
    }
    int out = block_excl_scan(n_take, s_warp, &tot);
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key(i);
            bool take = u > want;
            if (u == want) { take = r < kr; ++r; }
            if (take && out < k) {
                out_idx[out] = kept_idx[p0 + i];
                if (out_pos) out_pos[out] = int32_t(p0 + i);
                ++out;
            }
        }
    }
    if (threadIdx.x == 0) topk_cnt[b] = k;
}

// Register-resident variant for kept sets of up to kRegThreads * kKpt entries:
// thread t owns the contiguous positions [t*kKpt, (t+1)*kKpt) and loads their
// scores and entry indices in one unrolled batch (independent loads in flight
// instead of a chain of dependent ones); the radix passes count from
// registers into per-warp histograms; the ordered take needs two block scans
// and writes each thread's run in order.  Larger kept sets fall back to the
// shared-memory kernel above.
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
    if (n > kRegThreads * kKpt) return;   // left to the shared-memory kernel
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
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) s_hist[warp][i] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kKpt; ++j)
            if (lo + j < n && (key[j] & hmask) == want) atomicAdd(&s_hist[warp][(key[j] >> shift) & 0xFFu], 1);
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
                }
                above += h;
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= 0xFFu << shift;
    }
    int n_eq = 0;
#pragma unroll
    for (int j = 0; j < kKpt; ++j) n_eq += (lo + j < n && key[j] == want);
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
                if (key[j] > want) t = true;
                else if (key[j] == want) { t = r < kr; ++r; }
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
    if (kept_cap > int64_t(kRegThreads) * kKpt) {
        const size_t smem = size_t(kSmemKeys) * 4;
        LSA_CUDA(ensure_smem(topk_smem, smem));
        topk_smem<<<B, kTopkThreads, smem, st>>>(z, z_by_entry, seq_off, kept_idx, kept_off, kept_cap, k, topk_idx,
                                                 topk_pos, topk_cnt, kRegThreads * kKpt + 1);
        LSA_LAUNCHED("topk_smem");
    }
    return LSA_OK;
}

}  // namespace lsa
