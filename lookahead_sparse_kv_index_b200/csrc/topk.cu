// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One 512-thread block per sequence.  Scores map to an order-preserving 32-bit
// key (larger z -> larger key, -0.0 folded onto +0.0).  A most-significant-
// digit radix select (passes of 8 bits) finds the digits of the k-th
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

// Block-wide reductions for 512 threads.
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemKeys = 40960;   // keys staged in shared memory (160 KB)

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
        int s = lane < kWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kWarps) s_warp[lane] = s;
    }
    __syncthreads();
    const int res = (warp ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kWarps - 1];
    __syncthreads();
    return res;
}

// Kept sets of up to kSmemKeys entries are staged once in shared memory with
// batched (independent) loads; larger ones re-read the scores from global
// memory in every pass.  The radix digits start below the bits that every key
// shares (the common prefix of the block's min and max key): kept scores sit
// in a narrow positive range, so the leading bits are constant and a digit
// there would say nothing while funnelling every key into one histogram bin.
// Each warp counts into its own 256-bin histogram; each thread walks its own
// contiguous run of positions, so the final ordered take needs two block scans.
__global__ void __launch_bounds__(kThreads)
topk_select(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
            const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
            int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos, int32_t *__restrict__ topk_cnt) {
    extern __shared__ uint32_t s_keys[];
    __shared__ int s_hist[kWarps][256];
    __shared__ int s_warp[32];
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
            if (out_pos) out_pos[i] = i < n ? int32_t(p0 + i) : -1;
        }
        if (threadIdx.x == 0) topk_cnt[b] = n;
        return;
    }
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    const bool staged = n <= kSmemKeys;
    auto load_key = [&](int i) -> uint32_t {
        return order_key(z_by_entry ? z[sbase + kept_idx[p0 + i]] : z[p0 + i]);
    };
    auto key = [&](int i) -> uint32_t { return staged ? s_keys[i] : load_key(i); };

    // thread t owns positions [lo, hi)
    const int per = (n + kThreads - 1) / kThreads;
    const int lo = min(n, int(threadIdx.x) * per), hi = min(n, lo + per);

    // stage (8 loads in flight per thread) and reduce min / max
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i0 = lo; i0 < hi; i0 += 8) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = i0 + u < hi ? load_key(i0 + u) : 0u;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + u < hi) {
                if (staged) s_keys[i0 + u] = v[u];
                kmin = min(kmin, v[u]);
                kmax = max(kmax, v[u]);
            }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) { s_red[0][warp] = kmin; s_red[1][warp] = kmax; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0xFFFFFFFFu, c = 0u;
        for (int w = 0; w < kWarps; ++w) { a = min(a, s_red[0][w]); c = max(c, s_red[1][w]); }
        s_red[0][0] = a;
        s_red[1][0] = c;
    }
    __syncthreads();
    const uint32_t diff = s_red[0][0] ^ s_red[1][0];
    // bits above `top` are shared by every key
    int top = diff ? 31 - __clz(diff) : -1;

    uint32_t want = top >= 0 ? (s_red[0][0] & ~((2u << top) - 1u)) : s_red[0][0];
    uint32_t hmask = top >= 0 ? ~((2u << top) - 1u) : 0xFFFFFFFFu;
    if (top == 31) { want = 0; hmask = 0; }
    int kr = k;
    while (top >= 0) {
        const int width = top + 1 < 8 ? top + 1 : 8;
        const int shift = top + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        for (int i = lane; i < 256; i += 32) s_hist[warp][i] = 0;
        __syncthreads();
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key(i);
            if ((u & hmask) == want) atomicAdd(&s_hist[warp][(u >> shift) & dmask], 1);
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            int sum = 0;
#pragma unroll
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
                    s_done = (above + h == kr);   // the whole bin is taken
                }
                above += h;
            }
        }
        __syncthreads();
        want = s_want;
        kr = s_kr;
        hmask |= dmask << shift;
        top = shift - 1;
        if (s_done) break;
        __syncthreads();
    }
    // take every key whose resolved bits exceed `want`, and the first kr equal to it
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (key(i) & hmask) == want;
    int tot;
    const int eq_rank = block_excl_scan(n_eq, s_warp, &tot);
    int n_take = 0;
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = key(i) & hmask;
            if (u > want) ++n_take;
            else if (u == want) { n_take += r < kr; ++r; }
        }
    }
    int out = block_excl_scan(n_take, s_warp, &tot);
    int r = eq_rank;
    for (int i = lo; i < hi; ++i) {
        const uint32_t u = key(i) & hmask;
        bool take = u > want;
        if (u == want) { take = r < kr; ++r; }
        if (take) {
            if (out < k) {
                out_idx[out] = kept_idx[p0 + i];
                if (out_pos) out_pos[out] = int32_t(p0 + i);
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
    const size_t smem = size_t(kSmemKeys) * 4;
    LSA_CUDA(ensure_smem(topk_select, smem));
    LSA_CUDA(launch_pdl(topk_select, dim3(B), dim3(kThreads), smem, st, z, z_by_entry, seq_off, kept_idx, kept_off,
                        kept_cap, k, topk_idx, topk_pos, topk_cnt));
    LSA_LAUNCHED("topk_select");
    return LSA_OK;
}

}  // namespace lsa
