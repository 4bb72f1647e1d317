// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection").
//
// One 8-CTA cluster per sequence.  Scores map to an order-preserving 32-bit
// key (larger z -> larger key, -0.0 folded onto +0.0).  A most-significant-
// digit radix select (passes of 8 bits) finds the digits of the k-th
// largest key and how many entries sharing them must be taken; an ordered pass
// then takes every key above and the lowest-index entries at the threshold,
// and compacts them in kept-list order, which is ascending entry order.
#include <cooperative_groups.h>

#include "lsa_internal.cuh"

namespace lsa {
namespace {

__device__ __forceinline__ uint32_t order_key(float z) {
    uint32_t b = __float_as_uint(z);
    if (b == 0x80000000u) b = 0u;                      // -0.0 ranks as +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kCluster = 8;          // CTAs per sequence (one thread-block cluster)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStageKeys = 8192;     // keys per CTA staged in shared memory (32 KB)

// Exclusive block-wide prefix sum (kThreads threads); *total receives the sum.
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

// One cluster of kCluster CTAs per sequence; CTA r owns the kept positions
// [r*n/8, (r+1)*n/8) and, inside it, thread t a contiguous run.  Keys are
// staged in shared memory with batched (independent) loads.  Cluster-wide
// quantities (min / max key, the histogram of each radix pass, the counts
// feeding the ordered take) are combined through distributed shared memory:
// every CTA publishes its local values, the cluster synchronises, and every CTA
// reads all kCluster copies and reaches the same decision.
//
// The radix digits start below the bits that every key shares (the common
// prefix of the minimum and maximum key): kept scores sit in a narrow positive
// range, so the leading bits are constant and a digit there would say nothing
// while funnelling every key into one histogram bin.  The select stops as soon
// as the threshold bin holds exactly the entries still needed.
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
topk_select(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
            const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
            const int32_t *__restrict__ pos_map, int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos,
            int32_t *__restrict__ topk_cnt) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ uint32_t s_keys[kStageKeys];
    __shared__ int s_hist[kWarps][256];
    __shared__ int s_chist[256];          // this CTA's histogram, read by the whole cluster
    __shared__ int s_warp[32];
    __shared__ uint32_t s_red[2][kWarps];
    __shared__ uint32_t s_mm[2];          // this CTA's min / max key
    __shared__ int s_cnt[2];              // this CTA's (equal, taken) counts
    __shared__ uint32_t s_want;
    __shared__ int s_kr, s_done;

    pdl_launch_dependents();   // attention may stage its queries meanwhile
    pdl_wait();                // scores come from the preceding scan
    const int b = blockIdx.y;
    const int rank = int(cluster.block_rank());
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t p0 = kept_off[b];
    int64_t n64 = kept_off[b + 1] - p0;
    if (p0 >= kept_cap) n64 = 0;
    else if (p0 + n64 > kept_cap) n64 = kept_cap - p0;
    if (n64 < 0) n64 = 0;
    const int n = int(n64);
    int32_t *out_idx = topk_idx + int64_t(b) * k;
    int32_t *out_pos = topk_pos ? topk_pos + int64_t(b) * k : nullptr;

    if (n <= k) {   // everything kept is chosen (uniform over the cluster: no cluster barrier is reached)
        for (int i = rank * kThreads + int(threadIdx.x); i < k; i += kCluster * kThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? (pos_map ? pos_map[p0 + i] : int32_t(p0 + i)) : -1;
        }
        if (rank == 0 && threadIdx.x == 0) topk_cnt[b] = n;
        return;
    }
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    // this CTA's slice and this thread's run inside it
    const int c_lo = int(int64_t(n) * rank / kCluster), c_hi = int(int64_t(n) * (rank + 1) / kCluster);
    const int cn = c_hi - c_lo;
    const bool staged = cn <= kStageKeys;
    const int per = (cn + kThreads - 1) / kThreads;
    const int lo = min(cn, int(threadIdx.x) * per), hi = min(cn, lo + per);   // local positions
    auto load_key = [&](int i) -> uint32_t {   // i: local position
        const int64_t p = p0 + c_lo + i;
        return order_key(z_by_entry ? z[sbase + kept_idx[p]] : z[p]);
    };
    auto key = [&](int i) -> uint32_t { return staged ? s_keys[i] : load_key(i); };

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
        s_mm[0] = a;
        s_mm[1] = c;
    }
    cluster.sync();
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
    for (int r = 0; r < kCluster; ++r) {
        const uint32_t *mm = cluster.map_shared_rank(s_mm, r);
        gmin = min(gmin, mm[0]);
        gmax = max(gmax, mm[1]);
    }
    const uint32_t diff = gmin ^ gmax;
    int top = diff ? 31 - __clz(diff) : -1;   // bits above `top` are shared by every key
    uint32_t hmask = top >= 31 ? 0u : (top >= 0 ? ~((2u << top) - 1u) : 0xFFFFFFFFu);
    uint32_t want = gmin & hmask;
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
        {   // this CTA's histogram
            int sum = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += s_hist[w][threadIdx.x];
            s_chist[threadIdx.x] = sum;
        }
        cluster.sync();
        {   // the cluster's histogram (bin = thread)
            int sum = 0;
#pragma unroll
            for (int r = 0; r < kCluster; ++r) sum += cluster.map_shared_rank(s_chist, r)[threadIdx.x];
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
        const bool done = s_done;
        cluster.sync();   // every CTA has read the others' histograms before they are rewritten
        if (done) break;
    }
    // ordered take: keys whose resolved bits exceed `want`, then the first kr equal to it
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (key(i) & hmask) == want;
    int tot;
    int eq_rank = block_excl_scan(n_eq, s_warp, &tot);
    if (threadIdx.x == 0) s_cnt[0] = tot;
    cluster.sync();
    for (int r = 0; r < rank; ++r) eq_rank += cluster.map_shared_rank(s_cnt, r)[0];
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
    if (threadIdx.x == 0) s_cnt[1] = tot;
    cluster.sync();
    for (int r = 0; r < rank; ++r) out += cluster.map_shared_rank(s_cnt, r)[1];
    // the run in segments of 64 positions: take flags first, then the entry indices of the taken
    // positions in batches of independent loads
    int r = eq_rank;
    for (int s0 = lo; s0 < hi; s0 += 64) {
        const int s1 = min(hi, s0 + 64);
        uint64_t take = 0;
        for (int i = s0; i < s1; ++i) {
            const uint32_t u = key(i) & hmask;
            bool t = u > want;
            if (u == want) { t = r < kr; ++r; }
            if (t) take |= uint64_t(1) << (i - s0);
        }
        while (take) {
            int js[8], nj = 0;
            while (take && nj < 8) { js[nj++] = __ffsll(take) - 1; take &= take - 1; }
            int32_t ids[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) ids[u] = u < nj ? kept_idx[p0 + c_lo + s0 + js[u]] : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (u < nj) {
                    if (out < k) {
                        out_idx[out] = ids[u];
                        if (out_pos) {
                            const int64_t p = p0 + c_lo + s0 + js[u];
                            out_pos[out] = pos_map ? pos_map[p] : int32_t(p);
                        }
                    }
                    ++out;
                }
        }
    }
    if (rank == 0 && threadIdx.x == 0) topk_cnt[b] = k;
    cluster.sync();   // no CTA leaves while another may still read its shared memory
}

}  // namespace

lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, const int32_t *pos_map, int32_t *topk_idx, int32_t *topk_pos,
                       int32_t *topk_cnt, cudaStream_t st) {
    LSA_CUDA(launch_pdl(topk_select, dim3(kCluster, B), dim3(kThreads), 0, st, z, z_by_entry, seq_off, kept_idx,
                        kept_off, kept_cap, k, pos_map, topk_idx, topk_pos, topk_cnt));
    LSA_LAUNCHED("topk_select");
    return LSA_OK;
}

}  // namespace lsa
