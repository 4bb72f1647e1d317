// Fine-grained top-k inside the kept set ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection"): the k largest scores of a sequence's kept entries, ties
// to the lower kept-list position, returned in kept-list (= ascending entry)
// order.
//
// One CTA of 1024 threads per sequence; scores map to an order-preserving
// 32-bit key (larger z -> larger key, -0.0 folded onto +0.0) staged in shared
// memory.  With one CTA per sequence the kernel is bound by instruction issue
// and by shared-memory atomics (kept scores cluster in few histogram bins), so
// the common case touches every key only twice after staging, with no atomics:
//   1. 64 keys sampled at evenly spaced positions give two pivots lo <= hi that
//      bracket the k-th largest with high probability (a margin of 2.5 binomial
//      standard deviations around its expected sample rank);
//   2. one pass counts the keys above hi and copies the keys in [lo, hi] (about
//      a fifth of them) to a list, one region per warp, appended by ballots;
//   3. if the bracket holds (fewer than k above hi, at least k up to lo), a
//      radix-style select over the list alone narrows the key interval [lo, hi]
//      to the one holding the k-th largest: each pass splits the interval into
//      4096 equal bins (of a power-of-two width), counts the listed keys per bin
//      and keeps the bin holding it, until the bin holds only keys that are all
//      taken or one key value; otherwise the same select runs over every key,
//      from the whole key range (the exact fallback);
//   4. one ordered pass takes every key above the threshold interval and the
//      lowest-position keys inside it: warp w owns a contiguous segment, and
//      ballots give each taken key its output slot, the warps' offsets coming
//      from the list (or, on the fallback, from one counting pass).
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
constexpr int kStageKeys = 32768;   // keys staged in shared memory (128 KB)
constexpr int kMaxK = 4096;          // the largest k (the entry points check it); positions of the chosen in smem
constexpr int kListW = 256;          // listed keys per warp
constexpr int kList = kListW * kWarps;   // 8192 (32 KB)
constexpr int kDigit = 12;
constexpr int kBins = 1 << kDigit;   // 4096: four per thread
constexpr int kSamples = 64;         // two per lane of warp 0
constexpr size_t kSmemBytes = size_t(kStageKeys + 4 + kMaxK + kList + kBins) * 4;

// A compile-time flag for code specialised on where the keys live.
template <bool V>
struct Flag {
    static constexpr bool value = V;
};

__global__ void __launch_bounds__(kThreads, 1)
topk_select(const float *__restrict__ z, int z_by_entry, const int64_t *__restrict__ seq_off,
            const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int64_t kept_cap, int k,
            const int32_t *__restrict__ pos_map, int32_t *__restrict__ topk_idx, int32_t *__restrict__ topk_pos,
            int32_t *__restrict__ topk_cnt) {
    // [kStageKeys + 4] keys | [kMaxK] positions of the chosen | [kList] listed keys | [kBins] histogram
    extern __shared__ __align__(16) uint32_t s_keys[];
    int *s_pos = reinterpret_cast<int *>(s_keys + kStageKeys + 4);
    uint32_t *s_list = reinterpret_cast<uint32_t *>(s_pos + kMaxK);
    int *s_hist = reinterpret_cast<int *>(s_list + kList);
    __shared__ int s_warp[kWarps];
    __shared__ int s_chi[kWarps], s_cnt[kWarps];   // per warp: keys above hi, keys listed
    __shared__ int s_red[2][kWarps];
    __shared__ uint32_t s_lo, s_hi, s_ilo, s_ihi;
    __shared__ int s_kr, s_done, s_binc;

    pdl_launch_dependents();   // attention may stage its queries meanwhile
    pdl_wait();                // scores come from the preceding scan
    const int b = blockIdx.x;
    const int t = int(threadIdx.x), lane = t & 31, warp = t >> 5;
    const uint32_t full = 0xffffffffu, lt = (1u << lane) - 1u;
    const int64_t p0 = kept_off[b];
    int64_t n64 = kept_off[b + 1] - p0;
    if (p0 >= kept_cap) n64 = 0;
    else if (p0 + n64 > kept_cap) n64 = kept_cap - p0;
    if (n64 < 0) n64 = 0;
    const int n = int(n64);
    int32_t *out_idx = topk_idx + int64_t(b) * k;
    int32_t *out_pos = topk_pos ? topk_pos + int64_t(b) * k : nullptr;

    if (n <= k) {   // everything kept is chosen
        for (int i = t; i < k; i += kThreads) {
            out_idx[i] = i < n ? kept_idx[p0 + i] : -1;
            if (out_pos) out_pos[i] = i < n ? (pos_map ? pos_map[p0 + i] : int32_t(p0 + i)) : -1;
        }
        if (t == 0) topk_cnt[b] = n;
        return;
    }
    const int64_t sbase = z_by_entry ? seq_off[b] : 0;
    const bool staged = n <= kStageKeys;
    auto load_z = [&](int i) -> float {   // i: position in the sequence's kept list
        const int64_t p = p0 + i;
        return z_by_entry ? z[sbase + kept_idx[p]] : z[p];
    };
    const float *zs = z + p0;
    // listed scores are staged with 16-byte loads from their first 16-byte boundary (`head` scores in); the
    // staged copy is shifted by `aoff` so that those vectors land on 16-byte boundaries too
    const bool vec = !z_by_entry && staged;
    const int head = vec ? min(n, int((4 - ((reinterpret_cast<uintptr_t>(zs) >> 2) & 3)) & 3)) : 0;
    const int aoff = (4 - head) & 3;
    uint32_t *sk = s_keys + aoff;   // the key of position i is sk[i]
    // the key of position i, with the branch on where keys live taken at compile time
    auto key_of = [&](auto where, int i) -> uint32_t {
        if constexpr (decltype(where)::value) return sk[i];
        else return order_key(load_z(i));
    };
    auto specialised = [&](auto &&f) {
        if (staged) f(Flag<true>{});
        else f(Flag<false>{});
    };

#pragma unroll
    for (int q = 0; q < kBins / kThreads; ++q) s_hist[t + q * kThreads] = 0;   // readers re-zero their bins
    for (int j = t; j < k; j += kThreads) s_pos[j] = -1;   // a slot left unfilled yields -1, not a stray read

    if (warp == 0) {
        // 1. the sample, ranked by warp 0 alone while the other warps stage: the sample at descending index
        // i has gt <= i < gt + eq
        const uint32_t a = order_key(load_z(int((int64_t(2 * lane + 1) * n) / (2 * kSamples))));
        const uint32_t c = order_key(load_z(int((int64_t(2 * (lane + 32) + 1) * n) / (2 * kSamples))));
        int gta = 0, eqa = 0, gtc = 0, eqc = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const uint32_t x = __shfl_sync(full, a, j), y = __shfl_sync(full, c, j);
            gta += int(x > a) + int(y > a);
            eqa += int(x == a) + int(y == a);
            gtc += int(x > c) + int(y > c);
            eqc += int(x == c) + int(y == c);
        }
        // the k-th largest is expected at sample index r = 64 k / n, with binomial spread
        const float frac = float(k) / float(n);
        const float r = float(kSamples) * frac;
        const int margin = int(ceilf(2.5f * sqrtf(r * (1.f - frac)))) + 1;
        const int i_hi = int(r) - margin, i_lo = int(r) + margin;
        auto at = [&](int i, uint32_t *dst) {
            if (gta <= i && i < gta + eqa) *dst = a;   // equal samples write equal values
            if (gtc <= i && i < gtc + eqc) *dst = c;
        };
        if (i_hi >= 0) at(i_hi, &s_hi);
        else if (lane == 0) s_hi = 0xFFFFFFFFu;
        if (i_lo < kSamples) at(i_lo, &s_lo);
        else if (lane == 0) s_lo = 0u;
    } else if (vec) {
        // warps 1.. stage
        const int ts = t - 32, ns = kThreads - 32;
        const int nv = (n - head) >> 2;
        const float4 *z4 = reinterpret_cast<const float4 *>(zs + head);
        for (int j0 = ts; j0 < nv; j0 += 4 * ns) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (j0 + u * ns < nv) v[u] = z4[j0 + u * ns];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * ns;
                if (j < nv)
                    *reinterpret_cast<uint4 *>(sk + head + 4 * j) =
                        make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z), order_key(v[u].w));
            }
        }
        // the scores before the first boundary (threads 32..35) and after the last whole vector (36..39)
        if (ts < 8) {
            const int i = ts < 4 ? ts : head + 4 * nv + ts - 4;
            if (ts < 4 ? i < head : i < n) sk[i] = order_key(zs[i]);
        }
    } else if (staged) {
        const int ts = t - 32, ns = kThreads - 32;
        for (int i0 = ts; i0 < n; i0 += 8 * ns) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * ns < n) v[u] = load_z(i0 + u * ns);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * ns < n) sk[i0 + u * ns] = order_key(v[u]);
        }
    }
    __syncthreads();   // publishes the staged keys and the pivots

    // 2. keys above hi (counted) and in [lo, hi] (listed); warp w owns positions [w_lo, w_hi)
    uint32_t lo = s_lo, hi = s_hi;
    const int seg = ((n + kThreads - 1) / kThreads) * 32;
    const int w_lo = min(n, warp * seg), w_hi = min(n, w_lo + seg);
    uint32_t *reg = s_list + warp * kListW;
    int nlist;
    {
        const uint32_t span = hi - lo;
        int c_hi = 0, cnt = 0;
        specialised([&](auto where) {
            for (int q0 = w_lo; q0 < w_hi; q0 += 4 * 32) {   // warp-uniform trip count
                uint32_t u[4], m[4];
                bool v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int p = q0 + 32 * q + lane;
                    v[q] = p < w_hi;
                    u[q] = v[q] ? key_of(where, p) : 0u;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    c_hi += int(v[q] && u[q] > hi);
                    m[q] = __ballot_sync(full, v[q] && u[q] - lo <= span);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int slot = cnt + __popc(m[q] & lt);
                    if (((m[q] >> lane) & 1u) && slot < kListW) reg[slot] = u[q];
                    cnt += __popc(m[q]);
                }
            }
        });
        c_hi = __reduce_add_sync(full, c_hi);
        if (lane == 0) { s_chi[warp] = c_hi; s_cnt[warp] = cnt; }
        nlist = min(cnt, kListW);
    }
    __syncthreads();
    const int n_hi = __reduce_add_sync(full, s_chi[lane]);
    const int n_in = __reduce_add_sync(full, s_cnt[lane]);
    const bool bracket = !__any_sync(full, s_cnt[lane] > kListW) && n_hi < k && n_hi + n_in >= k;   // uniform

    // 3. select over the list (or every key): [ilo, ihi] holds the kr-th largest of the source's keys in it
    int kr, binc;   // binc: the source's keys in [ilo, ihi]
    uint32_t ilo, ihi;
    if (bracket) {
        kr = k - n_hi;
        ilo = lo;
        ihi = hi;
        binc = n_in;
    } else {
        kr = k;
        ilo = 0u;
        ihi = 0xFFFFFFFFu;
        binc = n;
    }
    while (ilo != ihi) {   // uniform
        const uint32_t span = ihi - ilo;
        const int bits = 32 - __clz(span);
        const int sh = bits > kDigit ? bits - kDigit : 0;   // 4096 bins of 2^sh key values cover the interval
        if (bracket) {
            for (int j = lane; j < nlist; j += 32) {
                const uint32_t u = reg[j] - ilo;
                if (u <= span) atomicAdd(&s_hist[u >> sh], 1);
            }
        } else {
            specialised([&](auto where) {
                for (int p = t; p < n; p += kThreads) {
                    const uint32_t u = key_of(where, p) - ilo;
                    if (u <= span) atomicAdd(&s_hist[u >> sh], 1);
                }
            });
        }
        __syncthreads();
        {   // thread t owns bins 4095 - 4t .. 4092 - 4t (descending key order).  The warp sums locate the warp
            // whose bins hold the kr-th key; that warp alone scans its lanes.
            const int bh = kBins - 1 - 4 * t;
            int h[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                h[q] = s_hist[bh - q];
                s_hist[bh - q] = 0;   // only this thread reads these bins
            }
            const int mine = h[0] + h[1] + h[2] + h[3];
            const int wsum = __reduce_add_sync(full, mine);
            if (lane == 0) s_warp[warp] = wsum;
            __syncthreads();
            const int above_w = __reduce_add_sync(full, lane < warp ? s_warp[lane] : 0);
            if (above_w < kr && above_w + wsum >= kr) {   // warp-uniform
                int x = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(full, x, o);
                    if (lane >= o) x += y;
                }
                int above = above_w + x - mine;   // keys in bins above bh
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (above < kr && above + h[q] >= kr) {
                        const uint32_t blo = ilo + (uint32_t(bh - q) << sh), wmax = (1u << sh) - 1u;
                        s_ilo = blo;
                        s_ihi = ihi - blo < wmax ? ihi : blo + wmax;
                        s_kr = kr - above;
                        s_done = (above + h[q] == kr);
                        s_binc = h[q];
                    }
                    above += h[q];
                }
            }
        }
        __syncthreads();
        ilo = s_ilo;
        ihi = s_ihi;
        kr = s_kr;
        binc = s_binc;
        if (s_done) break;   // uniform: read after the barrier, rewritten only after the next barrier
    }
    // keys in [e_lo, e_hi] (binc of them) are the candidates at the threshold, kr of them taken; keys above
    // e_hi are all taken
    const uint32_t e_lo = ilo, e_hi = ihi, espan = e_hi - e_lo;
    const bool all_eq = kr == binc;   // uniform

    // 4. ordered take.  Keys above and inside the interval in the warps before this one:
    int a_w = 0, e_w = 0;
    if (bracket) {
        for (int j = lane; j < nlist; j += 32) {
            const uint32_t u = reg[j];
            a_w += int(u > e_hi);
            e_w += int(u - e_lo <= espan);
        }
        a_w = __reduce_add_sync(full, a_w) + s_chi[warp];
    } else {
        specialised([&](auto where) {
            for (int p = w_lo + lane; p < w_hi; p += 32) {
                const uint32_t u = key_of(where, p);
                a_w += int(u > e_hi);
                e_w += int(u - e_lo <= espan);
            }
        });
        a_w = __reduce_add_sync(full, a_w);
    }
    e_w = __reduce_add_sync(full, e_w);
    if (lane == 0) { s_red[0][warp] = a_w; s_red[1][warp] = e_w; }
    __syncthreads();
    int a_run = __reduce_add_sync(full, lane < warp ? s_red[0][lane] : 0);
    int e_run = __reduce_add_sync(full, lane < warp ? s_red[1][lane] : 0);
    if (all_eq) a_run += e_run;   // one running count of taken keys
    // a taken key with `a` keys above and `e` inside the interval before it goes to slot a + min(e, kr)
    specialised([&](auto where) {
        for (int q0 = w_lo; q0 < w_hi; q0 += 4 * 32) {   // warp-uniform trip count
            uint32_t u[4], ba[4], be[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int p = q0 + 32 * q + lane;
                u[q] = p < w_hi ? key_of(where, p) : 0u;
            }
            if (all_eq) {   // every key from e_lo up is taken: a_run counts both kinds
#pragma unroll
                for (int q = 0; q < 4; ++q) ba[q] = __ballot_sync(full, q0 + 32 * q + lane < w_hi && u[q] >= e_lo);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int slot = a_run + __popc(ba[q] & lt);
                    if (((ba[q] >> lane) & 1u) && slot < k) s_pos[slot] = q0 + 32 * q + lane;
                    a_run += __popc(ba[q]);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const bool v = q0 + 32 * q + lane < w_hi;
                    ba[q] = __ballot_sync(full, v && u[q] > e_hi);
                    be[q] = __ballot_sync(full, v && u[q] - e_lo <= espan);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int eb = e_run + __popc(be[q] & lt);
                    const int slot = a_run + __popc(ba[q] & lt) + min(eb, kr);
                    const bool take = ((ba[q] >> lane) & 1u) || (((be[q] >> lane) & 1u) && eb < kr);
                    if (take && slot < k) s_pos[slot] = q0 + 32 * q + lane;
                    a_run += __popc(ba[q]);
                    e_run += __popc(be[q]);
                }
            }
        }
    });
    __syncthreads();
    // the entry indices of the chosen positions, fetched with independent loads
    for (int j = t; j < k; j += kThreads) {
        const int i = s_pos[j];
        const bool ok = 0 <= i && i < n;
        const int64_t p = p0 + (ok ? i : 0);
        out_idx[j] = ok ? kept_idx[p] : -1;
        if (out_pos) out_pos[j] = !ok ? -1 : (pos_map ? pos_map[p] : int32_t(p));
    }
    if (t == 0) topk_cnt[b] = k;
}

}  // namespace

lsa_status launch_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                       const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int32_t k,
                       int64_t kept_cap, const int32_t *pos_map, int32_t *topk_idx, int32_t *topk_pos,
                       int32_t *topk_cnt, cudaStream_t st) {
    const size_t smem = kSmemBytes;
    LSA_CUDA(ensure_smem(topk_select, smem));
    LSA_CUDA(launch_pdl(topk_select, dim3(B), dim3(kThreads), smem, st, z, z_by_entry, seq_off, kept_idx, kept_off,
                        kept_cap, k, pos_map, topk_idx, topk_pos, topk_cnt));
    LSA_LAUNCHED("topk_select");
    return LSA_OK;
}

}  // namespace lsa
