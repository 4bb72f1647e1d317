// Threshold selection ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse
// Attention", gist.science technical summary, section 2.1 "Dynamic
// Fetching"): keep every entry with I >= 0.5, i.e. z >= 0, as an ordered
// (stable) stream compaction on the flat entry axis.
//
// Three short kernels, no device-side waits:
//   1. flags:   per 1024-entry tile, warp ballots of (z >= 0) -> mask words,
//               popcount -> tile count;
//   2. scan:    one block scans the tile counts into tile bases (and checks
//               the capacity);
//   3. scatter: per tile, each kept entry's rank = tile base + prefix of the
//               mask bits before it; writes its local index, and the kept
//               offset of every sequence that starts inside the tile.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kSelTile = 1024;           // entries per tile
constexpr int kSelThreads = 256;         // 8 warps x 128 entries
constexpr int kWordsPerTile = kSelTile / 32;

__global__ void __launch_bounds__(kSelThreads)
select_flags(const float *__restrict__ z, int64_t n, uint32_t *__restrict__ mask,
             int32_t *__restrict__ tile_cnt) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t base = int64_t(blockIdx.x) * kSelTile + warp * 128;
    int cnt = 0;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int64_t e = base + it * 32 + lane;
        const bool keep = e < n && z[e] >= 0.0f;
        const uint32_t word = __ballot_sync(0xffffffffu, keep);
        const int64_t wi = (base + it * 32) >> 5;
        if (lane == 0 && (wi << 5) < n) mask[wi] = word;
        cnt += __popc(word);
    }
    __shared__ int s_cnt[kSelThreads / 32];
    if (lane == 0) s_cnt[warp] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int i = 0; i < kSelThreads / 32; ++i) t += s_cnt[i];
        tile_cnt[blockIdx.x] = t;
    }
}

// Exclusive scan of tile counts by one block of 1024 threads.
__global__ void __launch_bounds__(1024)
select_scan(const int32_t *__restrict__ tile_cnt, int64_t tiles, int64_t *__restrict__ tile_base,
            int64_t *__restrict__ kept_off, int B, int64_t capacity, int32_t *err) {
    __shared__ int64_t s_warp[32];
    __shared__ int64_t s_carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int64_t t0 = 0; t0 < tiles; t0 += 1024) {
        const int64_t t = t0 + threadIdx.x;
        const int64_t v = t < tiles ? tile_cnt[t] : 0;
        int64_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int64_t s = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int64_t y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            s_warp[lane] = s;  // inclusive over warps
        }
        __syncthreads();
        const int64_t warp_excl = warp ? s_warp[warp - 1] : 0;
        const int64_t carry = s_carry;
        if (t < tiles) tile_base[t] = carry + warp_excl + x - v;
        __syncthreads();
        if (threadIdx.x == 0) s_carry = carry + s_warp[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const int64_t total = s_carry;
        kept_off[B] = total;
        if (total > capacity) raise_err(err, LSA_ERR_CAPACITY);
    }
}

__global__ void __launch_bounds__(kSelThreads)
select_scatter(const uint32_t *__restrict__ mask, const int64_t *__restrict__ tile_base, int64_t n,
               const int64_t *__restrict__ seq_off, int B, int32_t *__restrict__ kept_idx,
               int64_t capacity, int64_t *__restrict__ kept_off) {
    __shared__ uint32_t s_words[kWordsPerTile];
    __shared__ int s_wpre[kWordsPerTile + 1];
    const int64_t tile = blockIdx.x;
    const int64_t e0 = tile * kSelTile;
    const int64_t nwords = (n + 31) >> 5;
    if (threadIdx.x < kWordsPerTile) {
        const int64_t wi = (e0 >> 5) + threadIdx.x;
        s_words[threadIdx.x] = wi < nwords ? mask[wi] : 0u;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int i = 0; i < kWordsPerTile; ++i) { s_wpre[i] = acc; acc += __popc(s_words[i]); }
        s_wpre[kWordsPerTile] = acc;
    }
    __syncthreads();
    const int64_t base = tile_base[tile];
    // every entry of the tile, 4 per thread, consecutive entries across a warp
    for (int i = threadIdx.x; i < kSelTile; i += kSelThreads) {
        const int64_t e = e0 + i;
        if (e >= n) break;
        const uint32_t word = s_words[i >> 5];
        const int bit = i & 31;
        if ((word >> bit) & 1u) {
            const int64_t rank = base + s_wpre[i >> 5] + __popc(word & ((1u << bit) - 1u));
            if (rank < capacity) {
                const int b = seq_of(seq_off, B, e);
                kept_idx[rank] = int32_t(e - seq_off[b]);
            }
        }
    }
    // kept offsets of the sequences that start in this tile
    for (int b = threadIdx.x; b < B; b += kSelThreads) {
        const int64_t s = seq_off[b];
        if (s >= e0 && s < e0 + kSelTile && s < n) {
            const int i = int(s - e0);
            const uint32_t word = s_words[i >> 5];
            const int bit = i & 31;
            kept_off[b] = base + s_wpre[i >> 5] + __popc(word & ((1u << bit) - 1u));
        }
    }
}

// Sequences that start at or past the end of the axis (empty trailing
// sequences, or n == 0) begin at the total.
__global__ void select_tail_offsets(const int64_t *__restrict__ seq_off, int B, int64_t n,
                                    int64_t *__restrict__ kept_off) {
    for (int b = threadIdx.x; b < B; b += blockDim.x)
        if (seq_off[b] >= n) kept_off[b] = kept_off[B];
}

}  // namespace

lsa_status launch_select(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B,
                         int32_t *kept_idx, int64_t capacity, int64_t *kept_off, uint32_t *mask,
                         void *workspace, int32_t *err, cudaStream_t st) {
    const int64_t tiles = (n_total + kSelTile - 1) / kSelTile;
    // workspace: tile_base [tiles] int64 | tile_cnt [tiles] int32 | mask words [words]
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int64_t *tile_base = reinterpret_cast<int64_t *>(ws);
    int32_t *tile_cnt = reinterpret_cast<int32_t *>(ws + align_up(size_t(tiles) * 8, 256));
    uint32_t *mwords = mask ? mask
                            : reinterpret_cast<uint32_t *>(ws + align_up(size_t(tiles) * 8, 256) +
                                                           align_up(size_t(tiles) * 4, 256));
    if (tiles > 0) {
        select_flags<<<unsigned(tiles), kSelThreads, 0, st>>>(z, n_total, mwords, tile_cnt);
        LSA_LAUNCHED("select_flags");
    }
    select_scan<<<1, 1024, 0, st>>>(tile_cnt, tiles, tile_base, kept_off, B, capacity, err);
    LSA_LAUNCHED("select_scan");
    if (tiles > 0) {
        select_scatter<<<unsigned(tiles), kSelThreads, 0, st>>>(mwords, tile_base, n_total, seq_off, B,
                                                               kept_idx, capacity, kept_off);
        LSA_LAUNCHED("select_scatter");
    }
    select_tail_offsets<<<1, 256, 0, st>>>(seq_off, B, n_total, kept_off);
    LSA_LAUNCHED("select_tail_offsets");
    return LSA_OK;
}

}  // namespace lsa
