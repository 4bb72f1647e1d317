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
//
// Fused with the tensor-core scan (select_tiles_*): the scan's epilogue takes
// the z >= 0 ballots of the rows it has just scored (one word per 32 rows of a
// scan tile, and the kept count of each quarter of the tile), so z is not read
// again; one block then turns the tile counts into tile bases and the kept
// offsets, and one CTA per scan tile scatters its kept rows.
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

// ---- selection fused with the scan: scan tile t covers rows [row0_t, row0_t + TR) of one sequence (the
// tiles of each sequence in turn, ceil(len / TR) of them); bits: TR / 32 words per tile; cnt: 4 counts per tile.

// One block: tile bases (exclusive prefix of the tiles' kept counts), each tile's first row and sequence, the
// kept offsets (kept_off[B] the true total; LSA_ERR_CAPACITY when it exceeds capacity) and the tile count.
__global__ void __launch_bounds__(1024)
select_tiles_scan(const int32_t *__restrict__ cnt, const int64_t *__restrict__ seq_off, int B, int TR,
                  int64_t *__restrict__ tile_base, int64_t *__restrict__ tile_row0, int32_t *__restrict__ tile_seq,
                  int64_t *__restrict__ n_tiles, int64_t *__restrict__ kept_off, int64_t capacity, int32_t *err) {
    extern __shared__ int64_t s_toff[];   // [B + 1] first tile of each sequence
    __shared__ int64_t s_warp[32];
    __shared__ int64_t s_carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();   // the counts come from the preceding scan
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int b = 0; b <= B; ++b) {
            s_toff[b] = acc;
            if (b < B) {
                const int64_t len = seq_off[b + 1] - seq_off[b];
                acc += len > 0 ? (len + TR - 1) / TR : 0;
            }
        }
        s_carry = 0;
    }
    __syncthreads();
    const int64_t T = s_toff[B];
    for (int64_t t0 = 0; t0 < T; t0 += 1024) {
        const int64_t t = t0 + threadIdx.x;
        int64_t v = 0;
        if (t < T) {
            const int4 c4 = reinterpret_cast<const int4 *>(cnt)[t];
            v = int64_t(c4.x) + c4.y + c4.z + c4.w;
            int lo = 0, hi = B - 1;   // the sequence of tile t: the last b with s_toff[b] <= t
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_toff[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            tile_seq[t] = lo;
            tile_row0[t] = seq_off[lo] + (t - s_toff[lo]) * TR;
        }
        int64_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int64_t sw = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, sw, o);
                if (lane >= o) sw += y;
            }
            s_warp[lane] = sw;
        }
        __syncthreads();
        const int64_t carry = s_carry;
        if (t < T) tile_base[t] = carry + (warp ? s_warp[warp - 1] : 0) + x - v;
        __syncthreads();
        if (threadIdx.x == 0) s_carry = carry + s_warp[31];
        __syncthreads();
    }
    // the kept offset of sequence b: the base of its first tile (the total for a sequence without tiles after
    // the last one); the tile bases written above are visible to the whole block after the barrier
    const int64_t total = s_carry;
    for (int b = threadIdx.x; b <= B; b += blockDim.x) kept_off[b] = s_toff[b] < T ? tile_base[s_toff[b]] : total;
    if (threadIdx.x == 0) {
        *n_tiles = T;
        if (total > capacity) raise_err(err, LSA_ERR_CAPACITY);
    }
}

// One CTA of TR threads per scan tile (tiles past the count exit): thread i places row row0 + i if it is kept.
__global__ void select_tiles_scatter(const uint32_t *__restrict__ bits, const int64_t *__restrict__ tile_base,
                                     const int64_t *__restrict__ tile_row0, const int32_t *__restrict__ tile_seq,
                                     const int64_t *__restrict__ n_tiles, const int64_t *__restrict__ seq_off,
                                     int32_t *__restrict__ kept_idx, int64_t capacity) {
    __shared__ int s_wpre[8];
    pdl_wait();
    const int64_t t = blockIdx.x;
    if (t >= *n_tiles) return;
    const int wpt = int(blockDim.x) >> 5, i = int(threadIdx.x), wi = i >> 5, lane = i & 31;
    const uint32_t word = bits[t * wpt + wi];
    if (lane == 0) s_wpre[wi] = __popc(word);
    __syncthreads();
    int before = 0;
    for (int j = 0; j < wi; ++j) before += s_wpre[j];
    if ((word >> lane) & 1u) {
        const int b = tile_seq[t];
        const int64_t row = tile_row0[t] + i;   // kept rows lie inside the sequence (ballots are masked)
        const int64_t rank = tile_base[t] + before + __popc(word & ((1u << lane) - 1u));
        if (rank < capacity) kept_idx[rank] = int32_t(row - seq_off[b]);
    }
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

#define LSA_TRY_STATUS(call)         \
    do {                             \
        lsa_status s_ = (call);      \
        if (s_ != LSA_OK) return s_; \
    } while (0)

size_t select_tiles_workspace(int64_t n_total, int32_t B) {
    const int64_t tmax = (n_total + 127) / 128 + B + 1;   // scan tiles of >= 128 rows
    return align_up(size_t(tmax) * 8 * 4, 256) + align_up(size_t(tmax) * 4 * 4, 256) +   // bits, counts
           align_up(size_t(tmax + 1) * 8, 256) * 2 + align_up(size_t(tmax) * 4, 256) + 256;
}

size_t index_score_select_workspace(int64_t n_total, int32_t B) {
    const size_t a = lsa_select_workspace_size(n_total), b = select_tiles_workspace(n_total, B);
    return a > b ? a : b;
}

lsa_status launch_index_score_select(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                                     lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                                     int64_t n_total, int32_t B, int32_t H, int32_t d, float *z, int32_t *kept_idx,
                                     int64_t capacity, int64_t *kept_off, void *workspace, int32_t *err,
                                     cudaStream_t st) {
    if (!(aligned16(q) && index_score_tc_supported(q_dtype, k_dtype, n_total, B, H, d))) {
        // no tensor-core scan for this shape: the CUDA-core scan, then the standalone selection
        LSA_TRY_STATUS(launch_index_score(q, q_dtype, w, k, k_dtype, k_scale, seq_off, n_total, nullptr, nullptr, 0,
                                          B, H, d, z, nullptr, 0, err, st));
        return launch_select(z, seq_off, n_total, B, kept_idx, capacity, kept_off, nullptr, workspace, err, st);
    }
    const int TR = index_score_tc_tile_rows(k_dtype);
    const int64_t tmax = (n_total + 127) / 128 + B + 1;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *bits = reinterpret_cast<uint32_t *>(ws);
    ws += align_up(size_t(tmax) * 8 * 4, 256);
    int32_t *cnt = reinterpret_cast<int32_t *>(ws);
    ws += align_up(size_t(tmax) * 4 * 4, 256);
    int64_t *tile_base = reinterpret_cast<int64_t *>(ws);
    ws += align_up(size_t(tmax + 1) * 8, 256);
    int64_t *tile_row0 = reinterpret_cast<int64_t *>(ws);
    ws += align_up(size_t(tmax + 1) * 8, 256);
    int32_t *tile_seq = reinterpret_cast<int32_t *>(ws);
    ws += align_up(size_t(tmax) * 4, 256);
    int64_t *n_tiles = reinterpret_cast<int64_t *>(ws);
    LSA_TRY_STATUS(launch_index_score_tc_select(q, w, k, k_dtype, k_scale, seq_off, n_total, B, H, d, z, bits, cnt,
                                                err, st));
    LSA_CUDA(launch_pdl(select_tiles_scan, dim3(1), dim3(1024), size_t(B + 1) * 8, st, cnt, seq_off, B, TR,
                        tile_base, tile_row0, tile_seq, n_tiles, kept_off, capacity, err));
    LSA_LAUNCHED("select_tiles_scan");
    const int64_t tiles = (n_total + TR - 1) / TR + B;   // at least the scan's tile count
    LSA_CUDA(launch_pdl(select_tiles_scatter, dim3(unsigned(tiles)), dim3(TR), 0, st, bits, tile_base, tile_row0,
                        tile_seq, n_tiles, seq_off, kept_idx, capacity));
    LSA_LAUNCHED("select_tiles_scatter");
    return LSA_OK;
}

}  // namespace lsa
