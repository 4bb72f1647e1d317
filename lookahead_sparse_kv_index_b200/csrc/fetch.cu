// Incremental cold-pool fetch ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse
// Attention", gist.science technical summary, section 2.1 "Dynamic Fetching":
// every entry with I >= 0.5 is brought from the CPU cold pool into GPU memory;
// blog page: critical chunks are fetched "just in time").
//
// The decode context keeps the HBM hot buffer as a cache of cold-pool rows:
//   slot_of[e]  hot slot holding entry e, or -1;
//   owner[s]    entry held by slot s, or -1   (slot_of and owner are inverse);
// so an entry that stays critical across refreshes is never fetched twice.
// At a refresh, for the new kept list:
//   1. fetch_mark:    a kept entry already resident keeps its slot (marked
//                     used); the others are listed as new;
//   2. fetch_free:    every unused slot is listed as free (it may still hold a
//                     row no longer kept: it stays valid until reused);
//   3. fetch_assign:  new item i takes free slot i, evicting that slot's owner;
//   4. fetch_rows:    only the new items' rows cross the host link, read
//                     zero-copy from page-locked memory by warps of the GPU.
// kept_slot[p] is the hot slot of kept position p; the top-k writes it for the
// chosen entries, so attention reads the right rows.  Lists are built with
// warp-aggregated atomics, so slot placement may differ between runs; nothing
// computed depends on it.  A kept list longer than the hot buffer raises
// LSA_ERR_CAPACITY and is truncated, like lsa_gather.
//
// Lookahead (the next window's kept set fetched while the current window's
// steps still attend the current set): the slots of a protected kept list
// (the current set's kept_slot) are marked used too, so the fetch never
// evicts a row the running steps read; entries left without a free slot
// raise LSA_ERR_CAPACITY.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;

// Appends `item` to list[*count] for every lane with `want`; one atomic per warp.
__device__ __forceinline__ void warp_append(bool want, int32_t item, int32_t *list, int32_t *count) {
    const unsigned mask = __ballot_sync(0xffffffffu, want);
    if (!mask) return;
    const int lane = threadIdx.x & 31;
    int base = 0;
    if (lane == __ffs(mask) - 1) base = atomicAdd(count, __popc(mask));
    base = __shfl_sync(0xffffffffu, base, __ffs(mask) - 1);
    if (want) list[base + __popc(mask & ((1u << lane) - 1u))] = item;
}

// counts[0] = new items, counts[1] = free slots.
__global__ void __launch_bounds__(kThreads)
fetch_mark(const int64_t *__restrict__ seq_off, const int32_t *__restrict__ kept_idx,
           const int64_t *__restrict__ kept_off, int B, int64_t cap, const int32_t *__restrict__ slot_of,
           int32_t *__restrict__ kept_slot, uint8_t *__restrict__ used, int32_t *__restrict__ new_list,
           int32_t *__restrict__ counts, const int32_t *__restrict__ prot_slot, const int64_t *__restrict__ prot_off,
           int32_t *err) {
    const int64_t total = kept_off[B];
    const int64_t n = total < cap ? total : cap;
    if (total > cap && blockIdx.x == 0 && threadIdx.x == 0) raise_err(err, LSA_ERR_CAPACITY);
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    if (prot_slot) {   // slots the running steps still read
        const int64_t pt = prot_off[B] < cap ? prot_off[B] : cap;
        for (int64_t p = int64_t(blockIdx.x) * kThreads + threadIdx.x; p < pt; p += stride) {
            const int32_t s = prot_slot[p];
            if (s >= 0 && s < cap) used[s] = 1;
        }
    }
    for (int64_t p0 = int64_t(blockIdx.x) * kThreads; p0 < n; p0 += stride) {   // uniform per warp
        const int64_t p = p0 + threadIdx.x;
        bool is_new = false;
        if (p < n) {
            const int b = seq_of(kept_off, B, p);
            const int64_t e = seq_off[b] + kept_idx[p];
            const int32_t s = slot_of[e];
            kept_slot[p] = s;
            if (s >= 0) used[s] = 1;
            else is_new = true;
        }
        warp_append(is_new, int32_t(p), new_list, &counts[0]);
    }
}

__global__ void __launch_bounds__(kThreads)
fetch_free(int64_t cap, const uint8_t *__restrict__ used, int32_t *__restrict__ free_list,
           int32_t *__restrict__ counts) {
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t s0 = int64_t(blockIdx.x) * kThreads; s0 < cap; s0 += stride) {
        const int64_t s = s0 + threadIdx.x;
        warp_append(s < cap && !used[s], int32_t(s), free_list, &counts[1]);
    }
}

__global__ void __launch_bounds__(kThreads)
fetch_assign(const int64_t *__restrict__ seq_off, const int32_t *__restrict__ kept_idx,
             const int64_t *__restrict__ kept_off, int B, const int32_t *__restrict__ new_list,
             const int32_t *__restrict__ free_list, const int32_t *__restrict__ counts,
             int32_t *__restrict__ kept_slot, int32_t *__restrict__ slot_of, int32_t *__restrict__ owner,
             int64_t *__restrict__ fetched, int32_t *err) {
    // free >= new whenever the kept list (with the protected one) fits the hot buffer; the clamp keeps every
    // slot index in range, and an entry left without a slot is a capacity error
    const int n_new = min(counts[0], counts[1]);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *fetched = n_new;
        if (counts[0] > counts[1]) raise_err(err, LSA_ERR_CAPACITY);
    }
    for (int i = blockIdx.x * kThreads + threadIdx.x; i < n_new; i += gridDim.x * kThreads) {
        const int32_t p = new_list[i];
        const int32_t s = free_list[i];
        const int32_t old = owner[s];
        if (old >= 0) slot_of[old] = -1;   // evict: `old` is not kept (its slot was unused)
        const int b = seq_of(kept_off, B, p);
        const int64_t e = seq_off[b] + kept_idx[p];
        owner[s] = int32_t(e);
        slot_of[e] = s;
        kept_slot[p] = s;
    }
}

constexpr int kRowsPerWarp = 4;

// Copies the rows of the new items into their slots (zero-copy host reads).
__global__ void __launch_bounds__(kThreads)
fetch_rows(const uint4 *__restrict__ cold, int64_t row_vec, const int64_t *__restrict__ seq_off,
           const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int B,
           const int32_t *__restrict__ new_list, const int32_t *__restrict__ counts,
           const int32_t *__restrict__ kept_slot, uint4 *__restrict__ hot) {
    const int n_new = min(counts[0], counts[1]);
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * kThreads) >> 5;
    for (int64_t i0 = warp * kRowsPerWarp; i0 < n_new; i0 += nwarps * kRowsPerWarp) {
        const uint4 *src[kRowsPerWarp];
        uint4 *dst[kRowsPerWarp];
        bool ok[kRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kRowsPerWarp; ++j) {
            const int64_t i = i0 + j;
            ok[j] = i < n_new;
            src[j] = cold;
            dst[j] = hot;
            if (ok[j]) {
                const int32_t p = new_list[i];
                const int b = seq_of(kept_off, B, p);
                src[j] = cold + (seq_off[b] + kept_idx[p]) * row_vec;
                dst[j] = hot + int64_t(kept_slot[p]) * row_vec;
            }
        }
        for (int64_t v0 = 0; v0 < row_vec; v0 += 64) {
            uint4 buf[kRowsPerWarp][2];
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; ++j)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int64_t v = v0 + u * 32 + lane;
                    if (ok[j] && v < row_vec) buf[j][u] = src[j][v];
                }
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; ++j)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int64_t v = v0 + u * 32 + lane;
                    if (ok[j] && v < row_vec) dst[j][v] = buf[j][u];
                }
        }
    }
}

}  // namespace

// Scratch: used [cap] u8 | new_list [cap] i32 | free_list [cap] i32 | counts [2] i32.
size_t fetch_workspace(int64_t cap) {
    return align_up(size_t(cap), 256) + 2 * align_up(size_t(cap) * 4, 256) + 256;
}

lsa_status launch_fetch(const void *cold_dev, int64_t row_bytes, const int64_t *seq_off, const int32_t *kept_idx,
                        const int64_t *kept_off, int32_t B, void *hot, int64_t cap, int32_t *slot_of,
                        int32_t *owner, int32_t *kept_slot, int64_t *fetched, void *workspace, int32_t *err,
                        cudaEvent_t assigned, cudaStream_t st, const int32_t *prot_slot, const int64_t *prot_off,
                        int row_ctas) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *used = ws;
    int32_t *new_list = reinterpret_cast<int32_t *>(ws + align_up(size_t(cap), 256));
    int32_t *free_list = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(new_list) + align_up(size_t(cap) * 4, 256));
    int32_t *counts = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(free_list) + align_up(size_t(cap) * 4, 256));
    LSA_CUDA(cudaMemsetAsync(used, 0, size_t(cap), st));
    LSA_CUDA(cudaMemsetAsync(counts, 0, 8, st));
    const int blocks = sm_count() * 4;
    fetch_mark<<<blocks, kThreads, 0, st>>>(seq_off, kept_idx, kept_off, B, cap, slot_of, kept_slot, used, new_list,
                                            counts, prot_slot, prot_off, err);
    LSA_LAUNCHED("fetch_mark");
    fetch_free<<<blocks, kThreads, 0, st>>>(cap, used, free_list, counts);
    LSA_LAUNCHED("fetch_free");
    fetch_assign<<<blocks, kThreads, 0, st>>>(seq_off, kept_idx, kept_off, B, new_list, free_list, counts, kept_slot,
                                              slot_of, owner, fetched, err);
    LSA_LAUNCHED("fetch_assign");
    if (assigned) LSA_CUDA(cudaEventRecord(assigned, st));
    fetch_rows<<<row_ctas > 0 ? row_ctas : sm_count() * 8, kThreads, 0, st>>>(static_cast<const uint4 *>(cold_dev),
                                                                             row_bytes / 16, seq_off,
                                                    kept_idx, kept_off, B, new_list, counts, kept_slot,
                                                    static_cast<uint4 *>(hot));
    LSA_LAUNCHED("fetch_rows");
    return LSA_OK;
}

}  // namespace lsa
