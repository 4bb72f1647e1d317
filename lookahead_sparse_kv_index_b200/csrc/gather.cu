// Cold-pool fetch ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse Attention",
// gist.science technical summary, section 2.1 "Dynamic Fetching"; blog page:
// critical chunks move from the "CPU Cold Pool" to "GPU HBM" just in time).
//
// Zero-copy gather: the kernel reads the kept rows straight out of page-locked
// host memory over the host link and writes them densely into the HBM hot
// buffer in kept order.  Each warp moves several rows at once with 16-byte
// loads, so many host-link reads are in flight per SM; the copy engine is not
// involved and no per-row API call is made.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kRowsPerWarp = 4;   // rows in flight per warp
constexpr int kVecPerLane = 2;    // 16-byte vectors per lane per row step

__global__ void __launch_bounds__(kGatherThreads)
gather_rows(const uint4 *__restrict__ cold, int64_t row_vec, const int64_t *__restrict__ seq_off,
            const int32_t *__restrict__ kept_idx, const int64_t *__restrict__ kept_off, int B,
            uint4 *__restrict__ hot, int64_t hot_cap, int32_t *__restrict__ slot_of,
            int32_t *err) {
    const int64_t total = kept_off[B];
    const int64_t n = total < hot_cap ? total : hot_cap;
    if (total > hot_cap && blockIdx.x == 0 && threadIdx.x == 0) raise_err(err, LSA_ERR_CAPACITY);
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * kGatherThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * kGatherThreads) >> 5;
    for (int64_t r0 = warp * kRowsPerWarp; r0 < n; r0 += nwarps * kRowsPerWarp) {
        const uint4 *src[kRowsPerWarp];
        uint4 *dst[kRowsPerWarp];
        bool ok[kRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kRowsPerWarp; ++j) {
            const int64_t r = r0 + j;
            ok[j] = r < n;
            src[j] = cold;
            dst[j] = hot;
            if (ok[j]) {
                const int b = seq_of(kept_off, B, r);
                const int64_t e = seq_off[b] + kept_idx[r];
                src[j] = cold + e * row_vec;
                dst[j] = hot + r * row_vec;
                if (lane == 0 && slot_of) slot_of[e] = int32_t(r);
            }
        }
        for (int64_t v0 = 0; v0 < row_vec; v0 += 32 * kVecPerLane) {
            uint4 buf[kRowsPerWarp][kVecPerLane];
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; ++j)
#pragma unroll
                for (int u = 0; u < kVecPerLane; ++u) {
                    const int64_t v = v0 + u * 32 + lane;
                    if (ok[j] && v < row_vec) buf[j][u] = src[j][v];
                }
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; ++j)
#pragma unroll
                for (int u = 0; u < kVecPerLane; ++u) {
                    const int64_t v = v0 + u * 32 + lane;
                    if (ok[j] && v < row_vec) dst[j][v] = buf[j][u];
                }
        }
    }
}

}  // namespace

lsa_status launch_gather(const void *cold_dev, int64_t row_bytes, const int64_t *seq_off,
                         int64_t n_total, const int32_t *kept_idx, const int64_t *kept_off,
                         int32_t B, void *hot, int64_t hot_capacity, int32_t *slot_of,
                         int32_t *err, cudaStream_t st) {
    if (slot_of && n_total > 0) LSA_CUDA(cudaMemsetAsync(slot_of, 0xFF, size_t(n_total) * 4, st));
    const int blocks = sm_count() * 8;
    gather_rows<<<blocks, kGatherThreads, 0, st>>>(static_cast<const uint4 *>(cold_dev), row_bytes / 16,
                                                   seq_off, kept_idx, kept_off, B,
                                                   static_cast<uint4 *>(hot), hot_capacity, slot_of, err);
    LSA_LAUNCHED("gather_rows");
    return LSA_OK;
}

}  // namespace lsa
