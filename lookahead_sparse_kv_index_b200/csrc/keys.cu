// Compacted copy of the kept entries' indexer keys ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection": between refreshes every decode step re-ranks the kept
// set with its own indexer query).
//
// At a refresh the decode context copies the key row (and the e4m3 row scale)
// of every kept entry into kept-list order, once; each of the following decode
// steps then re-scores the kept set with the full tensor-core scan streaming
// this dense array by TMA (its z lands at the kept position), instead of
// gathering scattered rows every step.  One thread per 16-byte piece of a row.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
gather_keys(const uint4 *__restrict__ k, int64_t row_vec, const float *__restrict__ k_scale,
            const int64_t *__restrict__ seq_off, const int32_t *__restrict__ kept_idx,
            const int64_t *__restrict__ kept_off, int B, int64_t cap, uint4 *__restrict__ kc, float *__restrict__ sc) {
    const int64_t total = kept_off[B] < cap ? kept_off[B] : cap;
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < total * row_vec; i += stride) {
        const int64_t p = i / row_vec, c = i - p * row_vec;
        const int b = seq_of(kept_off, B, p);
        const int64_t e = seq_off[b] + kept_idx[p];
        kc[p * row_vec + c] = k[e * row_vec + c];
        if (sc && c == 0) sc[p] = k_scale[e];
    }
}

}  // namespace

lsa_status launch_gather_keys(const void *k, int64_t row_bytes, const float *k_scale, const int64_t *seq_off,
                              const int32_t *kept_idx, const int64_t *kept_off, int32_t B, int64_t cap, void *kc,
                              float *sc, cudaStream_t st) {
    gather_keys<<<sm_count() * 8, kThreads, 0, st>>>(static_cast<const uint4 *>(k), row_bytes / 16, k_scale, seq_off,
                                                     kept_idx, kept_off, B, cap, static_cast<uint4 *>(kc), sc);
    LSA_LAUNCHED("gather_keys");
    return LSA_OK;
}

}  // namespace lsa
