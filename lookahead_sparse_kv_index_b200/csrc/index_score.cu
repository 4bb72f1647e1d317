// Lookahead index score ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse
// Attention", gist.science technical summary, section 2.1 "Scoring
// Mechanism"):  z_s = sum_j w_j ReLU(q_j . k_s),  I_s = sigmoid(z_s).
//
// This file holds the CUDA-core path: one thread per entry, the sequence's
// indexer queries staged in shared memory as fp32, per-head accumulators in
// registers.  It runs every supported shape and dtype (fp32 keys included)
// and the listed (gathered) variant used between refreshes.  Scans of bf16 /
// e4m3 keys of the shapes index_score_tc.cu supports, full or listed, go to the
// tensor-core kernel unless the caller asks for this path.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kTile = 256;  // entries per block (one per thread)

template <lsa_dtype KT>
struct KeyChunk;

template <>
struct KeyChunk<LSA_F32> {
    static constexpr int N = 4;
    __device__ static void load(const void *row, int c, float *out) {
        float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(row) + c);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
};

template <>
struct KeyChunk<LSA_BF16> {
    static constexpr int N = 8;
    __device__ static void load(const void *row, int c, float *out) {
        uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(row) + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            out[2 * t] = __uint_as_float(u[t] << 16);
            out[2 * t + 1] = __uint_as_float(u[t] & 0xFFFF0000u);
        }
    }
};

template <>
struct KeyChunk<LSA_E4M3> {
    static constexpr int N = 16;
    __device__ static void load(const void *row, int c, float *out) {
        uint4 v = *reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(row) + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>((u[t] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
                float2 f = __half22float2(*reinterpret_cast<__half2 *>(&hr));
                out[4 * t + 2 * h] = f.x;
                out[4 * t + 2 * h + 1] = f.y;
            }
        }
    }
};

// Finds the sequence and the entry range of this block's tile.  Tiles are
// laid out sequence after sequence, ceil(len / kTile) per sequence, over the
// CSR offsets `off` (the entry axis in full mode, the list axis in listed mode).
__device__ bool find_tile(const int64_t *off, int B, int64_t tile, int &b, int64_t &lo, int64_t &hi) {
    int64_t acc = 0;
    for (int s = 0; s < B; ++s) {
        int64_t len = off[s + 1] - off[s];
        int64_t nt = (len + kTile - 1) / kTile;
        if (tile < acc + nt) {
            b = s;
            lo = off[s] + (tile - acc) * kTile;
            hi = off[s + 1];
            return true;
        }
        acc += nt;
    }
    return false;
}

template <lsa_dtype KT, int HMAX>
__global__ void __launch_bounds__(kTile)
score_cuda_core(const void *__restrict__ q, int q_is_bf16, const float *__restrict__ w,
                const void *__restrict__ k, const float *__restrict__ k_scale,
                const int64_t *__restrict__ seq_off, const int32_t *__restrict__ idx,
                const int64_t *__restrict__ idx_off, int64_t n_cap, int B, int H, int d,
                float *__restrict__ z, float *__restrict__ I) {
    extern __shared__ float smem[];
    float *qs = smem;            // [H][d] fp32
    float *ws = smem + H * d;    // [H]
    __shared__ int s_b;
    __shared__ long long s_lo, s_hi;
    __shared__ int s_ok;

    const bool listed = idx != nullptr;
    if (threadIdx.x == 0) {
        int b = 0;
        int64_t lo = 0, hi = 0;
        s_ok = find_tile(listed ? idx_off : seq_off, B, blockIdx.x, b, lo, hi);
        s_b = b; s_lo = lo; s_hi = hi;
    }
    __syncthreads();
    if (!s_ok) return;
    const int b = s_b;

    for (int i = threadIdx.x; i < H * d; i += blockDim.x) {
        int64_t gi = int64_t(b) * H * d + i;
        qs[i] = q_is_bf16 ? bf16_to_f32(static_cast<const uint16_t *>(q)[gi])
                          : static_cast<const float *>(q)[gi];
    }
    for (int j = threadIdx.x; j < H; j += blockDim.x) ws[j] = w[int64_t(b) * H + j];
    __syncthreads();

    const int64_t p = s_lo + threadIdx.x;
    if (p >= s_hi || p >= n_cap) return;
    const int64_t e = listed ? seq_off[b] + idx[p] : p;

    const size_t esz = KT == LSA_F32 ? 4 : KT == LSA_BF16 ? 2 : 1;
    const void *row = static_cast<const uint8_t *>(k) + size_t(e) * d * esz;

    float acc[HMAX];
#pragma unroll
    for (int j = 0; j < HMAX; ++j) acc[j] = 0.f;

    constexpr int NC = KeyChunk<KT>::N;
    for (int c = 0; c < d; c += NC) {
        float kf[NC];
        KeyChunk<KT>::load(row, c, kf);
#pragma unroll
        for (int j = 0; j < HMAX; ++j) {
            if (j < H) {
                const float *qj = qs + j * d + c;
                float a = acc[j];
#pragma unroll
                for (int t = 0; t < NC; t += 4) {
                    float4 qv = *reinterpret_cast<const float4 *>(qj + t);
                    a = fmaf(qv.x, kf[t], a);
                    a = fmaf(qv.y, kf[t + 1], a);
                    a = fmaf(qv.z, kf[t + 2], a);
                    a = fmaf(qv.w, kf[t + 3], a);
                }
                acc[j] = a;
            }
        }
    }
    float zs = 0.f;
#pragma unroll
    for (int j = 0; j < HMAX; ++j)
        if (j < H) zs = fmaf(ws[j], fmaxf(acc[j], 0.f), zs);
    if (KT == LSA_E4M3) zs *= k_scale[e];   // scale > 0 and ReLU(a x) = a ReLU(x)
    z[p] = zs;
    if (I) I[p] = 1.f / (1.f + expf(-zs));
}

template <lsa_dtype KT>
lsa_status launch_kt(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                     const float *k_scale, const int64_t *seq_off, int64_t n_axis,
                     const int32_t *idx, const int64_t *idx_off, int B, int H, int d, float *z,
                     float *I, cudaStream_t st) {
    const int64_t grid = (n_axis + kTile - 1) / kTile + B;
    const size_t smem = size_t(H) * d * 4 + size_t(H) * 4;
    const int qb = q_dtype == LSA_BF16;
#define LSA_SCORE_LAUNCH(HM)                                                                    \
    do {                                                                                        \
        auto kern = score_cuda_core<KT, HM>;                                                    \
        if (smem > 48 * 1024) LSA_CUDA(ensure_smem(kern, smem));                                \
        kern<<<dim3(unsigned(grid)), kTile, smem, st>>>(q, qb, w, k, k_scale, seq_off, idx,     \
                                                         idx_off, n_axis, B, H, d, z, I);       \
    } while (0)
    if (H <= 8) LSA_SCORE_LAUNCH(8);
    else if (H <= 16) LSA_SCORE_LAUNCH(16);
    else if (H <= 32) LSA_SCORE_LAUNCH(32);
    else LSA_SCORE_LAUNCH(64);
#undef LSA_SCORE_LAUNCH
    LSA_LAUNCHED("score_cuda_core");
    return LSA_OK;
}

}  // namespace

lsa_status launch_index_score(const void *q, lsa_dtype q_dtype, const float *w, const void *k,
                              lsa_dtype k_dtype, const float *k_scale, const int64_t *seq_off,
                              int64_t n_total, const int32_t *idx, const int64_t *idx_off,
                              int64_t list_capacity, int32_t B, int32_t H, int32_t d, float *z,
                              float *I, int32_t flags, int32_t *err, cudaStream_t st) {
    const int64_t n_axis = idx ? list_capacity : n_total;
    // the tensor-core kernel reads query rows with 16-byte loads
    if (!(flags & LSA_SCORE_CUDA_CORE) && aligned16(q) && index_score_tc_supported(q_dtype, k_dtype, n_total, B, H, d))
        return launch_index_score_tc(q, w, k, k_dtype, k_scale, seq_off, n_total, idx, idx_off, list_capacity, B,
                                     H, d, z, I, err, st);
    switch (k_dtype) {
    case LSA_F32:
        return launch_kt<LSA_F32>(q, q_dtype, w, k, k_scale, seq_off, n_axis, idx, idx_off, B, H, d, z, I, st);
    case LSA_BF16:
        return launch_kt<LSA_BF16>(q, q_dtype, w, k, k_scale, seq_off, n_axis, idx, idx_off, B, H, d, z, I, st);
    default:
        return launch_kt<LSA_E4M3>(q, q_dtype, w, k, k_scale, seq_off, n_axis, idx, idx_off, B, H, d, z, I, st);
    }
}

}  // namespace lsa
