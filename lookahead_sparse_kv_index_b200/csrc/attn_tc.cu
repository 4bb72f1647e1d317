// Tensor-core (tcgen05) split-K multi-query decode attention over the selected
// rows ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse Attention", gist.science
// technical summary, section 2.1 "Tiered Selection": the top-k inside the
// fetched subset feeds the final core attention).
//
// Shape run here: 128 query heads over one latent KV head of dim 512 (the same
// bf16 row serves as K and V).  One CTA per (sequence, chunk of 64 selected
// rows), ten warps; 2048 rows per sequence give 128 CTAs of short chains:
//   * warp 9 (loads): loads all of Q[b] (128 x 512 bf16, 8 slices of 64
//     columns, 128 KB resident) by TMA before the dependency on the preceding
//     kernel is resolved; reads the chunk's row indices;
//   * warps 0-7 first gather the chunk's rows (1 KB each, arbitrary hot-buffer
//     rows) with cp.async straight into the 128-byte-swizzled K-major layout
//     the tensor core reads, 8 column blocks of 64 elements, each signalled on
//     its own barrier as soon as it lands so that the S MMAs of block 0 start
//     while the others are in flight; padding rows are zero-filled.  (A TMA
//     row gather, tile::gather4, moved the same rows at about a third of this
//     rate: its instructions are serialised through the SM's one TMA unit.);
//   * warp 8 (MMA): S = Q K^T (M = 128 heads, N = 64 rows, K = 512) into TMEM
//     columns 0..63; then O = P V (M = 128, N = 2 x 256, K = 64) into TMEM
//     columns 0..511, reading the SAME shared rows as V through an MN-major
//     descriptor (no transpose, no second copy);
//   * warps 0-7 (then softmax, epilogue): warp w owns TMEM lanes 32 (w % 4) ..
//     (heads) and the 32 chunk rows 32 (w / 4) ..; S stays in registers from
//     the row max to the weights; the two warps of a head meet in shared
//     memory for its max and sum; P goes to shared memory as bf16 in the
//     K-major layout (one [128 heads x 64 rows] block over Q's first slice);
//     after O, each half converts 256 output columns to bf16 in 64-column
//     blocks staged in the freed Q buffer and writes them with TMA stores (a
//     lane per 1 KB partial row with plain stores was much slower); (m, l) per
//     head in fp32.
// The combine kernel (attn.cu) merges the chunks (merging them inside this
// kernel, with the CTAs of a sequence meeting on a counter, was slower: each CTA
// had to wait for its partial stores to complete and then read 128 KB of
// partials back).  Every wait is bounded.
#include <cuda.h>

#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace ptx;

constexpr int kHq = 128;
constexpr int kD = 512;
constexpr int kRowsPerCta = 64;
constexpr int kQSlices = 8;   // all of Q[b] resident: 8 x 16 KB; P and the O staging reuse it once S is done
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 32 * (kSoftWarps + 2);
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kTmemCols = 512;

constexpr int kKvBytes = kRowsPerCta * kD * 2;   // 64 KB: 8 blocks of [64 rows x 128 B]
constexpr int kKvBlock = kRowsPerCta * 128;      // 8 KB
constexpr int kQStageBytes = kHq * 128;          // 16 KB: one 64-column slice of Q
constexpr int kPBytes = kHq * kRowsPerCta * 2;   // 16 KB: one block of [128 heads x 128 B]
constexpr int kOStageBytes = kHq * 64 * 2;       // 16 KB: [128 heads][64 bf16] staging of one O block
static_assert((kD / 64) * kOStageBytes <= kQSlices * kQStageBytes, "every O block has its own staging buffer");
static_assert(kPBytes <= kQStageBytes, "P lives in Q's first slice");
static_assert(kRowsPerCta == 64, "the row mask, the gather and the softmax split assume 64 rows per CTA");

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on `bar` once every cp.async this thread has issued so far has landed (counted in the barrier's
// expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 2^x (the hardware approximation, as the fast exponential uses).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// 64-element (128-byte) blocks along MN `lbo` bytes apart, 8-row groups along
// K 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t(1024 >> 4) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap,
        const uint16_t *__restrict__ kv, int64_t stride, const int32_t *__restrict__ rows, int k, float scale,
        float *__restrict__ part_ml, int32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kvs = smem;                         // 64 KB
    uint8_t *qs = kvs + kKvBytes;                // kQSlices x 16 KB
    // P (16 KB) overwrites Q's first slice: it is written only after every S MMA has completed, and by
    // then every Q load has landed (each was waited for by an S MMA)
    uint8_t *ps = qs;
    uint64_t *qfull = reinterpret_cast<uint64_t *>(qs + kQSlices * kQStageBytes);
    uint64_t *kv_full = qfull + kQSlices;        // [kD / 64] column blocks of the rows
    uint64_t *s_full = kv_full + kD / 64;
    uint64_t *p_full = s_full + 1;
    uint64_t *o_full = p_full + 1;               // [2]: O columns 0..255 and 256..511 done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_full + 2);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    int *s_nvalid = abort_flag + 1;
    uint32_t *s_valid = reinterpret_cast<uint32_t *>(s_nvalid + 1);   // [2] bit j % 32 of word j / 32: row j selected
    float *s_max = reinterpret_cast<float *>(s_valid + 2);             // [128 heads][2 halves]
    float *s_sum = s_max + 2 * kHq;                                    // [128 heads][2 halves]
    // [64] the chunk's rows (-1: padding), written as int2: 8-byte aligned
    int *s_rows = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(s_sum + 2 * kHq) + 15) & ~uintptr_t(15));

    const int chunk = blockIdx.x, b = blockIdx.y, nchunks = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_v = abort_flag;
    const int64_t pbase = (int64_t(b) * nchunks + chunk) * kHq;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kQSlices; ++s) mbar_init(&qfull[s], 1);
        for (int kb = 0; kb < kD / 64; ++kb) mbar_init(&kv_full[kb], 32 * kSoftWarps);
        mbar_init(s_full, 1);
        mbar_init(p_full, kSoftWarps);
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    if (warp == kLoadWarp && lane == 0) {
        // Q does not depend on the preceding kernel: load all of it now
        prefetch_tmap(&qmap);
        for (int kd = 0; kd < kQSlices; ++kd) {
            mbar_arrive_expect_tx(&qfull[kd], kQStageBytes);
            tma_load_2d(qs + kd * kQStageBytes, &qmap, &qfull[kd], kd * 64, b * kHq);
        }
    }
    pdl_wait();   // the selected rows (and the hot buffer) come from preceding kernels
    if (warp == kLoadWarp) {
        // lane l owns chunk rows l and 32 + l: word w of the row mask is the ballot of rows 32w + lane
        int r[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = chunk * kRowsPerCta + 32 * j + lane;
            r[j] = i < k ? rows[int64_t(b) * k + i] : -1;
            if (r[j] < 0) r[j] = -1;   // any negative index is padding
        }
        const uint32_t w0 = __ballot_sync(0xffffffffu, r[0] >= 0), w1 = __ballot_sync(0xffffffffu, r[1] >= 0);
        if (lane == 0) {
            s_valid[0] = w0;
            s_valid[1] = w1;
            *s_nvalid = __popc(w0) + __popc(w1);
        }
        s_rows[lane] = r[0];
        s_rows[32 + lane] = r[1];
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool empty_chunk = *s_nvalid == 0;

    if (empty_chunk) {
        // nothing selected here: the combine skips a chunk with m = -inf
        if (threadIdx.x < kHq) {
            part_ml[(pbase + threadIdx.x) * 2] = -INFINITY;
            part_ml[(pbase + threadIdx.x) * 2 + 1] = 0.f;
        }
        if (warp == kLoadWarp && lane == 0)   // let the early Q loads land before the CTA exits
            for (int kd = 0; kd < kQSlices; ++kd) mbar_wait(&qfull[kd], 0, abort_v, kWaitLimitNs);
    } else if (warp < kSoftWarps) {
        // ---- the row gather: thread t copies 16-byte chunk t % 8 of each 128-byte piece of rows
        // t / 8 + 32 j (j < 2), column block by column block; a column block is signalled once every
        // thread's copies into it have landed (cp.async-tracked arrivals)
        {
            const int t = threadIdx.x, c = t & 7;
            const uint32_t kv_u32 = smem_u32(kvs);
            const uint16_t *src[2];
            uint32_t nbytes[2], dst[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int rr = (t >> 3) + 32 * j;
                const int row = s_rows[rr];
                src[j] = kv + (row >= 0 ? int64_t(row) * stride : 0) + c * 8;
                nbytes[j] = row >= 0 ? 16u : 0u;
                dst[j] = kv_u32 + rr * 128 + ((c ^ (rr & 7)) << 4);
            }
#pragma unroll
            for (int kb = 0; kb < kD / 64; ++kb) {
#pragma unroll
                for (int j = 0; j < 2; ++j) cp_async_16(dst[j] + kb * kKvBlock, src[j] + kb * 64, nbytes[j]);
                cp_async_arrive_noinc(&kv_full[kb]);
            }
        }
        // ---- softmax: thread (quarter, lane) owns head 32 * quarter + lane (its TMEM lane) and chunk rows
        // 32 * half .. 32 * half + 31 (TMEM columns)
        const int quarter = warp & 3, half = warp >> 2;
        const int head = 32 * quarter + lane;
        const uint32_t taddr = tmem + (uint32_t(quarter * 32) << 16);
        bool ok = mbar_wait(s_full, 0, abort_v, kWaitLimitNs);
        float m = -INFINITY, l = 0.f;
        // the softmax warps take every branch below together (they meet at named barriers)
        if (named_barrier_and(1, 32 * kSoftWarps, ok)) {
            tc_fence_after();
            uint32_t sv[32];
#pragma unroll
            for (int c = 0; c < 2; ++c)
                tmem_ld_32x32b_x16(taddr + half * 32 + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[c * 16]));
            tmem_ld_wait();
            const uint32_t v0 = s_valid[half];
            const bool all_valid = v0 == 0xffffffffu;
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const bool valid = all_valid || ((v0 >> u) & 1u);
                if (valid) mq[u & 3] = fmaxf(mq[u & 3], scale * __uint_as_float(sv[u]));
            }
            s_max[2 * head + half] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            named_barrier(1, 32 * kSoftWarps);
            m = fmaxf(s_max[2 * head], s_max[2 * head + 1]);   // a head with a valid row has m > -inf
            // exp(scale s - m) = 2^(scale log2(e) s - m log2(e)): one FFMA and one ex2 per weight
            const float c1 = scale * 1.4426950408889634f, c0 = -m * 1.4426950408889634f;
            // P in bf16, K-major swizzled: row `head`, 16-byte chunk 4 half + c (chunk rows 8 (4 half + c) ..)
            float lq[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t p_u32 = smem_u32(ps) + head * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t packed[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j0 = 8 * c + 2 * e, j1 = j0 + 1;
                    const bool ok0 = all_valid || ((v0 >> j0) & 1u);
                    const bool ok1 = all_valid || ((v0 >> j1) & 1u);
                    const float p0 = ok0 ? ex2_approx(fmaf(c1, __uint_as_float(sv[j0]), c0)) : 0.f;
                    const float p1 = ok1 ? ex2_approx(fmaf(c1, __uint_as_float(sv[j1]), c0)) : 0.f;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    // the normaliser sums the bf16-rounded weights the MMA actually uses
                    const float2 back = __bfloat1622float2(h2);
                    lq[e] += back.x + back.y;
                    packed[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                const uint32_t dst = p_u32 + (((4 * half + c) ^ (head & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[0]), "r"(packed[1]),
                             "r"(packed[2]), "r"(packed[3])
                             : "memory");
            }
            s_sum[2 * head + half] = (lq[0] + lq[1]) + (lq[2] + lq[3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            // ---- O: each half converts its 256 columns as soon as their MMAs are done, 64-column blocks
            // staged in the (now free) Q buffer, each in its own 16 KB buffer, one TMA store per block
            ok = mbar_wait(&o_full[half], 0, abort_v, kWaitLimitNs);
            // the block loop below synchronises the 128 threads of this half: agree on one outcome first
            if (named_barrier_and(2 + half, 128, ok)) {
                tc_fence_after();
                l = s_sum[2 * head] + s_sum[2 * head + 1];
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    const int cb = 4 * half + c;                   // output column block
                    uint8_t *sb = qs + cb * kOStageBytes;         // [128 rows x 128 B]
                    uint32_t o[64];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        tmem_ld_32x32b_x16(taddr + cb * 64 + q4 * 16, *reinterpret_cast<uint32_t(*)[16]>(&o[q4 * 16]));
                    tmem_ld_wait();
                    // [128 rows x 64 bf16] in the 128-byte-swizzled layout (16-byte chunk u of row t at
                    // chunk u ^ (t % 8)): conflict-free writes
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[8 * u + 2 * e]),
                                                                            __uint_as_float(o[8 * u + 2 * e + 1]));
                            w4[e] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                        const uint32_t dst = smem_u32(sb) + head * 128 + ((u ^ (head & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w4[0]), "r"(w4[1]),
                                     "r"(w4[2]), "r"(w4[3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    named_barrier(2 + half, 128);   // the four warps of this half
                    if (quarter == 0 && lane == 0) {
                        tma_store_2d(&omap, sb, cb * 64, int(pbase));
                        bulk_commit();
                    }
                }
                // the staging buffers must outlive the stores' reads of them; the partials are visible to
                // the combine once this grid has completed
                if (quarter == 0 && lane == 0) bulk_wait_read<0>();
                if (half == 0) {
                    part_ml[(pbase + head) * 2] = m;
                    part_ml[(pbase + head) * 2 + 1] = l;
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(128, kRowsPerCta);
            constexpr uint32_t IDESC_O = idesc_bf16(128, 256) | (1u << 16);   // B (V) is MN-major
            const uint32_t kv_u32 = smem_u32(kvs);
            bool ok = true;
            for (int kd = 0; kd < kD / 64 && ok; ++kd) {
                ok = mbar_wait(&kv_full[kd], 0, abort_v, kWaitLimitNs) &&
                     mbar_wait(&qfull[kd], 0, abort_v, kWaitLimitNs);
                if (!ok) break;
                tc_fence_after();
                const uint32_t q_u32 = smem_u32(qs + kd * kQStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tmem, desc_sw128(q_u32 + kk * 32), desc_sw128(kv_u32 + kd * kKvBlock + kk * 32), IDESC_S,
                            (kd | kk) != 0);
            }
            if (ok) {
                mma_commit(s_full);
                if (mbar_wait(p_full, 0, abort_v, kWaitLimitNs)) {
                    tc_fence_after();
                    const uint32_t p_u32 = smem_u32(ps);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int kk = 0; kk < kRowsPerCta / 16; ++kk)
                            mma_f16(tmem + half * 256, desc_sw128(p_u32 + kk * 32),
                                    desc_sw128_mn(kv_u32 + half * 4 * kKvBlock + kk * 2048, kKvBlock), IDESC_O,
                                    kk != 0);
                        mma_commit(&o_full[half]);   // this half's epilogue may start
                    }
                }
            }
            if (!ok) {
                // let the row gathers land before the CTA exits
                for (int kb = 0; kb < kD / 64; ++kb) {
                    volatile int no_abort = 0;
                    mbar_wait(&kv_full[kb], 0, &no_abort, kWaitLimitNs);
                }
            }
        }
    }
    // (the load warp issued every Q slice before the dependency wait; each is waited for by an S MMA, or
    // above when the chunk is empty)
    __syncwarp();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_v) raise_err(err, LSA_ERR_TIMEOUT);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

constexpr size_t kSmemBytes = 1024 + size_t(kKvBytes) + size_t(kQSlices) * kQStageBytes +
                              (kQSlices + kD / 64 + 4) * 8 + 16 + 16 + 4 * kHq * 4 + 16 + kRowsPerCta * 4 + 64;

}  // namespace

bool sparse_attn_tc_supported(lsa_dtype dtype, int64_t k_off, int64_t v_off, int32_t Hq, int32_t D) {
    return dtype == LSA_BF16 && k_off == v_off && Hq == kHq && D == kD;
}

int sparse_attn_tc_chunk() { return kRowsPerCta; }

lsa_status launch_sparse_attn_tc(const void *Q, const void *kv, int64_t stride, int64_t k_off,
                                 const int32_t *rows, int32_t B, int32_t k, float scale, void *part_o,
                                 float *part_ml, int32_t *err, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        set_error("lsa_sparse_attn: cuTensorMapEncodeTiled is unavailable");
        return LSA_ERR_CUDA;
    }
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap qmap;
    const cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(B) * kHq};
    const cuuint64_t strides[1] = {cuuint64_t(kD) * 2};
    const cuuint32_t box[2] = {64, 128};
    CUresult r = enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(Q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("lsa_sparse_attn: cuTensorMapEncodeTiled failed (%d)", int(r));
        return LSA_ERR_CUDA;
    }
    CUtensorMap omap;   // partial O [B * nchunks * 128 rows, 512] bf16, stored in swizzled [128 x 64] boxes
    const int nchunks = (k + kRowsPerCta - 1) / kRowsPerCta;
    const cuuint64_t odims[2] = {cuuint64_t(kD), cuuint64_t(B) * nchunks * kHq};
    const cuuint64_t ostrides[1] = {cuuint64_t(kD) * 2};
    const cuuint32_t obox[2] = {64, 128};
    r = enc(&omap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, part_o, odims, ostrides, obox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("lsa_sparse_attn: cuTensorMapEncodeTiled (partials) failed (%d)", int(r));
        return LSA_ERR_CUDA;
    }
    LSA_CUDA(ensure_smem(attn_tc, size_t(int(kSmemBytes))));
    LSA_CUDA(launch_pdl(attn_tc, dim3(nchunks, B), dim3(kThreads), kSmemBytes, st, qmap, omap,
                        static_cast<const uint16_t *>(kv) + k_off, stride, rows, k, scale, part_ml, err));
    LSA_LAUNCHED("attn_tc");
    return LSA_OK;
}

}  // namespace lsa
