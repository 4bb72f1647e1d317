// Tensor-core (tcgen05) split-K multi-query decode attention over the selected
// rows ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse Attention", gist.science
// technical summary, section 2.1 "Tiered Selection": the top-k inside the
// fetched subset feeds the final core attention).
//
// Shape run here: 128 query heads over one latent KV head of dim 512 (the same
// bf16 row serves as K and V).  One CTA per (sequence, chunk of 128 selected
// rows):
//   1. warps 0-3 gather the chunk's 128 rows (1 KB each, arbitrary hot-buffer
//      rows) with cp.async straight into the 128-byte-swizzled K-major layout
//      the tensor core reads (8 column blocks of 64 elements), block by block,
//      each block signalled as soon as it lands so that the S MMAs of block 0
//      start while the others are still in flight; padding rows are
//      zero-filled;
//   2. warp 5 streams Q[b] (128 x 512 bf16) by TMA in 8 slices of 64 columns
//      through a 5-stage ring (P later reuses its memory);
//   3. warp 4 issues S = Q K^T (M = 128 heads, N = 128 rows, K = 512) into
//      TMEM columns 0..127;
//   4. warps 0-3 (one head per thread) read S, compute the chunk's row max m,
//      p = exp(scale*s - m), l = sum p, and write P as bf16 in the K-major
//      swizzled layout;
//   5. warp 4 issues O = P V (M = 128, N = 2 x 256, K = 128) into TMEM columns
//      0..511, reading the SAME smem rows as V through an MN-major descriptor
//      (no transpose, no second copy of the rows);
//   6. warps 0-3 read O in 64-column blocks into the freed row buffer
//      (128-byte swizzle, one staging buffer per block) and write the
//      partial in bf16 with TMA stores; (m, l) per head in fp32.
// The combine kernel (attn.cu) merges the chunks.  Every wait is bounded.
#include <cuda.h>

#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace ptx;

constexpr int kHq = 128;
constexpr int kD = 512;
constexpr int kRowsPerCta = 128;
constexpr int kQStages = 5;   // 5 x 16 KB of Q in flight; P reuses this ring once S is done
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kTmemCols = 512;

constexpr int kKvBytes = kRowsPerCta * kD * 2;   // 128 KB: 8 blocks of [128 rows x 128 B]
constexpr int kKvBlock = kRowsPerCta * 128;      // 16 KB
constexpr int kQStageBytes = kHq * 128;          // 16 KB: one 64-column slice of Q
constexpr int kPBytes = kHq * kRowsPerCta * 2;   // 32 KB: 2 blocks of [128 heads x 128 B]
constexpr int kOStageBytes = kHq * 64 * 2;       // 16 KB: [128 heads][64 bf16] staging of one O block
static_assert((kD / 64) * kOStageBytes <= kKvBytes, "every O block has its own staging buffer in the row buffer");

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
        const uint16_t *__restrict__ kv, int64_t stride, int64_t k_off, const int32_t *__restrict__ rows, int k,
        float scale, float *__restrict__ part_ml, int32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kvs = smem;                         // 128 KB
    uint8_t *qs = kvs + kKvBytes;                // kQStages x 16 KB
    // P (32 KB) overwrites the Q ring: it is written only after every S MMA has completed, and by then
    // every Q load has landed (each was waited for by an S MMA)
    uint8_t *ps = qs;
    static_assert(kQStages * kQStageBytes >= kPBytes, "P lives in the Q ring");
    uint64_t *qfull = reinterpret_cast<uint64_t *>(qs + kQStages * kQStageBytes);
    uint64_t *qempty = qfull + kQStages;
    uint64_t *kv_full = qempty + kQStages;       // [kD / 64] column blocks of the rows
    uint64_t *s_full = kv_full + kD / 64;
    uint64_t *p_full = s_full + 1;
    uint64_t *o_full = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_full + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    int *s_rows = abort_flag + 1;                // [128]
    int *s_nvalid = s_rows + kRowsPerCta;
    uint32_t *s_valid = reinterpret_cast<uint32_t *>(s_nvalid + 1);   // [4] bit j % 32 of word j / 32: row j selected

    const int chunk = blockIdx.x, b = blockIdx.y, nchunks = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_v = abort_flag;
    const int64_t pbase = (int64_t(b) * nchunks + chunk) * kHq;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *s_nvalid = 0;
        for (int s = 0; s < kQStages; ++s) { mbar_init(&qfull[s], 1); mbar_init(&qempty[s], 1); }
        for (int kb = 0; kb < kD / 64; ++kb) mbar_init(&kv_full[kb], 128);
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(o_full, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 5 && lane == 0) {
        // Q does not depend on the preceding kernel: start streaming it now
        prefetch_tmap(&qmap);
        for (int kd = 0; kd < kQStages; ++kd) {
            mbar_arrive_expect_tx(&qfull[kd], kQStageBytes);
            tma_load_2d(qs + kd * kQStageBytes, &qmap, &qfull[kd], kd * 64, b * kHq);
        }
    }
    pdl_wait();   // the selected rows (and the hot buffer) come from preceding kernels
    if (threadIdx.x < kRowsPerCta) {
        const int i = chunk * kRowsPerCta + threadIdx.x;
        const int r = i < k ? rows[int64_t(b) * k + i] : -1;
        s_rows[threadIdx.x] = r;
        if (r >= 0) atomicAdd(s_nvalid, 1);
        const uint32_t bal = __ballot_sync(0xffffffffu, r >= 0);   // threads 0..127: whole warps
        if ((threadIdx.x & 31) == 0) s_valid[threadIdx.x >> 5] = bal;
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
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
        if (warp == 5 && lane == 0)   // let the early Q loads land before the CTA exits
            for (int kd = 0; kd < kQStages; ++kd) mbar_wait(&qfull[kd], 0, abort_v, kWaitLimitNs);
    } else if (warp < 4) {
        const int t = threadIdx.x;   // 0..127
        // ---- 1. gather the chunk's rows: 8 column blocks of 128 rows x 8 sixteen-byte chunks, one
        // cp.async group per block (8 consecutive threads read one row's 128 contiguous bytes)
        const uint32_t kv_u32 = smem_u32(kvs);
#pragma unroll
        for (int kb = 0; kb < kD / 64; ++kb) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = t + 128 * u;
                const int r = i >> 3, c = kb * 8 + (i & 7);
                const int row = s_rows[r];
                const uint32_t dst = kv_u32 + kb * kKvBlock + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                const uint16_t *src = kv + (row >= 0 ? int64_t(row) * stride + k_off + c * 8 : 0);
                cp_async_16(dst, src, row >= 0 ? 16u : 0u);
            }
            cp_async_commit();
        }
        // block kb has landed once at most 7 - kb younger groups are pending
        cp_async_wait_group<7>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[0]);
        cp_async_wait_group<6>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[1]);
        cp_async_wait_group<5>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[2]);
        cp_async_wait_group<4>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[3]);
        cp_async_wait_group<3>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[4]);
        cp_async_wait_group<2>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[5]);
        cp_async_wait_group<1>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[6]);
        cp_async_wait_group<0>(); fence_proxy_async_smem(); mbar_arrive(&kv_full[7]);

        // ---- 4. softmax of the chunk: thread t owns head t (TMEM lane t)
        const int quarter = warp;   // warps 0-3 -> TMEM lanes 32*warp ..
        bool ok = mbar_wait(s_full, 0, abort_v, kWaitLimitNs);
        float m = -INFINITY, l = 0.f;
        // warps 0-3 take every branch below together (they meet at named barriers)
        if (named_barrier_and(1, 128, ok)) {
            tc_fence_after();
            const uint32_t taddr = tmem + (uint32_t(quarter * 32) << 16);
            // S is read from TMEM 32 columns at a time, in two passes (row max, then weights): rolled
            // loops keep this phase's code and registers small.  Selected rows come from a bit mask; a
            // full chunk (the common case) skips the tests.  Max and sum run as four chains.
            const bool all_valid = (s_valid[0] & s_valid[1] & s_valid[2] & s_valid[3]) == 0xffffffffu;
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
            for (int c = 0; c < kRowsPerCta / 32; ++c) {
                uint32_t r32[32];
                tmem_ld_32x32b_x16(taddr + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&r32[0]));
                tmem_ld_32x32b_x16(taddr + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r32[16]));
                tmem_ld_wait();
                const uint32_t vb = all_valid ? 0xffffffffu : s_valid[c];
#pragma unroll
                for (int u = 0; u < 32; ++u)
                    if ((vb >> u) & 1u) mq[u & 3] = fmaxf(mq[u & 3], scale * __uint_as_float(r32[u]));
            }
            m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            float lq[4] = {0.f, 0.f, 0.f, 0.f};
            // P in bf16, K-major swizzled: block (j / 64), row t, 16-byte chunk (j % 64) / 8
            const uint32_t p_u32 = smem_u32(ps);
#pragma unroll 1
            for (int c = 0; c < kRowsPerCta / 32; ++c) {
                uint32_t r32[32];
                tmem_ld_32x32b_x16(taddr + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&r32[0]));
                tmem_ld_32x32b_x16(taddr + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r32[16]));
                tmem_ld_wait();
                const uint32_t vb = all_valid ? 0xffffffffu : s_valid[c];
                uint32_t packed[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j0 = 2 * u, j1 = j0 + 1;
                    const float p0 = ((vb >> j0) & 1u) ? __expf(scale * __uint_as_float(r32[j0]) - m) : 0.f;
                    const float p1 = ((vb >> j1) & 1u) ? __expf(scale * __uint_as_float(r32[j1]) - m) : 0.f;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    // the normaliser sums the bf16-rounded weights the MMA actually uses
                    const float2 back = __bfloat1622float2(h2);
                    lq[u & 3] += back.x + back.y;
                    packed[u] = *reinterpret_cast<const uint32_t *>(&h2);
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int cc = 4 * c + h;   // 16-byte chunk of the row (8 weights)
                    const uint32_t dst = p_u32 + (cc >> 3) * (kHq * 128) + t * 128 + (((cc & 7) ^ (t & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[4 * h]),
                                 "r"(packed[4 * h + 1]), "r"(packed[4 * h + 2]), "r"(packed[4 * h + 3])
                                 : "memory");
                }
            }
            l = (lq[0] + lq[1]) + (lq[2] + lq[3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
            // ---- 6. read O and write the chunk's partial (bf16): 64-column blocks staged in the (now
            // free) row buffer, each in its own 16 KB buffer, one TMA store per block
            ok = mbar_wait(o_full, 0, abort_v, kWaitLimitNs);
            // the block loop below synchronises these 128 threads: agree on one outcome first
            if (named_barrier_and(1, 128, ok)) {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < kD / 64; ++c) {
                    uint8_t *sb = kvs + c * kOStageBytes;   // [128 rows x 128 B]
                    uint32_t o[64];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        tmem_ld_32x32b_x16(taddr + c * 64 + q4 * 16, *reinterpret_cast<uint32_t(*)[16]>(&o[q4 * 16]));
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
                        const uint32_t dst = smem_u32(sb) + t * 128 + ((u ^ (t & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w4[0]), "r"(w4[1]),
                                     "r"(w4[2]), "r"(w4[3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    named_barrier(1, 128);
                    if (t == 0) {
                        tma_store_2d(&omap, sb, c * 64, int(pbase));
                        bulk_commit();
                    }
                }
                if (t == 0) bulk_wait_all();
                part_ml[(pbase + t) * 2] = m;
                part_ml[(pbase + t) * 2 + 1] = l;
            }
        }
    } else if (warp == 4) {
        // ---- 3./5. MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(128, 128);
            constexpr uint32_t IDESC_O = idesc_bf16(128, 256) | (1u << 16);   // B (V) is MN-major
            bool issued = false;
            {
                const uint32_t kv_u32 = smem_u32(kvs);
                int st = 0;
                uint32_t ph = 0;
                bool ok = true;
                for (int kd = 0; kd < kD / 64 && ok; ++kd) {
                    ok = mbar_wait(&kv_full[kd], 0, abort_v, kWaitLimitNs) &&
                         mbar_wait(&qfull[st], ph, abort_v, kWaitLimitNs);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t q_u32 = smem_u32(qs + st * kQStageBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem, desc_sw128(q_u32 + kk * 32), desc_sw128(kv_u32 + kd * kKvBlock + kk * 32),
                                IDESC_S, (kd | kk) != 0);
                    issued = true;
                    mma_commit(&qempty[st]);
                    if (++st == kQStages) { st = 0; ph ^= 1; }
                }
                if (ok) {
                    mma_commit(s_full);
                    if (mbar_wait(p_full, 0, abort_v, kWaitLimitNs)) {
                        tc_fence_after();
                        const uint32_t p_u32 = smem_u32(ps);
#pragma unroll
                        for (int half = 0; half < 2; ++half)
#pragma unroll
                            for (int kk = 0; kk < kRowsPerCta / 16; ++kk)
                                mma_f16(tmem + half * 256,
                                        desc_sw128(p_u32 + (kk >> 2) * (kHq * 128) + (kk & 3) * 32),
                                        desc_sw128_mn(kv_u32 + half * 4 * kKvBlock + kk * 2048, kKvBlock),
                                        IDESC_O, kk != 0);
                        mma_commit(o_full);
                    }
                }
            }
            (void)issued;
        }
    } else {
        // ---- 2. Q producer (the first kQStages slices were issued before the dependency wait)
        if (lane == 0) {
            int st = 0;
            uint32_t ph = 1;
            for (int kd = kQStages; kd < kD / 64; ++kd) {
                if (!mbar_wait(&qempty[st], ph ^ 1, abort_v, kWaitLimitNs)) break;
                mbar_arrive_expect_tx(&qfull[st], kQStageBytes);
                tma_load_2d(qs + st * kQStageBytes, &qmap, &qfull[st], kd * 64, b * kHq);
                if (++st == kQStages) { st = 0; ph ^= 1; }
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 4) {
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

constexpr size_t kSmemBytes = 1024 + size_t(kKvBytes) + size_t(kQStages) * kQStageBytes +
                              (2 * kQStages + kD / 64 + 3) * 8 + 16 + (kRowsPerCta + 2) * 4 + 16 + 64;

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
    CUtensorMap qmap;
    const cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(B) * kHq};
    const cuuint64_t strides[1] = {cuuint64_t(kD) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(Q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("lsa_sparse_attn: cuTensorMapEncodeTiled failed (%d)", int(r));
        return LSA_ERR_CUDA;
    }
    CUtensorMap omap;   // partial O [B * nchunks * 128 rows, 512] bf16, stored in swizzled [128 x 64] boxes
    const int nchunks_o = (k + kRowsPerCta - 1) / kRowsPerCta;
    const cuuint64_t odims[2] = {cuuint64_t(kD), cuuint64_t(B) * nchunks_o * kHq};
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
    const int nchunks = (k + kRowsPerCta - 1) / kRowsPerCta;
    LSA_CUDA(launch_pdl(attn_tc, dim3(nchunks, B), dim3(kThreads), kSmemBytes, st, qmap, omap,
                        static_cast<const uint16_t *>(kv), stride, k_off, rows, k, scale, part_ml, err));
    LSA_LAUNCHED("attn_tc");
    return LSA_OK;
}

}  // namespace lsa
