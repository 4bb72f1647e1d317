// Core attention over the selected entries ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1
// "Tiered Selection": the top-k inside the fetched subset feeds the final core
// attention).  Multi-query decode: every query head of a sequence attends
// over the same selected K/V rows.
//
// Split-K over the selected rows: each block takes one sequence, one chunk of
// kChunk selected rows and a group of kHeads query heads, stages the chunk's
// K/V rows and the group's queries in shared memory, and writes a partial
// (row max m, exp-sum l, unnormalised output o) per head.  A combine kernel
// merges the chunks:  M = max m_c,  L = sum l_c e^{m_c - M},
// o = sum o_c e^{m_c - M} / L,  lse = M + log L.
//
// This file holds the CUDA-core partial kernel (fp32 FMA; every supported
// shape, both dtypes) and the combine kernel; the 128-head x 512 latent bf16
// shape runs its partials on the tensor cores (attn_tc.cu).
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kChunk = 64;          // selected rows per block
constexpr int kHeads = 16;          // query heads per block
constexpr int kAttnThreads = 256;   // 8 warps, 2 heads each
constexpr int kMaxColsPerLane = 16; // D <= 512

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int kPad = 1;   // row stride D+1 words: conflict-free row-wise reads
    __device__ static float get(const float *p, int i) { return p[i]; }
    __device__ static float2 get2(const float *p, int i) { return make_float2(p[i], p[i + 1]); }
    __device__ static void put(float *p, int64_t i, float v) { p[i] = v; }
};
template <>
struct Elem<uint16_t> {
    static constexpr int kPad = 2;   // row stride D+2 halves = odd number of words
    __device__ static float get(const uint16_t *p, int i) { return bf16_to_f32(p[i]); }
    __device__ static float2 get2(const uint16_t *p, int i) {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p + i);
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    __device__ static void put(uint16_t *p, int64_t i, float v) {
        __nv_bfloat16 h = __float2bfloat16_rn(v);
        p[i] = *reinterpret_cast<uint16_t *>(&h);
    }
};

template <typename T>
__global__ void __launch_bounds__(kAttnThreads)
attn_partial(const T *__restrict__ Q, const T *__restrict__ kv, int64_t stride, int64_t k_off,
             int64_t v_off, const int32_t *__restrict__ rows, int Hq, int D, int k, float scale,
             float *__restrict__ part_o, float *__restrict__ part_ml) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int ld = D + Elem<T>::kPad;
    const bool alias = k_off == v_off;
    T *Ks = reinterpret_cast<T *>(smem_raw);
    T *Vs = alias ? Ks : Ks + kChunk * ld;
    float *Qs = reinterpret_cast<float *>(
        smem_raw + align_up(size_t(kChunk) * ld * sizeof(T) * (alias ? 1 : 2), 16));
    float *Ps = Qs + kHeads * D;
    __shared__ int s_rows[kChunk];

    const int chunk = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int nchunks = gridDim.x;
    const int h0 = hg * kHeads;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    if (threadIdx.x < kChunk) {
        const int i = chunk * kChunk + threadIdx.x;
        s_rows[threadIdx.x] = i < k ? rows[int64_t(b) * k + i] : -1;
    }
    __syncthreads();
    // stage K (and V) rows: element-wise copy, zero for padding rows
    for (int t = threadIdx.x; t < kChunk * D; t += kAttnThreads) {
        const int i = t / D, c = t - i * D;
        const int r = s_rows[i];
        T kvv{}, vvv{};
        if (r >= 0) {
            kvv = kv[int64_t(r) * stride + k_off + c];
            if (!alias) vvv = kv[int64_t(r) * stride + v_off + c];
        }
        Ks[i * ld + c] = kvv;
        if (!alias) Vs[i * ld + c] = vvv;
    }
    for (int t = threadIdx.x; t < kHeads * D; t += kAttnThreads) {
        const int hh = t / D, c = t - hh * D;
        const int h = h0 + hh;
        Qs[t] = h < Hq ? Elem<T>::get(Q, int((int64_t(b) * Hq + h) * D + c)) : 0.f;
    }
    __syncthreads();

    const int ncols = D / 32;
    for (int hh = warp; hh < kHeads; hh += kAttnThreads / 32) {
        const int h = h0 + hh;
        if (h >= Hq) break;
        const float *qh = Qs + hh * D;
        // logits for rows lane and lane + 32
        float s0 = 0.f, s1 = 0.f;
        for (int c = 0; c < D; c += 2) {
            const float2 q2 = make_float2(qh[c], qh[c + 1]);
            const float2 ka = Elem<T>::get2(Ks + lane * ld, c);
            const float2 kb = Elem<T>::get2(Ks + (lane + 32) * ld, c);
            s0 = fmaf(q2.x, ka.x, fmaf(q2.y, ka.y, s0));
            s1 = fmaf(q2.x, kb.x, fmaf(q2.y, kb.y, s1));
        }
        const bool v0 = s_rows[lane] >= 0, v1 = s_rows[lane + 32] >= 0;
        s0 = v0 ? s0 * scale : -INFINITY;
        s1 = v1 ? s1 * scale : -INFINITY;
        float m = fmaxf(s0, s1);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float p0 = v0 ? expf(s0 - m) : 0.f;
        const float p1 = v1 ? expf(s1 - m) : 0.f;
        float l = p0 + p1;
#pragma unroll
        for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        float *ph = Ps + hh * kChunk;
        ph[lane] = p0;
        ph[lane + 32] = p1;
        __syncwarp();
        float acc[kMaxColsPerLane];
#pragma unroll
        for (int j = 0; j < kMaxColsPerLane; ++j) acc[j] = 0.f;
        if (m != -INFINITY) {
            for (int i = 0; i < kChunk; ++i) {
                const float p = ph[i];
                const T *vr = Vs + i * ld;
#pragma unroll
                for (int j = 0; j < kMaxColsPerLane; ++j)
                    if (j < ncols) acc[j] = fmaf(p, Elem<T>::get(vr, lane + 32 * j), acc[j]);
            }
        }
        const int64_t pi = (int64_t(b) * nchunks + chunk) * Hq + h;
        float *dst = part_o + pi * D;
#pragma unroll
        for (int j = 0; j < kMaxColsPerLane; ++j)
            if (j < ncols) dst[lane + 32 * j] = acc[j];
        if (lane == 0) {
            part_ml[pi * 2] = m;
            part_ml[pi * 2 + 1] = l;
        }
        __syncwarp();
    }
}

// Raw partial values, converted where they are used (bf16 partials stay packed: two registers per
// chunk in flight instead of four).
template <typename TP>
struct Raw4;
template <>
struct Raw4<float> {
    using type = float4;
    __device__ static type load(const float *p, int64_t i) { return *reinterpret_cast<const float4 *>(p + i); }
    __device__ static float4 f(const type &v) { return v; }
    __device__ static type zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <>
struct Raw4<uint16_t> {
    using type = uint2;
    __device__ static type load(const uint16_t *p, int64_t i) { return *reinterpret_cast<const uint2 *>(p + i); }
    __device__ static float4 f(const type &w) {
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                           __uint_as_float(w.y & 0xFFFF0000u));
    }
    __device__ static type zero() { return make_uint2(0u, 0u); }
};

template <typename T>
__device__ __forceinline__ void put4(T *out, int64_t i, float4 a, float inv) {
    Elem<T>::put(out, i, a.x * inv);
    Elem<T>::put(out, i + 1, a.y * inv);
    Elem<T>::put(out, i + 2, a.z * inv);
    Elem<T>::put(out, i + 3, a.w * inv);
}

// Merge of the chunk partials of one (head, sequence):
//   M = max_c m_c,  w_c = e^{m_c - M},  L = sum_c l_c w_c,  o = sum_c w_c o_c / L,
//   lse = M + log L;  a chunk with m_c = -inf (no selected row) has weight 0 and
// its o is never read into the sum.
// The kernel is a chain of dependent L2 round trips unless the loads go out
// together.  Up to kMax (16) chunks: every thread issues its four columns
// of every chunk at once; meanwhile warp 0 turns the chunks' (m, l), the same
// for the whole block, into the weights w_c and 1 / L in shared memory.
template <typename T, typename TP, int kMax>
__global__ void __launch_bounds__(128, 4)   // 4 CTAs per SM: the whole grid (Hq x B) resident at once
attn_combine_few(const TP *__restrict__ part_o, const float *__restrict__ part_ml, int nchunks, int Hq, int D,
                 T *__restrict__ out, float *__restrict__ lse) {
    static_assert(kMax <= 32, "warp 0 holds one chunk per lane");
    using PR = Raw4<TP>;
    __shared__ float s_w[kMax];
    __shared__ float s_inv;
    pdl_wait();   // partials come from the preceding kernel
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t p0 = int64_t(b) * nchunks * Hq + h;   // partial index of chunk 0; chunk c adds c * Hq
    const int64_t ob = (int64_t(b) * Hq + h) * D;
    const int64_t cstride = int64_t(Hq) * D;
    for (int col0 = 0; col0 < D; col0 += 4 * int(blockDim.x)) {   // uniform trip count: barrier inside
        const int col = col0 + 4 * int(threadIdx.x);
        const bool act = col < D;
        typename PR::type v[kMax];
        const TP *base = part_o + p0 * D + col;
#pragma unroll
        for (int u = 0; u < kMax; ++u) v[u] = (act && u < nchunks) ? PR::load(base, int64_t(u) * cstride) : PR::zero();
        if (col0 == 0 && threadIdx.x < 32) {
            const int c = int(threadIdx.x);
            const float2 x = c < kMax && c < nchunks ? reinterpret_cast<const float2 *>(part_ml)[p0 + int64_t(c) * Hq]
                                                     : make_float2(-INFINITY, 0.f);
            float M = x.x;
#pragma unroll
            for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            // an empty chunk (m = -inf, or past nchunks) has weight 0 and its o is never read into the sum
            const float w = x.x == -INFINITY ? 0.f : expf(x.x - M);
            float L = x.y * w;
#pragma unroll
            for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            if (c < kMax) s_w[c] = w;
            if (c == 0) {
                s_inv = M == -INFINITY ? 0.f : 1.f / L;
                if (lse) lse[int64_t(b) * Hq + h] = M == -INFINITY ? -INFINITY : M + logf(L);
            }
        }
        __syncthreads();
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kMax; ++u) {
            const float w = s_w[u];
            if (w == 0.f) continue;   // empty chunk (or u >= nchunks), or a weight below the float range
            const float4 o = PR::f(v[u]);
            a.x = fmaf(w, o.x, a.x); a.y = fmaf(w, o.y, a.y);
            a.z = fmaf(w, o.z, a.z); a.w = fmaf(w, o.w, a.w);
        }
        if (act) put4(out, ob + col, a, s_inv);
    }
}

// 17..32 chunks of bf16 partials at the tensor-core shape (Hq x D fixed): the
// same scheme with two columns per thread and 256 threads, so that the 32
// chunks' values in flight fit in 64 registers (four CTAs per SM keep the whole
// grid resident; at four columns per thread the values spilled and the spill
// serialised the loads).  The chunk stride is a compile-time constant, so every
// load addresses off one base register.
template <typename T, int kHqC, int kDC>
__global__ void __launch_bounds__(256, 4)
attn_combine32(const uint16_t *__restrict__ part_o, const float *__restrict__ part_ml, int nchunks,
               T *__restrict__ out, float *__restrict__ lse) {
    constexpr int kMax = 32, Hq = kHqC, D = kDC;
    __shared__ float s_w[kMax];
    __shared__ float s_inv;
    pdl_wait();   // partials come from the preceding kernel
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t p0 = int64_t(b) * nchunks * Hq + h;   // partial index of chunk 0; chunk c adds c * Hq
    const int64_t ob = (int64_t(b) * Hq + h) * D;
    constexpr int64_t cstride = int64_t(Hq) * D;
    for (int col0 = 0; col0 < D; col0 += 2 * int(blockDim.x)) {   // uniform trip count: barrier inside
        const int col = col0 + 2 * int(threadIdx.x);
        const bool act = col < D;
        uint32_t v[kMax];
        const uint16_t *base = part_o + p0 * D + col;
#pragma unroll
        for (int u = 0; u < kMax; ++u)
            v[u] = (act && u < nchunks) ? *reinterpret_cast<const uint32_t *>(base + u * cstride) : 0u;
        if (col0 == 0 && threadIdx.x < 32) {
            const int c = int(threadIdx.x);
            const float2 x = c < nchunks ? reinterpret_cast<const float2 *>(part_ml)[p0 + int64_t(c) * Hq]
                                         : make_float2(-INFINITY, 0.f);
            float M = x.x;
#pragma unroll
            for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            // an empty chunk (m = -inf, or past nchunks) has weight 0 and its o is never read into the sum
            const float w = x.x == -INFINITY ? 0.f : expf(x.x - M);
            float L = x.y * w;
#pragma unroll
            for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            s_w[c] = w;
            if (c == 0) {
                s_inv = M == -INFINITY ? 0.f : 1.f / L;
                if (lse) lse[int64_t(b) * Hq + h] = M == -INFINITY ? -INFINITY : M + logf(L);
            }
        }
        __syncthreads();
        float ax = 0.f, ay = 0.f;
#pragma unroll
        for (int u = 0; u < kMax; ++u) {
            const float w = s_w[u];
            if (w == 0.f) continue;   // empty chunk (or u >= nchunks), or a weight below the float range
            ax = fmaf(w, __uint_as_float(v[u] << 16), ax);
            ay = fmaf(w, __uint_as_float(v[u] & 0xFFFF0000u), ay);
        }
        if (act) {
            Elem<T>::put(out, ob + col, ax * s_inv);
            Elem<T>::put(out, ob + col + 1, ay * s_inv);
        }
    }
}

// Any number of chunks: (m, l) in batches, then the columns in batches of 16 chunks.
template <typename T, typename TP>
__global__ void __launch_bounds__(128)
attn_combine(const TP *__restrict__ part_o, const float *__restrict__ part_ml, int nchunks, int Hq, int D,
             T *__restrict__ out, float *__restrict__ lse) {
    constexpr int kBatch = 16;
    using PR = Raw4<TP>;
    pdl_wait();   // partials come from the preceding kernel
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t p0 = int64_t(b) * nchunks * Hq + h;
    const float2 *ml = reinterpret_cast<const float2 *>(part_ml);
    const int64_t ob = (int64_t(b) * Hq + h) * D;
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, ml[p0 + int64_t(c) * Hq].x);
    float L = 0.f;
    if (M != -INFINITY)
        for (int c = 0; c < nchunks; ++c) {
            const float2 x = ml[p0 + int64_t(c) * Hq];
            if (x.x != -INFINITY) L += x.y * expf(x.x - M);
        }
    const float inv = M == -INFINITY ? 0.f : 1.f / L;
    for (int col = 4 * int(threadIdx.x); col < D; col += 4 * blockDim.x) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY)
            for (int c0 = 0; c0 < nchunks; c0 += kBatch) {
                typename PR::type v[kBatch];
                float mv[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int c = c0 + u;
                    mv[u] = c < nchunks ? ml[p0 + int64_t(c) * Hq].x : -INFINITY;
                    v[u] = c < nchunks ? PR::load(part_o, (p0 + int64_t(c) * Hq) * D + col) : PR::zero();
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    if (mv[u] == -INFINITY) continue;   // an empty chunk's o is never read into the sum
                    const float w = expf(mv[u] - M);
                    const float4 o = PR::f(v[u]);
                    a.x = fmaf(w, o.x, a.x); a.y = fmaf(w, o.y, a.y);
                    a.z = fmaf(w, o.z, a.z); a.w = fmaf(w, o.w, a.w);
                }
            }
        put4(out, ob + col, a, inv);
    }
    if (threadIdx.x == 0 && lse) lse[int64_t(b) * Hq + h] = M == -INFINITY ? -INFINITY : M + logf(L);
}

template <typename T, typename TP>
lsa_status launch_combine(const TP *part_o, const float *part_ml, int nchunks, int B, int Hq, int D, void *out,
                          float *lse, cudaStream_t st) {
    if constexpr (sizeof(TP) == 2) {
        if (nchunks > 16 && nchunks <= 32 && Hq == 128 && D == 512) {   // two columns per thread
            LSA_CUDA(launch_pdl(attn_combine32<T, 128, 512>, dim3(Hq, B), dim3(256), 0, st, part_o, part_ml, nchunks,
                                static_cast<T *>(out), lse));
            LSA_LAUNCHED("attn_combine32");
            return LSA_OK;
        }
    }
    auto kern = nchunks <= 16 ? attn_combine_few<T, TP, 16> : attn_combine<T, TP>;
    LSA_CUDA(launch_pdl(kern, dim3(Hq, B), dim3(128), 0, st, part_o, part_ml, nchunks, Hq, D, static_cast<T *>(out),
                        lse));
    LSA_LAUNCHED("attn_combine");
    return LSA_OK;
}

// Partial workspace: o [B, nchunks, Hq, D] fp32 (bf16 from the tensor-core chunks, which use the
// first half), then (m, l) [B, nchunks, Hq, 2] fp32.
struct Parts {
    float *o, *ml;
};
Parts parts(void *workspace, int B, int Hq, int D, int nchunks) {
    float *o = static_cast<float *>(workspace);
    return {o, o + align_up(size_t(B) * nchunks * Hq * D, 64)};
}

template <typename T>
lsa_status launch_t(const void *Q, const void *kv, int64_t stride, int64_t k_off, int64_t v_off,
                    const int32_t *rows, int B, int Hq, int D, int k, float scale, void *out, float *lse,
                    void *workspace, int32_t *err, cudaStream_t st) {
    int nchunks;
    Parts pp;
    if (sparse_attn_tc_supported(sizeof(T) == 2 ? LSA_BF16 : LSA_F32, k_off, v_off, Hq, D)) {
        // tensor-core chunks write bf16 partials (the fp32 workspace has room for them)
        nchunks = (k + sparse_attn_tc_chunk() - 1) / sparse_attn_tc_chunk();
        pp = parts(workspace, B, Hq, D, nchunks);
        lsa_status s = launch_sparse_attn_tc(Q, kv, stride, k_off, rows, B, k, scale, pp.o, pp.ml, err, st);
        if (s != LSA_OK) return s;
        return launch_combine<T, uint16_t>(reinterpret_cast<const uint16_t *>(pp.o), pp.ml, nchunks, B, Hq, D, out,
                                           lse, st);
    } else {
        nchunks = (k + kChunk - 1) / kChunk;
        pp = parts(workspace, B, Hq, D, nchunks);
        const int ld = D + Elem<T>::kPad;
        const bool alias = k_off == v_off;
        const size_t smem = align_up(size_t(kChunk) * ld * sizeof(T) * (alias ? 1 : 2), 16) +
                            size_t(kHeads) * D * 4 + size_t(kHeads) * kChunk * 4;
        auto kern = attn_partial<T>;
        LSA_CUDA(ensure_smem(kern, size_t(int(smem))));
        dim3 grid(nchunks, (Hq + kHeads - 1) / kHeads, B);
        kern<<<grid, kAttnThreads, smem, st>>>(static_cast<const T *>(Q), static_cast<const T *>(kv), stride,
                                               k_off, v_off, rows, Hq, D, k, scale, pp.o, pp.ml);
        LSA_LAUNCHED("attn_partial");
        return launch_combine<T, float>(pp.o, pp.ml, nchunks, B, Hq, D, out, lse, st);
    }
}

}  // namespace

size_t sparse_attn_workspace(int32_t B, int32_t Hq, int32_t D, int32_t k) {
    const int nchunks = (k + kChunk - 1) / kChunk;   // the finer of the two chunkings
    return (align_up(size_t(B) * nchunks * Hq * D, 64) + size_t(B) * nchunks * Hq * 2) * sizeof(float);
}

lsa_status launch_sparse_attn(const void *Q, lsa_dtype dtype, const void *kv, int64_t stride,
                              int64_t k_off, int64_t v_off, const int32_t *rows, int32_t B,
                              int32_t Hq, int32_t D, int32_t k, float scale, void *out, float *lse,
                              void *workspace, int32_t *err, cudaStream_t st) {
    if (dtype == LSA_F32)
        return launch_t<float>(Q, kv, stride, k_off, v_off, rows, B, Hq, D, k, scale, out, lse, workspace, err, st);
    return launch_t<uint16_t>(Q, kv, stride, k_off, v_off, rows, B, Hq, D, k, scale, out, lse, workspace, err, st);
}

}  // namespace lsa
