// Indexer query encoder ("FlashMemory-DeepSeek-V4 ... Lookahead Sparse
// Attention", gist.science technical summary, section 2.1 "Memory Indexer":
// the current query token's hidden state h_t is mapped to low-rank indexer
// queries; section 2.3 "Query Optimization": the encoder's trained part is its
// low-rank projection matrices).  Read as a rank-r factorisation:
//     c = W_dq h,   q_j = rows j*d .. j*d+d-1 of W_uq c,   w = W_w h.
//
// At decode batch sizes every product is a skinny matrix-vector product whose
// cost is streaming the bf16 weight matrices from HBM (rank*hidden +
// H*hidden + H*d*rank elements, ~48 MB at hidden 7168, rank 1536, H 64,
// d 128); the batch rows are too few for a tensor-core tile to pay.  Two
// passes, each one weight stream:
//   pass 1: the rows of W_dq and W_w (stacked) against h  -> c, w (fp32)
//   pass 2: the rows of W_uq against c                    -> q (bf16 / fp32)
// A warp owns 4 weight rows and a strided set of 256-element chunks of their
// K range; each lane streams 16 bytes of each row per chunk (coalesced
// 512-byte row segments per warp) into its own slots of a 4-deep shared-memory
// ring with cp.async, so four chunks per warp are in flight without holding
// registers, and reads back only what it copied itself (no barriers).  The
// warps of a CTA split K when there are too few row groups to fill the GPU;
// their partial sums are added in a fixed order, so results are
// deterministic.  The grid is sized to one wave.  Pass 1 also prefetches
// W_uq into L2 (a bulk prefetch per CTA), so both passes' weights share one
// HBM stream and pass 2 reads its weights from L2.  Batch rows beyond 4 are
// further grid rows that read the same weights.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 4;      // weight rows per warp
constexpr int kChunk = 256;   // K elements per warp chunk: 32 lanes x 8

// Chunks in flight per warp: three keep ~144 KB per SM in flight at three
// CTAs per SM (measured: two to four stages time the same at batch 4).
constexpr int kDepth = 3;
constexpr int kStageU4 = kRows * 32;     // 16-byte slots of one warp stage (4 rows x 32 lanes)
constexpr size_t kRingBytes = size_t(kWarps) * kDepth * kStageU4 * 16;   // 48 KB per CTA
constexpr int kMinCtasPerSm = 3;

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// The 8 bf16 values of a 16-byte word, widened to fp32 (exact).
__device__ __forceinline__ void widen8(const uint4 v, float *f) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// x[b, k0 .. k0+8) as fp32; x is bf16 (X_F32 false) or fp32, row-major [B, K].
// Plain (coherent) loads: in pass 2 x was written by the kernel before.
template <bool X_F32>
__device__ __forceinline__ void load_x8(const void *x, int64_t off, float *f) {
    if constexpr (X_F32) {
        const float4 a = *reinterpret_cast<const float4 *>(static_cast<const float *>(x) + off);
        const float4 b = *reinterpret_cast<const float4 *>(static_cast<const float *>(x) + off + 4);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        widen8(*reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + off), f);
    }
}

// y[b, n] = sum_k W_n[k] x[b, k] for the stacked rows n < n0 (W0, into y0) and
// n0 <= n < n0 + n1 (W1, into y1).  Warp w of a CTA takes row group
// w / ks and K split w % ks; grid.y runs over groups of NB batch rows.  When
// pf is set, blockIdx.y == 0 CTAs bulk-prefetch their share of pf_bytes
// bytes at pf into L2.
template <int NB, bool X_F32, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, kMinCtasPerSm)
    encode_rows(const uint16_t *__restrict__ W0, int n0, const uint16_t *__restrict__ W1, int n1, int K, int ks,
                const void *x, int B, void *y0, float *y1, const uint8_t *pf, int64_t pf_bytes) {
    extern __shared__ uint4 ring[];
    __shared__ float red[kWarps][kRows * NB];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups_per_cta = kWarps / ks;
    const int g = warp / ks, split = warp % ks;
    const int nrows = n0 + n1;
    const int row0 = (blockIdx.x * groups_per_cta + g) * kRows;
    const int b0 = blockIdx.y * NB;

    const uint16_t *wrow[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int n = min(row0 + r, nrows - 1);   // rows past the end re-read the last row; not written
        wrow[r] = n < n0 ? W0 + int64_t(n) * K : W1 + int64_t(n - n0) * K;
    }
    uint4 *mine = ring + size_t(warp) * kDepth * kStageU4 + lane;   // this lane's slot, stage 0, row 0
    const int nch = (K + kChunk - 1) / kChunk;
    const int count = split < nch ? (nch - split + ks - 1) / ks : 0;   // chunks of this warp

    // chunk i of this warp -> stage i % kDepth; one commit group per chunk (empty past the end)
    auto issue = [&](int i) {
        if (i < count) {
            const int k0 = (split + i * ks) * kChunk + lane * 8;
            if (k0 < K) {
                uint4 *st = mine + (i % kDepth) * kStageU4;
#pragma unroll
                for (int r = 0; r < kRows; ++r) cp_async16(st + r * 32, wrow[r] + k0);
            }
        }
        cp_async_commit();
    };

    pdl_launch_dependents();
    // the weights depend on no earlier kernel: start streaming them before waiting
#pragma unroll
    for (int i = 0; i < kDepth; ++i) issue(i);
    if (pf && blockIdx.y == 0 && threadIdx.x == 0) {
        const int64_t share = ((pf_bytes + gridDim.x - 1) / gridDim.x + 15) / 16 * 16;
        const int64_t end = min(pf_bytes, int64_t(blockIdx.x + 1) * share);
        for (int64_t o = int64_t(blockIdx.x) * share; o < end; o += 65536)
            prefetch_l2(pf + o, uint32_t(min(int64_t(65536), end - o)));
    }
    pdl_wait();

    float acc[kRows][NB];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) acc[r][bb] = 0.f;

    int64_t xoff[NB];
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) xoff[bb] = int64_t(min(b0 + bb, B - 1)) * K;   // rows past B: not written

    for (int i = 0; i < count; ++i) {
        const int k0 = (split + i * ks) * kChunk + lane * 8;
        const bool live = k0 < K;
        float xf[NB][8];
        if (live) {
#pragma unroll
            for (int bb = 0; bb < NB; ++bb) load_x8<X_F32>(x, xoff[bb] + k0, xf[bb]);
        }
        cp_async_wait<kDepth - 1>();   // chunk i's group has landed (groups complete in order)
        if (live) {
            const uint4 *st = mine + (i % kDepth) * kStageU4;
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                float wf[8];
                widen8(st[r * 32], wf);
#pragma unroll
                for (int bb = 0; bb < NB; ++bb)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[r][bb] = fmaf(wf[e], xf[bb][e], acc[r][bb]);
            }
        }
        issue(i + kDepth);   // refills the stage just read (this lane's own slots)
    }
    cp_async_wait<0>();

    // lanes -> warp total (butterfly: every lane ends with the sum), then the K splits in order
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
            float v = acc[r][bb];
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == r * NB + bb) red[warp][r * NB + bb] = v;
        }
    __syncthreads();
    const int t = threadIdx.x;
    if (t < groups_per_cta * kRows * NB) {
        const int gi = t / (kRows * NB), v = t % (kRows * NB);
        float s = 0.f;
        for (int sp = 0; sp < ks; ++sp) s += red[gi * ks + sp][v];
        const int n = (blockIdx.x * groups_per_cta + gi) * kRows + v / NB;
        const int b = b0 + v % NB;
        if (n < nrows && b < B) {
            if (n < n0) {
                if constexpr (OUT_BF16)
                    reinterpret_cast<__nv_bfloat16 *>(y0)[int64_t(b) * n0 + n] = __float2bfloat16_rn(s);
                else
                    reinterpret_cast<float *>(y0)[int64_t(b) * n0 + n] = s;
            } else {
                y1[int64_t(b) * n1 + (n - n0)] = s;
            }
        }
    }
}

// K splits per row group: as many as fit the grid in one wave of resident
// CTAs (more warps in flight), at most one split per chunk, at most the 8
// warps of a CTA.
int pick_splits(int nrows, int K, int batch_groups, int slots) {
    const int64_t groups = (nrows + kRows - 1) / kRows;
    const int nch = (K + kChunk - 1) / kChunk;
    int ks = 1;
    while (ks < kWarps && ks * 2 <= nch && (groups * ks * 2 + kWarps - 1) / kWarps * batch_groups <= slots) ks *= 2;
    return ks;
}

template <int NB, bool X_F32, bool OUT_BF16>
cudaError_t launch_nb(const uint16_t *W0, int n0, const uint16_t *W1, int n1, int K, const void *x, int B,
                      void *y0, float *y1, const void *pf, int64_t pf_bytes, cudaStream_t st) {
    auto kern = encode_rows<NB, X_F32, OUT_BF16>;
    cudaError_t e = ensure_smem(kern, kRingBytes);   // per device
    if (e != cudaSuccess) return e;
    static int per_sm = -1;   // resident CTAs per SM of this instance (one GPU model per process)
    if (per_sm < 0) {
        int n = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, kRingBytes);
        if (e != cudaSuccess) return e;
        per_sm = n < 1 ? 1 : n;
    }
    const int nrows = n0 + n1;
    const int bgroups = (B + NB - 1) / NB;
    const int ks = pick_splits(nrows, K, bgroups, per_sm * sm_count());
    const int gpc = kWarps / ks;
    const int groups = (nrows + kRows - 1) / kRows;
    const dim3 grid((groups + gpc - 1) / gpc, bgroups);
    return launch_pdl(kern, grid, dim3(kThreads), kRingBytes, st, W0, n0, W1, n1, K, ks, x, B, y0, y1,
                      static_cast<const uint8_t *>(pf), pf_bytes);
}

template <bool X_F32, bool OUT_BF16>
cudaError_t launch_pass(const uint16_t *W0, int n0, const uint16_t *W1, int n1, int K, const void *x, int B,
                        void *y0, float *y1, const void *pf, int64_t pf_bytes, cudaStream_t st) {
    if (B == 1) return launch_nb<1, X_F32, OUT_BF16>(W0, n0, W1, n1, K, x, B, y0, y1, pf, pf_bytes, st);
    if (B == 2) return launch_nb<2, X_F32, OUT_BF16>(W0, n0, W1, n1, K, x, B, y0, y1, pf, pf_bytes, st);
    return launch_nb<4, X_F32, OUT_BF16>(W0, n0, W1, n1, K, x, B, y0, y1, pf, pf_bytes, st);
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_query_encode(const void *h, int32_t B, int32_t hidden, const void *W_dq, int32_t rank,
                                       const void *W_uq, int32_t H, int32_t d, const void *W_w, void *q_out,
                                       lsa_dtype q_dtype, float *w_out, float *c_out, void *stream) {
    clear_error();
    LSA_CHECK_ARG(h && W_dq && W_uq && W_w && q_out && w_out && c_out,
                  "lsa_query_encode: h, W_dq, W_uq, W_w, q_out, w_out and c_out are required");
    LSA_CHECK_ARG(B >= 1 && B <= 65535 * 4, "lsa_query_encode: B=%d out of range", B);
    LSA_CHECK_ARG(hidden >= 8 && hidden % 8 == 0, "lsa_query_encode: hidden=%d must be a positive multiple of 8",
                  hidden);
    LSA_CHECK_ARG(rank >= 8 && rank % 8 == 0, "lsa_query_encode: rank=%d must be a positive multiple of 8", rank);
    LSA_CHECK_ARG(H >= 1 && d >= 1 && int64_t(H) * d <= (int64_t(1) << 30), "lsa_query_encode: H=%d d=%d", H, d);
    LSA_CHECK_ARG(int64_t(rank) + H <= (int64_t(1) << 30), "lsa_query_encode: rank + H too large");
    LSA_CHECK_SUPPORTED(q_dtype == LSA_BF16 || q_dtype == LSA_F32, "lsa_query_encode: q dtype must be BF16 or F32");
    LSA_CHECK_ARG(aligned16(h) && aligned16(W_dq) && aligned16(W_uq) && aligned16(W_w) && aligned16(c_out),
                  "lsa_query_encode: h, W_dq, W_uq, W_w and c_out must be 16-byte aligned");
    cudaStream_t st = as_stream(stream);
    const auto *Wd = static_cast<const uint16_t *>(W_dq);
    const auto *Ww = static_cast<const uint16_t *>(W_w);
    const auto *Wu = static_cast<const uint16_t *>(W_uq);
    const int64_t uq_bytes = int64_t(H) * d * rank * 2;
    LSA_CUDA((launch_pass<false, false>(Wd, rank, Ww, H, hidden, h, B, c_out, w_out, Wu, uq_bytes, st)));
    LSA_LAUNCHED("encode_rows (W_dq | W_w)");
    if (q_dtype == LSA_BF16)
        LSA_CUDA((launch_pass<true, true>(Wu, H * d, nullptr, 0, rank, c_out, B, q_out, nullptr, nullptr, 0, st)));
    else
        LSA_CUDA((launch_pass<true, false>(Wu, H * d, nullptr, 0, rank, c_out, B, q_out, nullptr, nullptr, 0, st)));
    LSA_LAUNCHED("encode_rows (W_uq)");
    return LSA_OK;
}
