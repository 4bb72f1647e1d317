// OR-mode union of several indexer layers ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.4
// "Optimal Configuration": independent Memory Indexers on three layers, whose
// predictions are united at inference to decide what is fetched).
//
// Layer l keeps entry s when I_l(s) >= 0.5, i.e. z_l(s) >= 0, so the union
// keeps s exactly when max_l z_l(s) >= 0.  This kernel writes that maximum:
// lsa_select on it gives the union's kept set, and it is the union's ranking
// score for the top-k.  The maximum of fp32 values is exact, so the result is
// bit-identical to any other correct evaluation (a NaN counts as "not kept"
// by its layer: fmaxf ignores it).
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kMaxLayers = kMaxUnionLayers;
constexpr int kThreads = 256;

struct LayerPtrs {
    const float *p[kMaxLayers];
};

// Grid-stride; four entries per thread step when every pointer is 16-byte aligned and n % 4 == 0.
__global__ void __launch_bounds__(kThreads) union_max(LayerPtrs zs, int n_layers, int64_t n, int vec4,
                                                      float *__restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();   // the layers' scores come from preceding kernels
    const int64_t stride = int64_t(gridDim.x) * kThreads;
    if (vec4) {
        const int64_t n4 = n / 4;
        for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n4; i += stride) {
            float4 m = reinterpret_cast<const float4 *>(zs.p[0])[i];
            for (int l = 1; l < n_layers; ++l) {
                const float4 v = reinterpret_cast<const float4 *>(zs.p[l])[i];
                m.x = fmaxf(m.x, v.x); m.y = fmaxf(m.y, v.y); m.z = fmaxf(m.z, v.z); m.w = fmaxf(m.w, v.w);
            }
            reinterpret_cast<float4 *>(out)[i] = m;
        }
        return;
    }
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride) {
        float m = zs.p[0][i];
        for (int l = 1; l < n_layers; ++l) m = fmaxf(m, zs.p[l][i]);
        out[i] = m;
    }
}

}  // namespace

lsa_status launch_union(const float *const *z_layers, int32_t n_layers, int64_t n_total, float *z_union,
                        cudaStream_t st) {
    LayerPtrs zs = {};
    bool aligned = (reinterpret_cast<uintptr_t>(z_union) & 15) == 0 && n_total % 4 == 0;
    for (int l = 0; l < n_layers; ++l) {
        zs.p[l] = z_layers[l];
        aligned = aligned && (reinterpret_cast<uintptr_t>(z_layers[l]) & 15) == 0;
    }
    if (n_total == 0) return LSA_OK;
    const int64_t units = aligned ? n_total / 4 : n_total;
    const int64_t want = (units + kThreads - 1) / kThreads;
    const int grid = int(want < int64_t(sm_count()) * 8 ? want : int64_t(sm_count()) * 8);
    LSA_CUDA(launch_pdl(union_max, dim3(grid), dim3(kThreads), 0, st, zs, int(n_layers), n_total, int(aligned),
                        z_union));
    LSA_LAUNCHED("union_max");
    return LSA_OK;
}

}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_index_union(const float *const *z_layers, int32_t n_layers, int64_t n_total, float *z_union,
                                      void *stream) {
    clear_error();
    LSA_CHECK_ARG(z_layers && z_union, "lsa_index_union: z_layers and z_union are required");
    LSA_CHECK_ARG(n_layers >= 1 && n_layers <= kMaxLayers, "lsa_index_union: n_layers=%d not in [1, %d]", n_layers,
                  kMaxLayers);
    LSA_CHECK_ARG(n_total >= 0, "lsa_index_union: n_total=%lld < 0", (long long)n_total);
    for (int l = 0; l < n_layers; ++l) LSA_CHECK_ARG(z_layers[l], "lsa_index_union: layer %d has no scores", l);
    return launch_union(z_layers, n_layers, n_total, z_union, as_stream(stream));
}
