// lsa_select_noalloc: the threshold selection of lsa_select with its scratch in
// a static device array, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) when they
// need the selection: code running while a stream is being captured in a mode
// that forbids allocation, runtimes that hand every byte of device memory to
// their own pool at start-up (a stray cudaMalloc fails or fragments it), and
// plugin-style hosts that invoke a kernel without passing a workspace.  This
// entry point needs no workspace from them: its scratch is the file-scope
// array below, which every GPU that loads the library holds until the process
// exits.
//
// The array's name is only a host-side stand-in in host code; its device
// address is looked up with cudaGetSymbolAddress on the first call made on
// each device (with that device current) and cached with the CUDA context it
// belongs to: after a device reset the next call finds a new context and looks
// the address up again.  With lazy module loading (the CUDA 12 default) that
// first call also loads the library's device code, which creates the array in
// device memory; so the first call on a device is the set-up call: make it
// before any stream capture and before a runtime claims the rest of the
// device's memory.  Every call on a device shares the one array, so calls that
// overlap on the GPU (different streams, no ordering between them) race on it.
// Nothing in it needs to start at zero: each call writes every scratch word it
// reads before reading it.
#include <cuda.h>

#include <mutex>

#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int64_t kNoallocMaxEntries = int64_t(1) << 22;   // 4,194,304 entries per call

constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }
// the select workspace for kNoallocMaxEntries: tile bases, tile counts, mask words
constexpr size_t kScratchBytes = align256(size_t((kNoallocMaxEntries + 1023) / 1024) * 8) +
                                 align256(size_t((kNoallocMaxEntries + 1023) / 1024) * 4) +
                                 align256(size_t((kNoallocMaxEntries + 31) / 32) * 4);

__device__ __align__(256) uint8_t g_select_scratch[kScratchBytes];

std::mutex g_mu;
struct Cached {
    CUcontext ctx;   // the context the address was looked up in
    void *addr;
};
Cached g_addr[64] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, through the runtime's entry-point query (the
// library links no driver import library).
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// Device address of the scratch on the current device, looked up once per
// device and context.
lsa_status scratch_address(void **out) {
    int dev = 0;
    LSA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) {
        set_error("lsa_select_noalloc: device ordinal %d out of range", dev);
        return LSA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (get && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    // no context current yet on this thread (or no way to ask): the lookup itself makes the device's primary
    // context current; the address is cached only together with a known context
    if (ctx == nullptr || !g_addr[dev].addr || g_addr[dev].ctx != ctx) {
        void *p = nullptr;
        LSA_CUDA(cudaGetSymbolAddress(&p, g_select_scratch));
        if (get && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
        g_addr[dev] = {ctx, p};
    }
    *out = g_addr[dev].addr;
    return LSA_OK;
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" {

int64_t lsa_select_noalloc_max_entries(void) { return kNoallocMaxEntries; }

lsa_status lsa_select_noalloc(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B, int32_t *kept_idx,
                              int64_t capacity, int64_t *kept_off, uint32_t *mask, int32_t *err, void *stream) {
    clear_error();
    LSA_CHECK_ARG(z && seq_off && kept_off, "lsa_select_noalloc: z, seq_off and kept_off are required");
    LSA_CHECK_ARG(B >= 1, "lsa_select_noalloc: B=%d", B);
    LSA_CHECK_ARG(n_total >= 0, "lsa_select_noalloc: n_total=%lld < 0", (long long)n_total);
    LSA_CHECK_ARG(n_total <= kNoallocMaxEntries,
                  "lsa_select_noalloc: n_total=%lld exceeds the static scratch limit of %lld entries "
                  "(use lsa_select with a workspace)",
                  (long long)n_total, (long long)kNoallocMaxEntries);
    LSA_CHECK_ARG(capacity >= 0 && (kept_idx || capacity == 0), "lsa_select_noalloc: bad capacity / kept_idx");
    if (lsa_select_workspace_size(n_total) > kScratchBytes) {   // the two layouts must agree
        set_error("lsa_select_noalloc: scratch layout mismatch");
        return LSA_ERR_UNSUPPORTED;
    }
    void *scratch = nullptr;
    const lsa_status s = scratch_address(&scratch);
    if (s != LSA_OK) return s;
    return launch_select(z, seq_off, n_total, B, kept_idx, capacity, kept_off, mask, scratch, err,
                         as_stream(stream));
}

}  // extern "C"
