// lsa_selftest_bounded_wait: runs the bounded device-side wait that every
// tcgen05 kernel of the library uses, on an mbarrier that nothing ever
// arrives at, so that its expiry path can be checked on a GPU without a
// fault or a hang: the wait gives up after limit_ns of %globaltimer time, the
// kernel records LSA_ERR_TIMEOUT in the caller's error word and returns, and
// the context stays usable.  A second warp then shows the early exit of the
// same wait when another warp of the CTA raises the abort flag.
#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace ptx;

__global__ void __launch_bounds__(64, 1) bounded_wait_probe(uint64_t limit_ns, int32_t *err, int64_t *waited_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    volatile int *abort_v = &abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // count 1; nothing arrives
        fence_mbar_init();
        abort_flag = 0;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        // 1. the wait runs out: it sets the abort flag and returns false
        const uint64_t t0 = global_timer_ns();
        const bool ok = mbar_wait(&bar, 0, abort_v, limit_ns);
        waited_ns[0] = int64_t(global_timer_ns() - t0);
        if (!ok) raise_err(err, LSA_ERR_TIMEOUT);
    } else if (warp == 1 && lane == 0) {
        // 2. a wait that sees the abort flag raised by another warp returns at once
        const uint64_t t0 = global_timer_ns();
        const bool ok = mbar_wait(&bar, 0, abort_v, 4 * limit_ns);
        waited_ns[1] = int64_t(global_timer_ns() - t0);
        waited_ns[2] = ok ? 1 : 0;
    }
    __syncwarp();
    __syncthreads();
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_selftest_bounded_wait(int64_t limit_ns, int32_t *err, int64_t *waited_ns, void *stream) {
    clear_error();
    LSA_CHECK_ARG(err && waited_ns, "lsa_selftest_bounded_wait: err and waited_ns are required");
    LSA_CHECK_ARG(limit_ns >= 1000 && limit_ns <= 100000000,
                  "lsa_selftest_bounded_wait: limit_ns=%lld outside [1 us, 100 ms]", (long long)limit_ns);
    bounded_wait_probe<<<1, 64, 0, as_stream(stream)>>>(uint64_t(limit_ns), err, waited_ns);
    LSA_LAUNCHED("bounded_wait_probe");
    return LSA_OK;
}
