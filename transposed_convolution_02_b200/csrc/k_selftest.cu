// Self-test of the bounded-wait failure path shared by the tensor-core and
// grouped kernels (no counterpart on the pages): a wait that runs out
// records its site in a device error word, the thread then waits for its
// own copy still in flight (bounded again) and returns, so the context
// stays usable and ct_take_device_error reports the site.
#include "ct_cuda_util.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

constexpr unsigned kSelftestBytes = 4096;

__device__ int g_selftest_err;
// source of the bulk copy that is in flight when the wait gives up
__device__ __align__(16) unsigned char g_selftest_src[kSelftestBytes];

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(long long limit) {
    using namespace sm100;
    __shared__ __align__(128) unsigned char buf[kSelftestBytes];
    __shared__ __align__(8) uint64_t bars[2];
    if (threadIdx.x != 0) return;
    const uint32_t copied = smem_u32(&bars[0]), never = smem_u32(&bars[1]);
    mbar_init(copied, 1);
    mbar_init(never, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(copied, kSelftestBytes);
    bulk_load(smem_u32(buf), g_selftest_src, kSelftestBytes, copied);
    // nothing arrives at `never`: this wait runs out after `limit` cycles
    if (!mbar_wait_for(never, 0, &g_selftest_err, 1, limit)) {
        // the give-up path: drain the copy into this CTA's shared memory
        // before the CTA exits (site 2 if even that does not complete)
        mbar_wait(copied, 0, &g_selftest_err, 2);
        return;
    }
    mbar_wait(copied, 0, &g_selftest_err, 3);   // not reached: `never` completed
}

}  // namespace

int selftest_take_error(cudaStream_t st) { return take_error_word(g_selftest_err, st); }

}  // namespace ct

extern "C" ct_status ct_selftest_wait_timeout(void *stream, int64_t limit_cycles) {
    if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 31)) return CT_ERR_ATTR;
    if (ct::current_device() < 0) return CT_ERR_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, ct::current_device()) != cudaSuccess ||
        major != 10) {
        cudaGetLastError();
        return CT_ERR_DEVICE;
    }
    ct::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((long long)limit_cycles);
    return ct::launch_status();
}
