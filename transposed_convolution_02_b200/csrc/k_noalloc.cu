// ct_run_noalloc: ct_run for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc (or any allocator)
// once they are running: a plugin hosted by an inference engine that owns
// every byte of device memory, or a latency-critical loop whose rules forbid
// allocation after start-up.  They still have to provide X, the packed
// weight, the bias and Y, but not the workspace: this entry point supplies
// the workspace from a fixed array compiled into the library.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library's device code holds CT_NOALLOC_SCRATCH_BYTES of it until the
// process exits.  Host code never hands the symbol itself to a kernel (on the
// host it only names a stand-in): every call looks up the array's device
// address with cudaGetSymbolAddress on the current device, which allocates
// nothing once the module is loaded and stays right after a device reset.
// With lazy module loading the first lookup on a device loads the module, and
// with it the array; callers make that first call at start-up.  All calls
// share the one array and it keeps the last call's contents: the kernels
// overwrite every workspace byte they later read, so nothing needs clearing,
// but calls whose GPU work overlaps (different streams) race on it.
#include "ct_cuda_util.h"
#include "ct_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_ct_noalloc_scratch[CT_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" ct_status ct_run_noalloc(const ct_plan_t *plan, const void *x, const void *w_packed,
                                    const void *bias, void *y, void *stream) {
    if (!plan) return CT_ERR_NULL;
    size_t need = 0;
    ct_status st = ct_workspace_bytes(plan, &need);
    if (st != CT_OK) return st;
    if (need > (size_t)CT_NOALLOC_SCRATCH_BYTES) return CT_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0) {
        if (ct::current_device() < 0) return CT_ERR_DEVICE;
        if (cudaGetSymbolAddress(&ws, g_ct_noalloc_scratch) != cudaSuccess || !ws) {
            cudaGetLastError();
            return CT_ERR_DEVICE;
        }
    }
    return ct_run(plan, x, w_packed, bias, y, ws, stream);
}
