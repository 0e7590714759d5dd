// Internal plan structure and kernel-module hooks of libct.so.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/ct.h"

namespace ct {

// One kernel tap of one output phase along one axis.  For output position
// o = s*J + r (r the phase, J the position inside the phase), the taps of the
// phase are the k with (r + pad_begin - k*d) divisible by s, and tap k reads
// the input at i = J + e with e = (r + pad_begin - k*d) / s.
struct Tap {
    int32_t k;
    int32_t e;
};

// A plan: the resolved geometry, padded to three spatial axes with leading
// axes of size 1 (kernel 1, stride 1, dilation 1, no pad), plus the phase
// tables and the chosen kernel.
struct Plan {
    ct_desc desc;
    int rank;                 // spatial rank as given (1..3)
    int dtype;                // ct_dtype
    int layout;               // ct_layout
    int64_t N, C, M, G, Cg, Mg;
    int64_t in[3], k[3], s[3], d[3], pb[3], pe[3], op[3], out[3];
    bool has_bias;
    int act;                  // ct_activation applied after the bias
    int algo;                 // chosen ct_algo
    size_t packed_bytes;
    size_t ws_bytes;
    int launches;                   // kernels one ct_run launches
    std::vector<Tap> taps[3][64];   // per axis, per phase r (< s <= 64 for tabled kernels)
    int64_t nJ[3][64];              // outputs per phase: ceil((out - r) / s)
    bool tabled;                    // phase tables filled (every stride <= 64)
    // kernel-specific precomputation (opaque to the API layer)
    std::vector<int64_t> aux;
};

inline int64_t numel_in(const Plan &p) { return p.in[0] * p.in[1] * p.in[2]; }
inline int64_t numel_out(const Plan &p) { return p.out[0] * p.out[1] * p.out[2]; }
inline int64_t numel_k(const Plan &p) { return p.k[0] * p.k[1] * p.k[2]; }
inline size_t elem_bytes(const Plan &p) { return p.dtype == CT_F16 ? 2 : 4; }

// ---- kernel modules -------------------------------------------------------
// Each module answers whether it serves a plan, how many packed-weight and
// workspace bytes it needs, and launches its prepack and run kernels.

bool generic_supports(const Plan &p);
size_t generic_packed_bytes(const Plan &p);
ct_status generic_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status generic_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                      cudaStream_t st);

// shared layout helpers (k_relayout.cu)
ct_status launch_nchw_to_nhwc_f16(const Plan &p, const void *x, void *xt, cudaStream_t st);
bool has_dead_phases(const Plan &p);
ct_status launch_dead_fill(const Plan &p, const void *bias, void *y, cudaStream_t st);

bool dense_pertap_supports(const Plan &p);
size_t dense_pertap_packed_bytes(const Plan &p);
size_t dense_pertap_ws_bytes(const Plan &p);
void dense_pertap_setup(Plan &p);
ct_status dense_pertap_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status dense_pertap_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                           void *ws, cudaStream_t st, int parts);

bool dense_tc_supports(const Plan &p);
size_t dense_tc_packed_bytes(const Plan &p);
size_t dense_tc_ws_bytes(const Plan &p);
void dense_tc_setup(Plan &p);
ct_status dense_tc_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status dense_tc_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                       void *ws, cudaStream_t st, int parts);

bool dense_pair_supports(const Plan &p);
bool dense_pair_preferred(const Plan &p);   // auto selection: where it measured fastest
size_t dense_pair_packed_bytes(const Plan &p);
size_t dense_pair_ws_bytes(const Plan &p);
void dense_pair_setup(Plan &p);
ct_status dense_pair_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status dense_pair_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                         void *ws, cudaStream_t st, int parts);

bool fp32_gemm_supports(const Plan &p);
void fp32_gemm_plan(Plan &p);
size_t fp32_gemm_packed_bytes(const Plan &p);
ct_status fp32_gemm_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status fp32_gemm_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                        cudaStream_t st, int parts);

bool grouped_supports(const Plan &p);
void grouped_plan(Plan &p);
size_t grouped_packed_bytes(const Plan &p);
ct_status grouped_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st);
ct_status grouped_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                      cudaStream_t st);

// Device error words of the tensor-core and grouped modules: the code of a
// bounded wait that ran out since the last read (0: none; -1: CUDA failed),
// read in order on the stream and cleared.
int dense_tc_take_error(cudaStream_t st);
int dense_pertap_take_error(cudaStream_t st);
int dense_pair_take_error(cudaStream_t st);
int grouped_take_error(cudaStream_t st);
int selftest_take_error(cudaStream_t st);

// Map the last CUDA error to a status (and clear it).
inline ct_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CT_OK : CT_ERR_DEVICE;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// The output activation (ct_activation), applied in fp32 after the bias.
#ifdef __CUDACC__
__device__ __forceinline__ float apply_act(float v, int act) { return act == CT_ACT_RELU ? fmaxf(v, 0.f) : v; }
#endif

}  // namespace ct
