// Generic direct ConvTranspose kernel: one thread per output element gathers
// every (channel, tap) pair that lands on it.  Serves any rank, stride,
// dilation, padding, group, layout and both dtypes; the specialised kernels
// take the shapes that matter for speed.
//
// For output position o on an axis with stride s, dilation d and begin pad pb,
// tap k contributes iff (o + pb - k*d) is a non-negative multiple of s, and
// it reads input position i = (o + pb - k*d) / s (ai.onnx.ConvTranspose
// README, "Description": the scatter o = i*s - pb + k*d read backwards).
#include "ct_internal.h"

namespace ct {
namespace {

struct GenericArgs {
    int64_t N, C, M, Cg, Mg;
    int64_t in[3], k[3], s[3], d[3], pb[3], out[3];
    int64_t total;
    int nhwc;
    int has_bias;
};

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }

template <typename T>
__global__ void __launch_bounds__(256) generic_kernel(GenericArgs a, const T *__restrict__ x,
                                                      const T *__restrict__ w,
                                                      const T *__restrict__ bias,
                                                      T *__restrict__ y) {
    const int64_t in_sz = a.in[0] * a.in[1] * a.in[2];
    const int64_t k_sz = a.k[0] * a.k[1] * a.k[2];
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < a.total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        int64_t n, m, o[3];
        int64_t rem = idx;
        if (a.nhwc) {
            m = rem % a.M; rem /= a.M;
            o[2] = rem % a.out[2]; rem /= a.out[2];
            o[1] = rem % a.out[1]; rem /= a.out[1];
            o[0] = rem % a.out[0]; rem /= a.out[0];
            n = rem;
        } else {
            o[2] = rem % a.out[2]; rem /= a.out[2];
            o[1] = rem % a.out[1]; rem /= a.out[1];
            o[0] = rem % a.out[0]; rem /= a.out[0];
            m = rem % a.M; rem /= a.M;
            n = rem;
        }
        const int64_t g = m / a.Mg, ml = m % a.Mg;
        float acc = 0.f;
        for (int64_t k0 = 0; k0 < a.k[0]; ++k0) {
            const int64_t t0 = o[0] + a.pb[0] - k0 * a.d[0];
            if (t0 < 0) break;
            if (t0 % a.s[0]) continue;
            const int64_t i0 = t0 / a.s[0];
            if (i0 >= a.in[0]) continue;
            for (int64_t k1 = 0; k1 < a.k[1]; ++k1) {
                const int64_t t1 = o[1] + a.pb[1] - k1 * a.d[1];
                if (t1 < 0) break;
                if (t1 % a.s[1]) continue;
                const int64_t i1 = t1 / a.s[1];
                if (i1 >= a.in[1]) continue;
                for (int64_t k2 = 0; k2 < a.k[2]; ++k2) {
                    const int64_t t2 = o[2] + a.pb[2] - k2 * a.d[2];
                    if (t2 < 0) break;
                    if (t2 % a.s[2]) continue;
                    const int64_t i2 = t2 / a.s[2];
                    if (i2 >= a.in[2]) continue;
                    const int64_t ipos = (i0 * a.in[1] + i1) * a.in[2] + i2;
                    const int64_t kpos = (k0 * a.k[1] + k1) * a.k[2] + k2;
                    for (int64_t cl = 0; cl < a.Cg; ++cl) {
                        const int64_t c = g * a.Cg + cl;
                        const T xv = a.nhwc ? x[(n * in_sz + ipos) * a.C + c]
                                            : x[(n * a.C + c) * in_sz + ipos];
                        const T wv = a.nhwc ? w[(c * k_sz + kpos) * a.Mg + ml]
                                            : w[(c * a.Mg + ml) * k_sz + kpos];
                        acc = fmaf(to_f(xv), to_f(wv), acc);
                    }
                }
            }
        }
        if (a.has_bias) acc += to_f(bias[m]);
        y[idx] = from_f<T>(acc);
    }
}

}  // namespace

bool generic_supports(const Plan &) { return true; }

// The generic kernel reads W in its declared layout: the packed form is a copy.
size_t generic_packed_bytes(const Plan &p) {
    size_t b = (size_t)(p.C * p.Mg * numel_k(p)) * elem_bytes(p);
    return b ? b : 16;
}

ct_status generic_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const size_t b = (size_t)(p.C * p.Mg * numel_k(p)) * elem_bytes(p);
    if (b == 0) return CT_OK;
    if (cudaMemcpyAsync(wp, w, b, cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
        cudaGetLastError();
        return CT_ERR_DEVICE;
    }
    return CT_OK;
}

ct_status generic_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                      cudaStream_t st) {
    GenericArgs a;
    a.N = p.N; a.C = p.C; a.M = p.M; a.Cg = p.Cg; a.Mg = p.Mg;
    for (int i = 0; i < 3; ++i) {
        a.in[i] = p.in[i]; a.k[i] = p.k[i]; a.s[i] = p.s[i]; a.d[i] = p.d[i];
        a.pb[i] = p.pb[i]; a.out[i] = p.out[i];
    }
    a.total = p.N * p.M * numel_out(p);
    a.nhwc = p.layout == CT_NHWC;
    a.has_bias = p.has_bias;
    if (a.total == 0) return CT_OK;
    const int threads = 256;
    int64_t blocks = ceil_div(a.total, threads);
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (p.dtype == CT_F16)
        generic_kernel<__half><<<(unsigned)blocks, threads, 0, st>>>(
            a, (const __half *)x, (const __half *)wp, (const __half *)bias, (__half *)y);
    else
        generic_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            a, (const float *)x, (const float *)wp, (const float *)bias, (float *)y);
    return launch_status();
}

}  // namespace ct
