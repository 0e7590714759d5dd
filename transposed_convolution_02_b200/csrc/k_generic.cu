// Generic direct ConvTranspose kernel: one thread per output element gathers
// every (channel, tap) pair that lands on it.  Serves any rank, stride,
// dilation, padding, group, layout and both dtypes; the specialised kernels
// take the shapes that matter for speed.
//
// Two forms: when every index fits in 32 bits and the strides have phase
// tables, a thread splits each output coordinate o into o = s*J + r (r the
// stride phase) once and walks only the taps of phase r, reading input
// J + e (e the tap's offset); every division is a precomputed multiply-shift.
// Otherwise a 64-bit form tests every tap.
//
// For output position o on an axis with stride s, dilation d and begin pad pb,
// tap k contributes iff (o + pb - k*d) is a non-negative multiple of s, and
// it reads input position i = (o + pb - k*d) / s (ai.onnx.ConvTranspose
// README, "Description": the scatter o = i*s - pb + k*d read backwards).
#include <algorithm>

#include "ct_divmagic.h"
#include "ct_internal.h"

namespace ct {
namespace {

struct GenericArgs {
    int64_t N, C, M, Cg, Mg;
    int64_t in[3], k[3], s[3], d[3], pb[3], out[3];
    int64_t total;
    int nhwc;
    int has_bias;
    int act;
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
        y[idx] = from_f<T>(apply_act(acc, a.act));
    }
}

constexpr int kG32MaxS = 64;      // phases per axis
constexpr int kG32MaxTaps = 64;   // taps per axis

struct Generic32Args {
    int32_t C, M, Cg, Mg, in_sz, k_sz, total, nhwc, has_bias, act;
    int32_t in[3], out[3], s[3], kst[3];     // kpos = k0*kst[0] + k1*kst[1] + k2*kst[2]
    DivMagic d_out[3], d_M, d_Mg, d_s[3];
    uint8_t ph_off[3][kG32MaxS], ph_cnt[3][kG32MaxS];   // taps of phase r of axis a
    int16_t tap_e[3][kG32MaxTaps], tap_k[3][kG32MaxTaps];
};

template <typename T>
__global__ void __launch_bounds__(256, 4) generic32_kernel(const __grid_constant__ Generic32Args a,
                                                        const T *__restrict__ x, const T *__restrict__ w,
                                                        const T *__restrict__ bias, T *__restrict__ y) {
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < a.total; idx += gridDim.x * blockDim.x) {
        // idx -> (n, m, o0, o1, o2) in the layout's order
        int rem = idx, m = 0;
        if (a.nhwc) {
            const int q = divq(rem, a.d_M);
            m = rem - q * a.M;
            rem = q;
        }
        int q = divq(rem, a.d_out[2]);
        const int o2 = rem - q * a.out[2];
        rem = q;
        q = divq(rem, a.d_out[1]);
        const int o1 = rem - q * a.out[1];
        rem = q;
        q = divq(rem, a.d_out[0]);
        const int o0 = rem - q * a.out[0];
        rem = q;
        if (!a.nhwc) {
            q = divq(rem, a.d_M);
            m = rem - q * a.M;
            rem = q;
        }
        const int n = rem;
        const int g = divq(m, a.d_Mg), ml = m - g * a.Mg;
        // o = s*J + r on every axis
        const int J0 = divq(o0, a.d_s[0]), r0 = o0 - J0 * a.s[0];
        const int J1 = divq(o1, a.d_s[1]), r1 = o1 - J1 * a.s[1];
        const int J2 = divq(o2, a.d_s[2]), r2 = o2 - J2 * a.s[2];
        float acc = 0.f;
        const int q0b = a.ph_off[0][r0], q0e = q0b + a.ph_cnt[0][r0];
        const int q1b = a.ph_off[1][r1], q1e = q1b + a.ph_cnt[1][r1];
        const int q2b = a.ph_off[2][r2], q2e = q2b + a.ph_cnt[2][r2];
        for (int q0 = q0b; q0 < q0e; ++q0) {
            const int i0 = J0 + a.tap_e[0][q0];
            if ((unsigned)i0 >= (unsigned)a.in[0]) continue;
            for (int q1 = q1b; q1 < q1e; ++q1) {
                const int i1 = J1 + a.tap_e[1][q1];
                if ((unsigned)i1 >= (unsigned)a.in[1]) continue;
                for (int q2 = q2b; q2 < q2e; ++q2) {
                    const int i2 = J2 + a.tap_e[2][q2];
                    if ((unsigned)i2 >= (unsigned)a.in[2]) continue;
                    const int ipos = (i0 * a.in[1] + i1) * a.in[2] + i2;
                    const int kpos = a.tap_k[0][q0] * a.kst[0] + a.tap_k[1][q1] * a.kst[1] + a.tap_k[2][q2] * a.kst[2];
                    const int c0 = g * a.Cg;
                    if (a.nhwc) {
                        const T *xp = x + (n * a.in_sz + ipos) * a.C + c0;
                        const T *wp = w + (c0 * a.k_sz + kpos) * a.Mg + ml;
                        for (int cl = 0; cl < a.Cg; ++cl)
                            acc = fmaf(to_f(xp[cl]), to_f(wp[cl * a.k_sz * a.Mg]), acc);
                    } else {
                        const T *xp = x + (n * a.C + c0) * a.in_sz + ipos;
                        const T *wp = w + (c0 * a.Mg + ml) * a.k_sz + kpos;
                        for (int cl = 0; cl < a.Cg; ++cl)
                            acc = fmaf(to_f(xp[cl * a.in_sz]), to_f(wp[cl * a.Mg * a.k_sz]), acc);
                    }
                }
            }
        }
        if (a.has_bias) acc += to_f(bias[m]);
        y[idx] = from_f<T>(apply_act(acc, a.act));
    }
}

// The 32-bit form's arguments; false when an index or table would not fit.
bool generic32_setup(const Plan &p, Generic32Args &a) {
    const int64_t lim = (int64_t)1 << 31;
    const int64_t total = p.N * p.M * numel_out(p);
    if (!p.tabled || total >= lim || p.N * p.C * numel_in(p) >= lim || p.C * p.Mg * numel_k(p) >= lim) return false;
    a = Generic32Args();
    a.C = (int32_t)p.C;
    a.M = (int32_t)p.M;
    a.Cg = (int32_t)p.Cg;
    a.Mg = (int32_t)p.Mg;
    a.in_sz = (int32_t)numel_in(p);
    a.k_sz = (int32_t)numel_k(p);
    a.total = (int32_t)total;
    a.nhwc = p.layout == CT_NHWC;
    a.has_bias = p.has_bias;
    a.act = p.act;
    a.kst[2] = 1;
    a.kst[1] = (int32_t)p.k[2];
    a.kst[0] = (int32_t)(p.k[1] * p.k[2]);
    for (int ax = 0; ax < 3; ++ax) {
        if (p.s[ax] > kG32MaxS || p.k[ax] > kG32MaxTaps || p.out[ax] < 1) return false;
        a.in[ax] = (int32_t)p.in[ax];
        a.out[ax] = (int32_t)p.out[ax];
        a.s[ax] = (int32_t)p.s[ax];
        a.d_out[ax] = make_magic((uint32_t)p.out[ax]);
        a.d_s[ax] = make_magic((uint32_t)p.s[ax]);
        int t = 0;
        for (int r = 0; r < p.s[ax]; ++r) {
            a.ph_off[ax][r] = (uint8_t)t;
            for (const Tap &tp : p.taps[ax][r]) {
                if (t >= kG32MaxTaps || tp.e < -32768 || tp.e > 32767) return false;
                a.tap_e[ax][t] = (int16_t)tp.e;
                a.tap_k[ax][t] = (int16_t)tp.k;
                ++t;
            }
            a.ph_cnt[ax][r] = (uint8_t)(t - a.ph_off[ax][r]);
        }
    }
    a.d_M = make_magic((uint32_t)std::max<int64_t>(1, p.M));
    a.d_Mg = make_magic((uint32_t)std::max<int64_t>(1, p.Mg));
    return true;
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
    a.act = p.act;
    if (a.total == 0) return CT_OK;
    const int threads = 256;
    {
        Generic32Args b;
        if (generic32_setup(p, b)) {
            int64_t blocks32 = ceil_div(b.total, threads);
            if (blocks32 > 148 * 64) blocks32 = 148 * 64;
            if (p.dtype == CT_F16)
                generic32_kernel<__half><<<(unsigned)blocks32, threads, 0, st>>>(
                    b, (const __half *)x, (const __half *)wp, (const __half *)bias, (__half *)y);
            else
                generic32_kernel<float><<<(unsigned)blocks32, threads, 0, st>>>(
                    b, (const float *)x, (const float *)wp, (const float *)bias, (float *)y);
            return launch_status();
        }
    }
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
