// Layout helpers shared by the tensor-core kernels: the channels-first ->
// channels-last re-layout of fp16 X, and the bias fill of outputs that no
// tap reaches (their stride phase has no tap on some axis).
#include "ct_internal.h"

namespace ct {
namespace {

// channels-first -> channels-last re-layout of X (fp16), X[n][c][sp] -> Xt[n][sp][c]

__global__ void __launch_bounds__(256) nchw_to_nhwc_kernel(const __half *__restrict__ x,
                                                           __half *__restrict__ xt, int C,
                                                           long long S) {
    __shared__ __half tile[32][66];
    const int n = blockIdx.z;
    const int c0 = blockIdx.y * 32;
    const long long s0 = (long long)blockIdx.x * 64;
    const int t = threadIdx.x;
    {
        const int cl = t >> 3, sv = t & 7;
        const int c = c0 + cl;
        const long long s = s0 + sv * 8;
        const __half *src = x + ((long long)n * C + c) * S + s;
        if (c < C && (S & 7) == 0 && s + 8 <= S) {
            uint4 v = *reinterpret_cast<const uint4 *>(src);
            const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<__half2 *>(&tile[cl][sv * 8 + 2 * j]) = h[j];
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                tile[cl][sv * 8 + j] = (c < C && s + j < S) ? src[j] : __float2half(0.f);
        }
    }
    __syncthreads();
    {
        const int sl = t >> 2, cv = t & 3;
        const long long s = s0 + sl;
        const int c = c0 + cv * 8;
        if (s < S && c < C) {
            __align__(16) __half v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = tile[cv * 8 + j][sl];
            *reinterpret_cast<uint4 *>(xt + ((long long)n * S + s) * C + c) =
                *reinterpret_cast<const uint4 *>(v);
        }
    }
}


struct FillArgs {
    int64_t N, M;
    int32_t out[3], s[3];
    uint64_t live[3];
    int32_t nhwc, has_bias, act;
};

__global__ void __launch_bounds__(256) dead_fill_kernel(const FillArgs a,
                                                        const __half *__restrict__ bias,
                                                        __half *__restrict__ y) {
    const long long per_img = (long long)a.out[0] * a.out[1] * a.out[2];
    const long long total = a.N * a.M * per_img;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        long long rem = i;
        int m, o0, o1, o2;
        if (a.nhwc) {
            m = (int)(rem % a.M); rem /= a.M;
            o2 = (int)(rem % a.out[2]); rem /= a.out[2];
            o1 = (int)(rem % a.out[1]); rem /= a.out[1];
            o0 = (int)(rem % a.out[0]);
        } else {
            o2 = (int)(rem % a.out[2]); rem /= a.out[2];
            o1 = (int)(rem % a.out[1]); rem /= a.out[1];
            o0 = (int)(rem % a.out[0]); rem /= a.out[0];
            m = (int)(rem % a.M);
        }
        const bool live = ((a.live[0] >> (o0 % a.s[0])) & 1) && ((a.live[1] >> (o1 % a.s[1])) & 1) &&
                          ((a.live[2] >> (o2 % a.s[2])) & 1);
        if (!live) y[i] = __float2half_rn(apply_act(a.has_bias ? __half2float(bias[m]) : 0.f, a.act));
    }
}

}  // namespace

ct_status launch_nchw_to_nhwc_f16(const Plan &p, const void *x, void *xt, cudaStream_t st) {
    const long long S = numel_in(p);
    dim3 grid((unsigned)ceil_div(S, 64), (unsigned)ceil_div(p.C, 32), (unsigned)p.N);
    nchw_to_nhwc_kernel<<<grid, 256, 0, st>>>((const __half *)x, (__half *)xt, (int)p.C, S);
    return launch_status();
}

bool has_dead_phases(const Plan &p) {
    for (int a = 0; a < 3; ++a)
        for (int r = 0; r < p.s[a]; ++r)
            if (p.taps[a][r].empty()) return true;
    return false;
}

ct_status launch_dead_fill(const Plan &p, const void *bias, void *y, cudaStream_t st) {
    FillArgs a;
    a.N = p.N;
    a.M = p.M;
    for (int i = 0; i < 3; ++i) {
        a.out[i] = (int32_t)p.out[i];
        a.s[i] = (int32_t)p.s[i];
        a.live[i] = 0;
        for (int r = 0; r < p.s[i] && r < 64; ++r)
            if (!p.taps[i][r].empty()) a.live[i] |= 1ull << r;
    }
    a.nhwc = p.layout == CT_NHWC;
    a.has_bias = p.has_bias;
    a.act = p.act;
    const long long total = p.N * p.M * numel_out(p);
    if (total == 0) return CT_OK;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 64) blocks = 148 * 64;
    dead_fill_kernel<<<(unsigned)blocks, 256, 0, st>>>(a, (const __half *)bias, (__half *)y);
    return launch_status();
}

}  // namespace ct
