// Layout helpers shared by the tensor-core kernels: the channels-first ->
// channels-last re-layout of fp16 X, and the bias fill of outputs that no
// tap reaches (their stride phase has no tap on some axis).
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

// channels-first -> channels-last re-layout of X (fp16), X[n][c][sp] -> Xt[n][sp][c].
// A CTA moves a tile of 64 channels x 128 positions: every thread first
// issues four 16-byte loads (four channel rows), the tile is transposed in
// shared memory by 8x8 blocks (ldmatrix.trans, then stmatrix), and every
// thread stores four 16-byte pieces (8 channels of one position each), so
// each position's 64 channels leave as one 128-byte run.  Chunk q of tile
// row r sits at chunk q ^ (r & 7) in both layouts, so the eight rows of an
// 8x8 block fall in distinct banks.

constexpr int kRlC = 64, kRlS = 128;

__global__ void __launch_bounds__(256) nchw_to_nhwc_kernel(const __half *__restrict__ x,
                                                           __half *__restrict__ xt, int C,
                                                           long long S) {
    __shared__ __align__(16) __half tile[kRlC][kRlS];
    sm100::griddep_launch_dependents();   // the tensor-core kernel may set up while this one runs
    const int n = blockIdx.z;
    const int c0 = blockIdx.y * kRlC;
    const long long s0 = (long long)blockIdx.x * kRlS;
    const int t = threadIdx.x;
    const bool vec = (S & 7) == 0;
    {
        // 16 threads per channel row (16 x 8 positions), 16 rows per pass
        const int cl = t >> 4, sv = t & 15;
        const long long s = s0 + sv * 8;
        uint4 v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = c0 + cl + 16 * r;
            const __half *src = x + ((long long)n * C + c) * S + s;
            if (vec && c < C && s + 8 <= S) {
                v[r] = __ldg(reinterpret_cast<const uint4 *>(src));
            } else {
                __align__(16) __half h[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) h[j] = (c < C && s + j < S) ? src[j] : __float2half(0.f);
                v[r] = *reinterpret_cast<const uint4 *>(h);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int row = cl + 16 * r;
            *reinterpret_cast<uint4 *>(&tile[row][(sv ^ (row & 7)) * 8]) = v[r];
        }
    }
    __syncthreads();
    // [64 channels][128 positions] -> [128 positions][64 channels], in place
    sm100::transpose_64x128_b16(reinterpret_cast<uint16_t *>(&tile[0][0]), t >> 5, t & 31);
    const __half *tout = &tile[0][0];
    {
        // 8 threads per position (8 x 8 channels), 32 positions per pass
        const int sl = t >> 3, cv = t & 7;
        const int c = c0 + cv * 8;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int sp = sl + 32 * r;
            const long long s = s0 + sp;
            if (s < S && c < C)
                *reinterpret_cast<uint4 *>(xt + ((long long)n * S + s) * C + c) =
                    *reinterpret_cast<const uint4 *>(tout + sp * 64 + ((cv ^ (sp & 7)) * 8));
        }
    }
}


struct FillArgs {
    int64_t N, M;
    int32_t out[3], s[3];
    uint64_t live[3];
    int32_t nhwc, has_bias, act;
};

template <typename E>
__global__ void __launch_bounds__(256) dead_fill_kernel(const FillArgs a, const E *__restrict__ bias,
                                                        E *__restrict__ y) {
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
        if (!live) y[i] = (E)apply_act(a.has_bias ? (float)bias[m] : 0.f, a.act);
    }
}

}  // namespace

ct_status launch_nchw_to_nhwc_f16(const Plan &p, const void *x, void *xt, cudaStream_t st) {
    const long long S = numel_in(p);
    if (ceil_div(p.C, kRlC) > 65535 || p.N > 65535 || ceil_div(S, kRlS) > 0x7fffffffLL) return CT_ERR_UNSUPPORTED;
    dim3 grid((unsigned)ceil_div(S, kRlS), (unsigned)ceil_div(p.C, kRlC), (unsigned)p.N);
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
    if (p.dtype == CT_F32)
        dead_fill_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(a, (const float *)bias, (float *)y);
    else
        dead_fill_kernel<__half><<<(unsigned)blocks, 256, 0, st>>>(a, (const __half *)bias, (__half *)y);
    return launch_status();
}

}  // namespace ct
