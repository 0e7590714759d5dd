// fp32 ConvTranspose (group 1) as stride-phase GEMMs on the FP32 FMA pipes.
//
// ai.onnx.ConvTranspose README, implementation notes: the exact-tiling f32
// variant keeps the register GEMM contraction and stores straight into the
// output, with no column intermediate and no gather pass.  Here every live
// stride phase r is a GEMM
//
//     Y_r[m, J] = sum_{tap, c} W[c, m, k_tap] * X[c, J + e_tap]    (+ bias[m])
//
// where output o = s*J + r and e_tap = (r + pad_begin - k*d) / s, computed by
// a register-tiled SGEMM: a CTA owns 128 output channels x 128 positions J of
// one phase, each thread an 8 x 8 block, K walked 8 (tap, channel) rows at a
// time through double-buffered shared memory.  Input rows are read at the
// tap's signed offset with bounds checks (the zero padding), weights come
// pre-packed as [phase][tap, channel][m].  CTAs of the phases of one tile run
// next to each other, so their interleaved output writes meet in L2.
#include <stdint.h>

#include <algorithm>

#include "ct_cuda_util.h"
#include "ct_internal.h"

namespace ct {
namespace {

constexpr int kFMaxPhases = 64;
constexpr int kFMaxPairs = 256;

struct F32Args {
    int32_t N, C, M, Cp, Mp;                 // Cp = C rounded to 8, Mp = M rounded to 128
    int32_t in[3], out[3], s[3], nJ[3];
    int32_t P, tiles_p, tiles_m, n_phases, nhwc, has_bias, act;
    int32_t ph_r[kFMaxPhases][3];
    int32_t ph_q0[kFMaxPhases], ph_nq[kFMaxPhases], ph_krow[kFMaxPhases];   // first pair, pairs, packed row
    int16_t q_e[kFMaxPairs][3], q_k[kFMaxPairs][3];
    int32_t k[3];
    int32_t total_rows;
};

const F32Args &fargs(const Plan &p) { return *reinterpret_cast<const F32Args *>(p.aux.data()); }

__global__ void __launch_bounds__(256, 2) fp32_gemm_kernel(const __grid_constant__ F32Args A,
                                                          const float *__restrict__ x,
                                                          const float *__restrict__ wp,
                                                          const float *__restrict__ bias,
                                                          float *__restrict__ y) {
    __shared__ __align__(16) float As[2][8][128];
    __shared__ __align__(16) float Bs[2][8][128 + 4];
    const int tid = threadIdx.x;
    int b = blockIdx.x;
    const int ph = b % A.n_phases;
    b /= A.n_phases;
    const int mt = b % A.tiles_m;
    b /= A.tiles_m;
    const int pt = b % A.tiles_p;
    const int n = b / A.tiles_p;
    const int m0 = mt * 128, p0 = pt * 128;
    const int nq = A.ph_nq[ph], q0 = A.ph_q0[ph];
    const int ksteps = nq * A.Cp / 8;
    const float *wph = wp + (size_t)A.ph_krow[ph] * A.Mp;

    // loader roles: A row lr = tid/32 (of 8), 4 consecutive m at (tid%32)*4;
    // B row lr, 4 consecutive positions at (tid%32)*4
    const int lr = tid >> 5, lc = (tid & 31) * 4;
    // decode this thread's 4 positions once
    int pj[4][3];
    bool pv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int p = p0 + lc + i;
        pv[i] = p < A.P;
        const int jx = p % A.nJ[2];
        p /= A.nJ[2];
        pj[i][2] = jx;
        pj[i][1] = p % A.nJ[1];
        pj[i][0] = p / A.nJ[1];
    }
    const long long in_sz = (long long)A.in[0] * A.in[1] * A.in[2];
    // Cp is a multiple of 8, so the 8 rows of one K stage share a tap: the
    // tap changes every Cp/8 stages, and only then are the 4 positions' input
    // offsets and bounds recomputed; in between the channel advances by adds.
    const long long cstep = A.nhwc ? 1 : in_sz;          // between channels
    long long xo[4];                                     // element offset of channel 0 at this tap
    bool xok[4];
    int ql = -1, c = 0;                                  // current tap of the phase, channel of row lr
    auto set_tap = [&](int q) {
        const int e0 = A.q_e[q][0], e1 = A.q_e[q][1], e2 = A.q_e[q][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int iz = pj[i][0] + e0, iy = pj[i][1] + e1, ix = pj[i][2] + e2;
            xok[i] = pv[i] && iz >= 0 && iz < A.in[0] && iy >= 0 && iy < A.in[1] && ix >= 0 && ix < A.in[2];
            const long long pos = xok[i] ? ((long long)iz * A.in[1] + iy) * A.in[2] + ix : 0;
            xo[i] = A.nhwc ? ((long long)n * in_sz + pos) * A.C : (long long)n * A.C * in_sz + pos;
        }
    };
    const float *wrow = wph + (size_t)lr * A.Mp + m0 + lc;   // this thread's W row of stage 0
    // the next stage's operands into registers; stages are visited in order
    auto load_tile = [&](float4 &ra, float (&rb)[4]) {
        if (c == 0 || ql < 0) {   // stage 0 of a tap
            ++ql;
            set_tap(q0 + ql);
            c = lr;
        }
        ra = *reinterpret_cast<const float4 *>(wrow);
        wrow += (size_t)8 * A.Mp;
        const bool cok = c < A.C;
#pragma unroll
        for (int i = 0; i < 4; ++i) rb[i] = (cok && xok[i]) ? x[xo[i] + (long long)c * cstep] : 0.f;
        c += 8;
        if (c >= A.Cp) c = 0;   // the next stage starts the next tap
    };

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    float4 ra;
    float rb[4];
    if (ksteps > 0) {
        load_tile(ra, rb);
        *reinterpret_cast<float4 *>(&As[0][lr][lc]) = ra;
#pragma unroll
        for (int i = 0; i < 4; ++i) Bs[0][lr][lc + i] = rb[i];
    }
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    for (int ks = 0; ks < ksteps; ++ks) {
        const int cur = ks & 1;
        if (ks + 1 < ksteps) load_tile(ra, rb);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[cur][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[cur][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[cur][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[cur][kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (ks + 1 < ksteps) {
            *reinterpret_cast<float4 *>(&As[cur ^ 1][lr][lc]) = ra;
#pragma unroll
            for (int i = 0; i < 4; ++i) Bs[cur ^ 1][lr][lc + i] = rb[i];
        }
        __syncthreads();
    }

    // epilogue: output o = s*J + r, bias added once
    const long long plane = (long long)A.out[0] * A.out[1] * A.out[2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int p = p0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
        if (p >= A.P) continue;
        const int jx = p % A.nJ[2];
        p /= A.nJ[2];
        const int jy = p % A.nJ[1], jz = p / A.nJ[1];
        const int oz = A.s[0] * jz + A.ph_r[ph][0];
        const int oy = A.s[1] * jy + A.ph_r[ph][1];
        const int ox = A.s[2] * jx + A.ph_r[ph][2];
        if (oz >= A.out[0] || oy >= A.out[1] || ox >= A.out[2]) continue;
        const long long opos = ((long long)oz * A.out[1] + oy) * A.out[2] + ox;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
            if (m >= A.M) continue;
            const float v = apply_act(acc[i][j] + (A.has_bias ? bias[m] : 0.f), A.act);
            if (A.nhwc)
                y[((long long)n * plane + opos) * A.M + m] = v;
            else
                y[((long long)n * A.M + m) * plane + opos] = v;
        }
    }
}

// weight pre-pack: Wp[row = phase K row][m < Mp], row = (tap of the phase, channel < Cp)
__global__ void __launch_bounds__(256) fp32_prepack_kernel(const __grid_constant__ F32Args A,
                                                           const float *__restrict__ w,
                                                           float *__restrict__ wp, int w_nhwc) {
    const long long total = (long long)A.total_rows * A.Mp;
    const long long ksz = (long long)A.k[0] * A.k[1] * A.k[2];
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i % A.Mp);
        const int row = (int)(i / A.Mp);
        int ph = 0;
        while (ph + 1 < A.n_phases && row >= A.ph_krow[ph + 1]) ++ph;
        const int kr = row - A.ph_krow[ph];
        const int ql = kr / A.Cp, c = kr - ql * A.Cp;
        const int q = A.ph_q0[ph] + ql;
        float v = 0.f;
        if (c < A.C && m < A.M) {
            const long long kpos = ((long long)A.q_k[q][0] * A.k[1] + A.q_k[q][1]) * A.k[2] + A.q_k[q][2];
            v = w_nhwc ? w[((long long)c * ksz + kpos) * A.M + m] : w[((long long)c * A.M + m) * ksz + kpos];
        }
        wp[i] = v;
    }
}

// bias (or zero) for outputs whose stride phase receives no tap (fp32)
__global__ void __launch_bounds__(256) fp32_dead_fill_kernel(const __grid_constant__ F32Args A,
                                                             const uint64_t m0, const uint64_t m1,
                                                             const uint64_t m2, const float *__restrict__ bias,
                                                             float *__restrict__ y) {
    const long long plane = (long long)A.out[0] * A.out[1] * A.out[2];
    const long long total = (long long)A.N * A.M * plane;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        long long rem = i;
        int m, o0, o1, o2;
        if (A.nhwc) {
            m = (int)(rem % A.M); rem /= A.M;
            o2 = (int)(rem % A.out[2]); rem /= A.out[2];
            o1 = (int)(rem % A.out[1]); rem /= A.out[1];
            o0 = (int)(rem % A.out[0]);
        } else {
            o2 = (int)(rem % A.out[2]); rem /= A.out[2];
            o1 = (int)(rem % A.out[1]); rem /= A.out[1];
            o0 = (int)(rem % A.out[0]); rem /= A.out[0];
            m = (int)(rem % A.M);
        }
        const bool live = ((m0 >> (o0 % A.s[0])) & 1) && ((m1 >> (o1 % A.s[1])) & 1) && ((m2 >> (o2 % A.s[2])) & 1);
        if (!live) y[i] = apply_act(A.has_bias ? bias[m] : 0.f, A.act);
    }
}

}  // namespace

void fp32_setup(const Plan &p, F32Args &A);

bool fp32_gemm_supports(const Plan &p) {
    if (p.dtype != CT_F32 || p.G != 1 || !p.tabled) return false;
    if (p.C < 1 || p.M < 1 || p.N < 1) return false;
    for (int a = 0; a < 3; ++a)
        if (p.in[a] < 1 || p.out[a] > (1 << 28)) return false;
    int np = 0, nq = 0;
    for (int r0 = 0; r0 < p.s[0]; ++r0)
        for (int r1 = 0; r1 < p.s[1]; ++r1)
            for (int r2 = 0; r2 < p.s[2]; ++r2) {
                const size_t t = p.taps[0][r0].size() * p.taps[1][r1].size() * p.taps[2][r2].size();
                if (t) {
                    ++np;
                    nq += (int)t;
                }
            }
    if (np == 0 || np > kFMaxPhases || nq > kFMaxPairs) return false;
    F32Args *A = new F32Args();
    fp32_setup(p, *A);
    const long long grid = (long long)A->n_phases * A->tiles_m * A->tiles_p * A->N;
    delete A;
    return grid > 0 && grid < 0x7fffffffLL;
}

void fp32_setup(const Plan &p, F32Args &A) {
    A = F32Args();
    A.N = (int32_t)p.N;
    A.C = (int32_t)p.C;
    A.M = (int32_t)p.M;
    A.Cp = (int32_t)((p.C + 7) / 8 * 8);
    A.Mp = (int32_t)((p.M + 127) / 128 * 128);
    for (int a = 0; a < 3; ++a) {
        A.in[a] = (int32_t)p.in[a];
        A.out[a] = (int32_t)p.out[a];
        A.s[a] = (int32_t)p.s[a];
        A.nJ[a] = (int32_t)ceil_div(p.out[a], p.s[a]);
        A.k[a] = (int32_t)p.k[a];
    }
    A.nhwc = p.layout == CT_NHWC;
    A.has_bias = p.has_bias;
    A.act = p.act;
    int np = 0, nq = 0, krow = 0;
    for (int r0 = 0; r0 < p.s[0]; ++r0)
        for (int r1 = 0; r1 < p.s[1]; ++r1)
            for (int r2 = 0; r2 < p.s[2]; ++r2) {
                const auto &t0 = p.taps[0][r0], &t1 = p.taps[1][r1], &t2 = p.taps[2][r2];
                if (t0.empty() || t1.empty() || t2.empty()) continue;
                A.ph_r[np][0] = r0;
                A.ph_r[np][1] = r1;
                A.ph_r[np][2] = r2;
                A.ph_q0[np] = nq;
                A.ph_krow[np] = krow;
                for (const Tap &a : t0)
                    for (const Tap &b : t1)
                        for (const Tap &c : t2) {
                            A.q_e[nq][0] = (int16_t)a.e;
                            A.q_e[nq][1] = (int16_t)b.e;
                            A.q_e[nq][2] = (int16_t)c.e;
                            A.q_k[nq][0] = (int16_t)a.k;
                            A.q_k[nq][1] = (int16_t)b.k;
                            A.q_k[nq][2] = (int16_t)c.k;
                            ++nq;
                        }
                A.ph_nq[np] = nq - A.ph_q0[np];
                krow += A.ph_nq[np] * A.Cp;
                ++np;
            }
    A.n_phases = np;
    A.total_rows = krow;
    A.P = A.nJ[0] * A.nJ[1] * A.nJ[2];
    A.tiles_p = (int32_t)ceil_div(A.P, 128);
    A.tiles_m = A.Mp / 128;
}

void fp32_gemm_plan(Plan &p) {
    p.aux.assign((sizeof(F32Args) + 7) / 8, 0);
    fp32_setup(p, *reinterpret_cast<F32Args *>(p.aux.data()));
    p.launches = 1 + (has_dead_phases(p) ? 1 : 0);
}

size_t fp32_gemm_packed_bytes(const Plan &p) {
    const F32Args &A = fargs(p);
    return (size_t)A.total_rows * A.Mp * 4;
}

ct_status fp32_gemm_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const F32Args &A = fargs(p);
    const long long total = (long long)A.total_rows * A.Mp;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    fp32_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(A, (const float *)w, (float *)wp, p.layout == CT_NHWC);
    return launch_status();
}

ct_status fp32_gemm_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                        cudaStream_t st, int parts) {
    const F32Args &A = fargs(p);
    if (has_dead_phases(p) && (parts & CT_PART_PREPARE)) {
        uint64_t lm[3] = {0, 0, 0};
        for (int a = 0; a < 3; ++a)
            for (int r = 0; r < p.s[a] && r < 64; ++r)
                if (!p.taps[a][r].empty()) lm[a] |= 1ull << r;
        const long long total = p.N * p.M * numel_out(p);
        long long blocks = ceil_div(total, 256);
        if (blocks > 148 * 64) blocks = 148 * 64;
        fp32_dead_fill_kernel<<<(unsigned)blocks, 256, 0, st>>>(A, lm[0], lm[1], lm[2], (const float *)bias,
                                                               (float *)y);
        ct_status s1 = launch_status();
        if (s1 != CT_OK) return s1;
    }
    if (!(parts & CT_PART_MAIN)) return CT_OK;
    const long long grid = (long long)A.n_phases * A.tiles_m * A.tiles_p * A.N;
    fp32_gemm_kernel<<<(unsigned)grid, 256, 0, st>>>(A, (const float *)x, (const float *)wp, (const float *)bias,
                                                    (float *)y);
    return launch_status();
}

}  // namespace ct
