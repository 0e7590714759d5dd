// Grouped fp16 ConvTranspose (small per-group channel counts), rank 1-2,
// channels-first: the grouped stride-phase kernel.
//
// ai.onnx.ConvTranspose README, implementation notes: the grouped
// stride-phase variant has one invocation own output pixels and a block of
// the group's output channels, every gathered input sample feeding the whole
// block, and the group's weight slab staged once per workgroup.  Here a CTA
// owns (image n, group g, a block of output rows, all output columns, all
// M/group output channels):
//   1. the group's input rows (plus the halo the taps need) are staged in
//      shared memory channel-contiguous, 16 channels per 32-byte pixel, with
//      the two 16-byte halves swapped on alternate groups of 4 pixels so the
//      ldmatrix rows are bank-conflict free;
//   2. the packed weights of the group are staged in the mma.sync B-fragment
//      order;
//   3. an output staging block (all channels x rows x columns) is filled with
//      the bias, which is the final value of every output whose stride phase
//      receives no tap;
//   4. every live phase runs as a GEMM over (pixels) x (output channels) with
//      the reduction over (tap, input channel) on mma.sync m16n8k16 (fp16 in,
//      fp32 accumulate); each lane's ldmatrix row address applies the tap's
//      input offset, so the zero-inserted input never exists;
//   5. bias + accumulator is rounded to fp16 into the staging block, and the
//      block -- whole output rows of every channel, contiguous in Y -- goes
//      out with bulk copies (or 16-byte stores when not aligned for them).
// Output o = s*J + r (r the phase) receives the taps k with
// (r + pad_begin - k*d) divisible by s, reading input J + (r + pad_begin - k*d)/s.
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "ct_cuda_util.h"
#include "ct_internal.h"

namespace ct {
namespace {

constexpr int kGThreads = 256;
constexpr int kGMaxPhases = 16;
constexpr int kGMaxPairs = 64;
constexpr int kGSmem = 200 * 1024;

struct GroupedArgs {
    int32_t N, C, M, G, Cg, Mg, KS, NT;     // KS = Cg/16 k-steps, NT = Mg/8 n-tiles
    int32_t in_y, in_x, out_y, out_x, s_y, s_x;
    int32_t nJx, JB, SR, SW, emin_y, emin_x;  // J-rows per CTA, slab rows/width
    int32_t n_rb, n_phases, n_pairs, has_bias, bulk_ok;
    int32_t ph_ry[kGMaxPhases], ph_rx[kGMaxPhases], ph_q0[kGMaxPhases], ph_nq[kGMaxPhases];
    int16_t q_ey[kGMaxPairs], q_ex[kGMaxPairs], q_ky[kGMaxPairs], q_kx[kGMaxPairs];
    int32_t k_y, k_x;
    int32_t smem_x, smem_w, smem_stage;      // byte sizes of the three regions
    int32_t cpitch;                          // staging halves per channel (rows * out_x + pad)
};

const GroupedArgs &gargs(const Plan &p) { return *reinterpret_cast<const GroupedArgs *>(p.aux.data()); }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-channel chunk `h` (0/1) of pixel `p` inside one channel
// block of the staged input (pixels of 32 bytes, halves swapped per 4 pixels).
__device__ __forceinline__ uint32_t xoff(int p, int h) { return (uint32_t)p * 32 + 16 * (h ^ ((p >> 2) & 1)); }

template <int NT>
__global__ void __launch_bounds__(kGThreads) grouped_kernel(const __grid_constant__ GroupedArgs A,
                                                            const __half *__restrict__ x,
                                                            const uint32_t *__restrict__ wp,
                                                            const __half *__restrict__ bias,
                                                            __half *__restrict__ y) {
    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t *sx = sm;                                   // [KS][SR*SW pixels][32 B]
    uint32_t *sw = reinterpret_cast<uint32_t *>(sm + A.smem_x);   // B fragments
    __half *st = reinterpret_cast<__half *>(sm + A.smem_x + A.smem_w);   // [Mg][rows][out_x]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rb = blockIdx.x % A.n_rb;
    const int g = (blockIdx.x / A.n_rb) % A.G;
    const int n = blockIdx.x / (A.n_rb * A.G);
    const int jy0 = rb * A.JB;
    const int oy0 = jy0 * A.s_y;
    const int orows = min(A.JB * A.s_y, A.out_y - oy0);
    const int npix = A.SR * A.SW;

    // 1. input slab: rows jy0 + emin_y + [0, SR), columns emin_x + [0, SW), zero
    //    outside the input.  A task is one pixel and 8 channels: the 8 loads are
    //    coalesced across the warp (consecutive pixels), the slab store is one
    //    16-byte write.
    {
        const int halves = A.Cg / 8;
        const long long cstride = (long long)A.in_y * A.in_x;
        const __half *xg = x + ((long long)n * A.C + (long long)g * A.Cg) * cstride;
        for (int t = tid; t < halves * npix; t += kGThreads) {
            const int pix = t % npix, hc = t / npix;
            const int row = pix / A.SW, sc = pix - row * A.SW;
            const int iy = jy0 + A.emin_y + row, ix = A.emin_x + sc;
            __align__(16) __half v[8];
            if (iy >= 0 && iy < A.in_y && ix >= 0 && ix < A.in_x) {
                const __half *src = xg + (long long)(hc * 8) * cstride + (long long)iy * A.in_x + ix;
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = src[(long long)i * cstride];
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __float2half(0.f);
            }
            const int ks = hc >> 1;
            *reinterpret_cast<uint4 *>(sx + (size_t)ks * npix * 32 + xoff(pix, hc & 1)) =
                *reinterpret_cast<const uint4 *>(v);
        }
    }
    // 2. weights of the group, already in fragment order
    {
        const int words = A.n_pairs * A.KS * A.NT * 64;
        const uint32_t *src = wp + (size_t)g * words;
        for (int i = tid; i < words; i += kGThreads) sw[i] = src[i];
    }
    // 3. staging block = bias (the value of every output no tap reaches)
    const int chunk = orows * A.out_x;   // halves of one channel's rows
    {
        if ((chunk & 7) == 0 && (A.cpitch & 7) == 0) {   // 16-byte aligned channel rows
            const int per = chunk / 8;
            for (int i = tid; i < A.Mg * per; i += kGThreads) {
                const int m = i / per, e = i - m * per;
                const __half b = A.has_bias ? bias[g * A.Mg + m] : __float2half(0.f);
                const __half2 b2 = __halves2half2(b, b);
                uint4 v;
                v.x = v.y = v.z = v.w = *reinterpret_cast<const uint32_t *>(&b2);
                *reinterpret_cast<uint4 *>(st + (size_t)m * A.cpitch + 8 * e) = v;
            }
        } else {
            for (int i = tid; i < A.Mg * chunk; i += kGThreads) {
                const int m = i / chunk;
                st[(size_t)m * A.cpitch + (i - m * chunk)] = A.has_bias ? bias[g * A.Mg + m] : __float2half(0.f);
            }
        }
    }
    __syncthreads();

    // 4. live phases: pixels (jy_local, jx) of this block, 16 per m-tile
    const int gid = lane >> 2, tig = lane & 3;
    float bsum[NT][2];   // this thread's output channels' bias
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < 2; ++j)
            bsum[t][j] = A.has_bias ? __half2float(bias[g * A.Mg + t * 8 + tig * 2 + j]) : 0.f;
    const int per_phase = A.JB * A.nJx;
    const int mtiles = (per_phase + 15) / 16;
    for (int ph = 0; ph < A.n_phases; ++ph) {
        const int ry = A.ph_ry[ph], rx = A.ph_rx[ph];
        for (int mt = warp; mt < mtiles; mt += kGThreads / 32) {
            float acc[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[t][j] = 0.f;
            // this lane's ldmatrix row: pixel mt*16 + (lane & 15), channel half lane >> 4
            const int q = mt * 16 + (lane & 15);
            const int qj = min(q, per_phase - 1);
            const int jyl = qj / A.nJx, jx = qj % A.nJx;
            for (int qi = A.ph_q0[ph]; qi < A.ph_q0[ph] + A.ph_nq[ph]; ++qi) {
                const int pix = (jyl + A.q_ey[qi] - A.emin_y) * A.SW + (jx + A.q_ex[qi] - A.emin_x);
                for (int ks = 0; ks < A.KS; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    const uint32_t addr = smem_addr(sx) + (uint32_t)ks * npix * 32 + xoff(pix, lane >> 4);
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                                 : "r"(addr));
                    const uint32_t *bf = sw + ((size_t)(qi * A.KS + ks) * NT) * 64;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const uint2 b = *reinterpret_cast<const uint2 *>(bf + t * 64 + lane * 2);
                        asm volatile(
                            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                            : "+f"(acc[t][0]), "+f"(acc[t][1]), "+f"(acc[t][2]), "+f"(acc[t][3])
                            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
                    }
                }
            }
            // 5a. bias + accumulator -> fp16 into the staging block
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int qq = mt * 16 + gid + 8 * half;
                if (qq >= per_phase) continue;
                const int jyq = qq / A.nJx;
                const int jy = jy0 + jyq, jxx = qq - jyq * A.nJx;
                const int oy = A.s_y * jy + ry, ox = A.s_x * jxx + rx;
                if (oy >= A.out_y || ox >= A.out_x) continue;
                __half *o = st + (oy - oy0) * A.out_x + ox;
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        o[(size_t)(t * 8 + tig * 2 + j) * A.cpitch] =
                            __float2half_rn(acc[t][2 * half + j] + bsum[t][j]);
            }
        }
    }
    __syncthreads();

    // 5b. the staging block is whole rows of every channel: contiguous in Y
    if (A.bulk_ok) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid < A.Mg) {
            const int m = tid;
            __half *dst = y + (((long long)n * A.M + (long long)g * A.Mg + m) * A.out_y + oy0) * A.out_x;
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                         "r"(smem_addr(st + (size_t)m * A.cpitch)), "r"((uint32_t)chunk * 2)
                         : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    } else {
        for (int i = tid; i < A.Mg * chunk; i += kGThreads) {
            const int m = i / chunk, e = i % chunk;
            y[(((long long)n * A.M + (long long)g * A.Mg + m) * A.out_y + oy0) * A.out_x + e] =
                st[(size_t)m * A.cpitch + e];
        }
    }
}

// weight pre-pack into mma.sync B fragments:
// [g][pair][ks][nt][lane][2 x half2], fragment element (k, n):
//   reg r (0/1), half h (0/1): k = ks*16 + (lane & 3)*2 + h + 8*r, n = nt*8 + (lane >> 2)
__global__ void __launch_bounds__(256) grouped_prepack_kernel(const __grid_constant__ GroupedArgs A,
                                                              const __half *__restrict__ w,
                                                              __half *__restrict__ wp) {
    const long long per_g = (long long)A.n_pairs * A.KS * A.NT * 128;   // halves
    const long long total = per_g * A.G;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        long long r = i;
        const int h = (int)(r & 1); r >>= 1;
        const int reg = (int)(r & 1); r >>= 1;
        const int lane = (int)(r % 32); r /= 32;
        const int nt = (int)(r % A.NT); r /= A.NT;
        const int ks = (int)(r % A.KS); r /= A.KS;
        const int q = (int)(r % A.n_pairs);
        const int g = (int)(r / A.n_pairs);
        const int k = ks * 16 + (lane & 3) * 2 + h + 8 * reg;
        const int m = nt * 8 + (lane >> 2);
        const long long c = (long long)g * A.Cg + k;
        const long long kpos = (long long)A.q_ky[q] * A.k_x + A.q_kx[q];
        wp[i] = w[(c * A.Mg + m) * ((long long)A.k_y * A.k_x) + kpos];
    }
}

}  // namespace

void grouped_setup(const Plan &p, GroupedArgs &A);

bool grouped_supports(const Plan &p) {
    if (p.dtype != CT_F16 || p.layout != CT_NCHW || !p.tabled) return false;
    if (p.rank > 2 || p.G < 2) return false;
    if (p.Cg % 16 != 0 || p.Cg > 64 || p.Mg % 8 != 0 || p.Mg > 64) return false;
    if (p.N < 1 || p.in[1] < 1 || p.in[2] < 1) return false;
    int np = 0, nq = 0;
    for (int ry = 0; ry < p.s[1]; ++ry)
        for (int rx = 0; rx < p.s[2]; ++rx) {
            const size_t t = p.taps[1][ry].size() * p.taps[2][rx].size();
            if (t) {
                ++np;
                nq += (int)t;
            }
        }
    if (np == 0 || np > kGMaxPhases || nq > kGMaxPairs) return false;
    GroupedArgs *A = new GroupedArgs();
    grouped_setup(p, *A);
    const size_t smem = (size_t)A->smem_x + A->smem_w + A->smem_stage;
    const bool ok = smem <= (size_t)kGSmem;
    delete A;
    return ok;
}

void grouped_setup(const Plan &p, GroupedArgs &A) {
    A = GroupedArgs();
    A.N = (int32_t)p.N;
    A.C = (int32_t)p.C;
    A.M = (int32_t)p.M;
    A.G = (int32_t)p.G;
    A.Cg = (int32_t)p.Cg;
    A.Mg = (int32_t)p.Mg;
    A.KS = A.Cg / 16;
    A.NT = A.Mg / 8;
    A.in_y = (int32_t)p.in[1];
    A.in_x = (int32_t)p.in[2];
    A.out_y = (int32_t)p.out[1];
    A.out_x = (int32_t)p.out[2];
    A.s_y = (int32_t)p.s[1];
    A.s_x = (int32_t)p.s[2];
    A.k_y = (int32_t)p.k[1];
    A.k_x = (int32_t)p.k[2];
    A.has_bias = p.has_bias;
    int np = 0, nq = 0;
    int emin_y = 1 << 20, emax_y = -(1 << 20), emin_x = 1 << 20, emax_x = -(1 << 20);
    for (int ry = 0; ry < p.s[1]; ++ry)
        for (int rx = 0; rx < p.s[2]; ++rx) {
            if (p.taps[1][ry].empty() || p.taps[2][rx].empty()) continue;
            A.ph_ry[np] = ry;
            A.ph_rx[np] = rx;
            A.ph_q0[np] = nq;
            for (const Tap &ty : p.taps[1][ry])
                for (const Tap &tx : p.taps[2][rx]) {
                    A.q_ey[nq] = (int16_t)ty.e;
                    A.q_ex[nq] = (int16_t)tx.e;
                    A.q_ky[nq] = (int16_t)ty.k;
                    A.q_kx[nq] = (int16_t)tx.k;
                    emin_y = std::min(emin_y, (int)ty.e);
                    emax_y = std::max(emax_y, (int)ty.e);
                    emin_x = std::min(emin_x, (int)tx.e);
                    emax_x = std::max(emax_x, (int)tx.e);
                    ++nq;
                }
            A.ph_nq[np] = nq - A.ph_q0[np];
            ++np;
        }
    A.n_phases = np;
    A.n_pairs = nq;
    A.emin_y = emin_y;
    A.emin_x = emin_x;
    A.nJx = (int32_t)ceil_div(p.out[2], p.s[2]);
    A.SW = A.nJx + (emax_x - emin_x);
    const int nJy = (int32_t)ceil_div(p.out[1], p.s[1]);
    // J-rows per CTA: staging <= 48 KB and slab <= 48 KB, at most what the image has
    int jb = 1;
    while (jb < nJy) {
        const int nb = jb * 2;
        const long long stage = (long long)A.Mg * nb * A.s_y * A.out_x * 2;
        const long long slab = (long long)A.Cg * (nb + emax_y - emin_y) * A.SW * 2;
        if (stage > 48 * 1024 || slab > 48 * 1024) break;
        jb = nb;
    }
    A.JB = jb;
    A.SR = jb + (emax_y - emin_y);
    A.n_rb = (int32_t)ceil_div(nJy, jb);
    A.smem_x = (int32_t)(((long long)A.KS * A.SR * A.SW * 32 + 127) / 128 * 128);
    A.smem_w = A.n_pairs * A.KS * A.NT * 64 * 4;
    // channel pitch padded by 16 halves (8 banks) against staging-store conflicts
    A.cpitch = jb * A.s_y * A.out_x + 16;
    A.smem_stage = A.Mg * A.cpitch * 2;
    // bulk copies need 16-byte aligned starts and sizes for every block
    A.bulk_ok = ((A.out_x * 2) % 16 == 0) && ((long long)A.out_y * A.out_x * 2 % 16 == 0);
}

size_t grouped_packed_bytes(const Plan &p) {
    GroupedArgs A;
    grouped_setup(p, A);
    return (size_t)A.G * A.n_pairs * A.KS * A.NT * 256;
}

void grouped_plan(Plan &p) {
    p.aux.assign((sizeof(GroupedArgs) + 7) / 8, 0);
    grouped_setup(p, *reinterpret_cast<GroupedArgs *>(p.aux.data()));
    p.launches = 1;
}

ct_status grouped_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const GroupedArgs &A = gargs(p);
    const long long total = (long long)A.G * A.n_pairs * A.KS * A.NT * 128;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    grouped_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(A, (const __half *)w, (__half *)wp);
    return launch_status();
}

template <int NT>
ct_status launch_grouped(const GroupedArgs &A, const void *x, const void *wp, const void *bias, void *y,
                         size_t smem, unsigned grid, cudaStream_t st) {
    static std::atomic<int> attr_set[64];
    if (!allow_smem(grouped_kernel<NT>, attr_set, kGSmem)) return CT_ERR_DEVICE;
    grouped_kernel<NT><<<grid, kGThreads, smem, st>>>(A, (const __half *)x, (const uint32_t *)wp,
                                                      (const __half *)bias, (__half *)y);
    return launch_status();
}

ct_status grouped_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                      cudaStream_t st) {
    const GroupedArgs &A = gargs(p);
    const size_t smem = (size_t)A.smem_x + A.smem_w + A.smem_stage;
    if (smem > (size_t)kGSmem) return CT_ERR_UNSUPPORTED;
    const long long grid = (long long)A.N * A.G * A.n_rb;
    if (grid > 0x7fffffffLL) return CT_ERR_UNSUPPORTED;
    switch (A.NT) {
        case 1: return launch_grouped<1>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 2: return launch_grouped<2>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 3: return launch_grouped<3>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 4: return launch_grouped<4>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 5: return launch_grouped<5>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 6: return launch_grouped<6>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 7: return launch_grouped<7>(A, x, wp, bias, y, smem, (unsigned)grid, st);
        case 8: return launch_grouped<8>(A, x, wp, bias, y, smem, (unsigned)grid, st);
    }
    return CT_ERR_UNSUPPORTED;
}

}  // namespace ct
