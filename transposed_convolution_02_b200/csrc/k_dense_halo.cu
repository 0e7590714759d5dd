// Dense fp16 ConvTranspose (group 1) on the sm_100a tensor cores, halo
// variant: the stride-phase implicit GEMMs of k_dense_pertap.cu with operand
// reuse sized for B200's shared-memory fill rate.
//
// Output o = s*J + r per axis (r the stride phase); tap k of phase r reads
// input i = J + e, e = (r + pad_begin - k*d) / s (ai.onnx.ConvTranspose
// README, implementation notes on the tap-reversed stride-1 form and the
// grouped stride-phase variant).  Pixels (J) sit on the MMA's M side, output
// channels on its N side, the reduction runs over (input channel, tap).
//
// Reuse:
//  * One TMA tile per (x-offset, z-offset, 64-channel block) holds the input
//    rows a whole unit needs plus the y halo; every tap with that x/z offset
//    reads it through a descriptor shifted by whole J-rows (a multiple of
//    1024 bytes, so the 128-byte swizzle phase is unchanged).
//  * (phase, tap) pairs with the same input offset whose phases own adjacent
//    TMEM accumulators run as one MMA with a wider N.
//  * A unit covers Mt tiles of 128 pixels, so each weight tile feeds Mt MMAs;
//    weights stay resident in shared memory when the whole packed weight fits.
// Warps: 0 loads input tiles, 1 issues MMAs, 2 loads weights, 4-7 drain TMEM
// (bias from shared memory, fp16 rounding, paired x phases stored as half2).
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "ct_cuda_util.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

constexpr int kMaxPhases = 64;
constexpr int kMaxGroups = 32;
constexpr int kMaxClasses = 64;
constexpr int kMaxItems = 320;
constexpr int kThreads = 256;
constexpr int kSmemBudget = 227 * 1024;

struct Item {
    int16_t e[3];       // input offset (z, y, x)
    int16_t row_shift;  // pixel rows into the class's input tile
    int16_t n;          // MMA N: run length x Np
    int16_t tcol;       // first TMEM column of the run inside the group
    int16_t phase0;     // first phase of the run (global live-phase index)
    int16_t first;      // first write of these columns (at channel block 0)
    int32_t brow;       // row offset of this item's weights inside one channel block
};

struct Class {
    int16_t ex, ez, ey_min, item0, nitems, pad;
};

struct HaloTables {
    int32_t N, C, M, Np, KB;
    int32_t out[3], s[3], nJ[3], pb[3], d[3], k[3];
    int32_t BX, R, Mt, BYh;
    int32_t TX, TY, TZ, n_units, n_groups;
    int32_t nbuf, bufcols, SA, SB, a_bytes, b_slot_bytes, BR;
    int32_t resident, res_rows;
    int32_t nhwc, has_bias, dead, pair_x;
    int32_t n_phases, n_items, n_classes;
    int32_t total_rows;
    int16_t phase_r[kMaxPhases][3];
    int16_t g_phase0[kMaxGroups], g_nphase[kMaxGroups], g_cls0[kMaxGroups], g_ncls[kMaxGroups];
    int32_t g_brow[kMaxGroups], g_rows_kb[kMaxGroups];
    Class cls[kMaxClasses];
    Item item[kMaxItems];
};

__device__ int g_dense_halo_err;

const HaloTables &tables(const Plan &p) { return *reinterpret_cast<const HaloTables *>(p.aux.data()); }

// ---------------------------------------------------------------------------
// weight pre-pack: rows of every group, channel block and item in the order
// the kernel consumes them; a row holds 64 input channels of one output
// channel m of one phase: W[kb*64 + cc][m][k], k the phase's tap at the
// item's offset, zero outside C and M.

__global__ void __launch_bounds__(256) halo_prepack_kernel(const __grid_constant__ HaloTables T,
                                                           const __half *__restrict__ w,
                                                           __half *__restrict__ wp, int w_nhwc) {
    const long long total = (long long)T.total_rows * 64;
    const long long ksz = (long long)T.k[0] * T.k[1] * T.k[2];
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int cc = (int)(i & 63);
        const int row = (int)(i >> 6);
        // find the group, channel block and item of this row
        int g = 0;
        while (g + 1 < T.n_groups && row >= T.g_brow[g + 1]) ++g;
        const int rg = row - T.g_brow[g];
        const int kb = rg / T.g_rows_kb[g];
        const int rk = rg % T.g_rows_kb[g];
        const int i0 = T.cls[T.g_cls0[g]].item0;
        const int i1 = T.cls[T.g_cls0[g] + T.g_ncls[g] - 1].item0 + T.cls[T.g_cls0[g] + T.g_ncls[g] - 1].nitems;
        int it = i0;
        while (it + 1 < i1 && rk >= T.item[it + 1].brow) ++it;
        const Item &I = T.item[it];
        const int rr = rk - I.brow;
        const int ph = I.phase0 + rr / T.Np;
        const int m = rr % T.Np;
        const int c = kb * 64 + cc;
        __half v = __float2half(0.f);
        if (c < T.C && m < T.M) {
            long long kpos = 0;
            bool ok = true;
            for (int a = 0; a < 3; ++a) {
                const int num = T.phase_r[ph][a] + T.pb[a] - I.e[a] * T.s[a];
                const int ka = num / T.d[a];
                ok = ok && (num % T.d[a] == 0) && ka >= 0 && ka < T.k[a];
                kpos = kpos * T.k[a] + ka;
            }
            if (ok)
                v = w_nhwc ? w[((long long)c * ksz + kpos) * T.M + m]
                           : w[((long long)c * T.M + m) * ksz + kpos];
        }
        wp[i] = v;
    }
}

// ---------------------------------------------------------------------------

struct Unit {
    int g, n, tz, ty, tx;
};

__device__ __forceinline__ Unit decode_unit(const HaloTables &T, int u) {
    Unit r;
    r.g = u % T.n_groups;
    int t = u / T.n_groups;
    r.tx = t % T.TX; t /= T.TX;
    r.ty = t % T.TY; t /= T.TY;
    r.tz = t % T.TZ;
    r.n = t / T.TZ;
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    dense_halo_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ HaloTables T, const __half *__restrict__ bias,
                      __half *__restrict__ y) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int SA = T.SA, SB = T.SB;
    uint8_t *sA = smem;
    uint8_t *sB = sA + (size_t)SA * T.a_bytes;       // ring slots, or the resident weights
    const size_t b_region = T.resident ? (size_t)T.res_rows * 128 : (size_t)SB * T.b_slot_bytes;
    float *bias_s = reinterpret_cast<float *>(sB + b_region);
    uint64_t *bars = reinterpret_cast<uint64_t *>(bias_s + T.Np);
    const uint32_t fullA = smem_u32(bars), emptyA = smem_u32(bars + SA);
    const uint32_t fullB = smem_u32(bars + 2 * SA), emptyB = smem_u32(bars + 2 * SA + SB);
    const uint32_t tfull = smem_u32(bars + 2 * SA + 2 * SB);
    const uint32_t tempty = tfull + 16;
    const uint32_t bres = tfull + 32, mdone = tfull + 40;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * SA + 2 * SB + 6);
    int *err = &g_dense_halo_err;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(fullA + 8 * s, 1);
            mbar_init(emptyA + 8 * s, 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(fullB + 8 * s, 1);
            mbar_init(emptyB + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + 8 * b, 1);
            mbar_init(tempty + 8 * b, 128);
        }
        mbar_init(bres, 1);
        mbar_init(mdone, 1);
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp >= 4) {
        for (int m = threadIdx.x - 128; m < T.Np; m += 128)
            bias_s[m] = (T.has_bias && m < T.M) ? __half2float(bias[m]) : 0.f;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- input tiles ----------------
        int ia = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < T.n_units && ok; u += gridDim.x) {
            const Unit U = decode_unit(T, u);
            const int J0x = U.tx * T.BX, J0y = U.ty * T.Mt * T.R, J0z = U.tz;
            for (int kb = 0; kb < T.KB && ok; ++kb) {
                for (int c = T.g_cls0[U.g]; c < T.g_cls0[U.g] + T.g_ncls[U.g]; ++c, ++ia) {
                    const int s = ia % SA;
                    if (ia >= SA && !mbar_wait(emptyA + 8 * s, ((ia / SA) - 1) & 1, err, 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(fullA + 8 * s, T.a_bytes);
                    tma_load_5d(smem_u32(sA + (size_t)s * T.a_bytes), &tmA, fullA + 8 * s, kb * 64,
                                J0x + T.cls[c].ex, J0y + T.cls[c].ey_min, J0z + T.cls[c].ez, U.n);
                }
            }
        }
        const int first = ia > SA ? ia - SA : 0;
        for (int j = first; j < ia; ++j) mbar_wait(fullA + 8 * (j % SA), (j / SA) & 1, err, 2);
    } else if (warp == 2 && lane == 0) {
        // ---------------- weight tiles ----------------
        if (T.resident) {
            mbar_arrive_expect_tx(bres, (uint32_t)T.res_rows * 128);
            for (int r = 0; r < T.res_rows; r += T.BR)
                tma_load_2d(smem_u32(sB + (size_t)r * 128), &tmB, bres, 0, r);
            mbar_wait(bres, 0, err, 3);
        } else {
            int ib = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < T.n_units && ok; u += gridDim.x) {
                const Unit U = decode_unit(T, u);
                for (int kb = 0; kb < T.KB && ok; ++kb) {
                    const int c0 = T.g_cls0[U.g];
                    const int i0 = T.cls[c0].item0;
                    const int i1 = T.cls[c0 + T.g_ncls[U.g] - 1].item0 + T.cls[c0 + T.g_ncls[U.g] - 1].nitems;
                    const int rowbase = T.g_brow[U.g] + kb * T.g_rows_kb[U.g];
                    for (int it = i0; it < i1; ++it, ++ib) {
                        const int s = ib % SB;
                        if (ib >= SB && !mbar_wait(emptyB + 8 * s, ((ib / SB) - 1) & 1, err, 4)) {
                            ok = false;
                            break;
                        }
                        const int n = T.item[it].n;
                        mbar_arrive_expect_tx(fullB + 8 * s, (uint32_t)n * 128);
                        for (int r = 0; r < n; r += T.BR)
                            tma_load_2d(smem_u32(sB + (size_t)s * T.b_slot_bytes + (size_t)r * 128), &tmB,
                                        fullB + 8 * s, 0, rowbase + T.item[it].brow + r);
                    }
                }
            }
            const int first = ib > SB ? ib - SB : 0;
            for (int j = first; j < ib; ++j) mbar_wait(fullB + 8 * (j % SB), (j / SB) & 1, err, 5);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issue ----------------
        bool ok = true;
        if (T.resident) ok = mbar_wait(bres, 0, err, 6);
        int ia = 0, ib = 0, local = 0;
        for (int u = blockIdx.x; u < T.n_units && ok; u += gridDim.x, ++local) {
            const Unit U = decode_unit(T, u);
            const int buf = T.nbuf == 2 ? (local & 1) : 0;
            const int use = T.nbuf == 2 ? (local >> 1) : local;
            if (use > 0 && !mbar_wait(tempty + 8 * buf, (use - 1) & 1, err, 7)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + buf * T.bufcols;
            const int gcols = T.g_nphase[U.g] * T.Np;
            for (int kb = 0; kb < T.KB && ok; ++kb) {
                for (int c = T.g_cls0[U.g]; c < T.g_cls0[U.g] + T.g_ncls[U.g] && ok; ++c, ++ia) {
                    const int sa = ia % SA;
                    if (!mbar_wait(fullA + 8 * sa, (ia / SA) & 1, err, 8)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + (size_t)sa * T.a_bytes);
                    for (int it = T.cls[c].item0; it < T.cls[c].item0 + T.cls[c].nitems; ++it) {
                        const Item &I = T.item[it];
                        uint32_t b_addr;
                        int sb = 0;
                        if (T.resident) {
                            b_addr = smem_u32(sB) + (uint32_t)((kb * T.g_rows_kb[U.g] + I.brow) * 128);
                        } else {
                            sb = ib % SB;
                            if (!mbar_wait(fullB + 8 * sb, (ib / SB) & 1, err, 9)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            b_addr = smem_u32(sB + (size_t)sb * T.b_slot_bytes);
                        }
                        const uint32_t idesc = idesc_f16_f32(128, I.n);
                        const uint64_t bd = desc_kmajor_sw128(b_addr);
                        const uint32_t acc0 = (kb == 0 && I.first) ? 0u : 1u;
                        for (int mt = 0; mt < T.Mt; ++mt) {
                            const uint64_t ad =
                                desc_kmajor_sw128(a_addr + (uint32_t)((I.row_shift + mt * 128) * 128));
                            const uint32_t d = dbase + mt * gcols + I.tcol;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_f16(d, ad + 2 * kk, bd + 2 * kk, idesc, kk == 0 ? acc0 : 1u);
                        }
                        if (!T.resident) {
                            mma_commit(emptyB + 8 * sb);
                            ++ib;
                        }
                    }
                    mma_commit(emptyA + 8 * sa);
                }
            }
            mma_commit(tfull + 8 * buf);
        }
        mma_commit(mdone);
        mbar_wait(mdone, 0, err, 10);
    } else if (warp >= 4) {
        // ---------------- epilogue ----------------
        const int lane_base = 32 * (warp & 3);
        const int p = lane_base + lane;
        const long long plane = (long long)T.out[0] * T.out[1] * T.out[2];
        int local = 0;
        for (int u = blockIdx.x; u < T.n_units; u += gridDim.x, ++local) {
            const Unit U = decode_unit(T, u);
            const int buf = T.nbuf == 2 ? (local & 1) : 0;
            const int use = T.nbuf == 2 ? (local >> 1) : local;
            if (!mbar_wait(tfull + 8 * buf, use & 1, err, 11)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + ((uint32_t)lane_base << 16) + buf * T.bufcols;
            const int gcols = T.g_nphase[U.g] * T.Np;
            const int ph0 = T.g_phase0[U.g], ph1 = ph0 + T.g_nphase[U.g];
            const int Jx = U.tx * T.BX + (p % T.BX);
            const int Jz = U.tz;
            for (int mt = 0; mt < T.Mt; ++mt) {
                const int Jy = U.ty * T.Mt * T.R + mt * T.R + p / T.BX;
                for (int ph = ph0; ph < ph1;) {
                    const int oz = T.s[0] * Jz + T.phase_r[ph][0];
                    const int oy = T.s[1] * Jy + T.phase_r[ph][1];
                    const int ox = T.s[2] * Jx + T.phase_r[ph][2];
                    const bool valid = oz < T.out[0] && oy < T.out[1] && ox < T.out[2];
                    const bool pair = T.pair_x && ph + 1 < ph1 && T.phase_r[ph][2] % 2 == 0 &&
                                      T.phase_r[ph + 1][2] == T.phase_r[ph][2] + 1 &&
                                      T.phase_r[ph + 1][1] == T.phase_r[ph][1] &&
                                      T.phase_r[ph + 1][0] == T.phase_r[ph][0];
                    const long long opos = ((long long)oz * T.out[1] + oy) * T.out[2] + ox;
                    const uint32_t col0 = dbase + mt * gcols + (ph - ph0) * T.Np;
                    for (int m0 = 0; m0 < T.Np; m0 += 16) {
                        uint32_t v0[16], v1[16];
                        tmem_ld16(col0 + m0, v0);
                        if (pair) tmem_ld16(col0 + T.Np + m0, v1);
                        tmem_ld_wait();
                        if (!valid) continue;
                        if (T.nhwc) {
                            __half *dst = y + ((long long)U.n * plane + opos) * T.M + m0;
                            __align__(16) __half h[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                h[j] = __float2half_rn(__uint_as_float(v0[j]) + bias_s[m0 + j]);
                            if ((T.M & 7) == 0 && m0 + 16 <= T.M) {
                                reinterpret_cast<uint4 *>(dst)[0] = reinterpret_cast<const uint4 *>(h)[0];
                                reinterpret_cast<uint4 *>(dst)[1] = reinterpret_cast<const uint4 *>(h)[1];
                            } else {
                                for (int j = 0; j < 16 && m0 + j < T.M; ++j) dst[j] = h[j];
                            }
                            if (pair) {
                                __half *dst1 = dst + T.M;   // x + 1
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    h[j] = __float2half_rn(__uint_as_float(v1[j]) + bias_s[m0 + j]);
                                if ((T.M & 7) == 0 && m0 + 16 <= T.M) {
                                    reinterpret_cast<uint4 *>(dst1)[0] = reinterpret_cast<const uint4 *>(h)[0];
                                    reinterpret_cast<uint4 *>(dst1)[1] = reinterpret_cast<const uint4 *>(h)[1];
                                } else {
                                    for (int j = 0; j < 16 && m0 + j < T.M; ++j) dst1[j] = h[j];
                                }
                            }
                        } else {
                            __half *dst = y + ((long long)U.n * T.M + m0) * plane + opos;
                            if (pair) {
#pragma unroll
                                for (int j = 0; j < 16; ++j) {
                                    if (m0 + j < T.M)
                                        *reinterpret_cast<__half2 *>(dst + j * plane) =
                                            __floats2half2_rn(__uint_as_float(v0[j]) + bias_s[m0 + j],
                                                              __uint_as_float(v1[j]) + bias_s[m0 + j]);
                                }
                            } else {
#pragma unroll
                                for (int j = 0; j < 16; ++j) {
                                    if (m0 + j < T.M)
                                        dst[j * plane] =
                                            __float2half_rn(__uint_as_float(v0[j]) + bias_s[m0 + j]);
                                }
                            }
                        }
                    }
                    ph += pair ? 2 : 1;
                }
            }
            tc_fence_before();
            mbar_arrive(tempty + 8 * buf);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

size_t smem_bytes(const HaloTables &T) {
    const size_t b_region = T.resident ? (size_t)T.res_rows * 128 : (size_t)T.SB * T.b_slot_bytes;
    return 1024 + (size_t)T.SA * T.a_bytes + b_region + (size_t)T.Np * 4 +
           (size_t)(2 * T.SA + 2 * T.SB + 6) * 8 + 16;
}

int ilog2(int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

// Build groups, classes and items for a given group policy.  Returns false if
// a table limit is exceeded.
bool build_tables(const Plan &p, HaloTables &T, int Mt_pref, bool single_row_groups) {
    T.N = (int32_t)p.N;
    T.C = (int32_t)p.C;
    T.M = (int32_t)p.M;
    T.Np = (int32_t)((p.M + 15) / 16 * 16);
    T.KB = (int32_t)ceil_div(p.C, 64);
    T.nhwc = p.layout == CT_NHWC;
    T.has_bias = p.has_bias;
    for (int a = 0; a < 3; ++a) {
        T.out[a] = (int32_t)p.out[a];
        T.s[a] = (int32_t)p.s[a];
        T.nJ[a] = (int32_t)ceil_div(p.out[a], p.s[a]);
        T.pb[a] = (int32_t)p.pb[a];
        T.d[a] = (int32_t)p.d[a];
        T.k[a] = (int32_t)p.k[a];
    }
    T.pair_x = (p.s[2] % 2 == 0) && (p.out[2] % 2 == 0);
    // live phases
    int np = 0;
    T.dead = has_dead_phases(p);
    for (int r0 = 0; r0 < p.s[0]; ++r0)
        for (int r1 = 0; r1 < p.s[1]; ++r1)
            for (int r2 = 0; r2 < p.s[2]; ++r2) {
                if (p.taps[0][r0].empty() || p.taps[1][r1].empty() || p.taps[2][r2].empty()) continue;
                if (np >= kMaxPhases) return false;
                T.phase_r[np][0] = (int16_t)r0;
                T.phase_r[np][1] = (int16_t)r1;
                T.phase_r[np][2] = (int16_t)r2;
                ++np;
            }
    if (np == 0) return false;
    T.n_phases = np;
    // groups: whole (r0, r1) rows of phases, merged while they fit 256 columns
    const int per = 256 / T.Np;
    auto same_row = [&](int a, int b) {
        return T.phase_r[a][0] == T.phase_r[b][0] && T.phase_r[a][1] == T.phase_r[b][1];
    };
    int ng = 0;
    for (int ph = 0; ph < np;) {
        int end = ph;
        while (end < np) {
            int row_end = end + 1;
            while (row_end < np && same_row(row_end, end)) ++row_end;
            if (row_end - ph <= per && (!single_row_groups || end == ph))
                end = row_end;
            else
                break;
        }
        if (end == ph) {
            end = ph + 1;
            while (end < np && end - ph < per && same_row(end, ph)) ++end;
        }
        if (ng >= kMaxGroups) return false;
        T.g_phase0[ng] = (int16_t)ph;
        T.g_nphase[ng] = (int16_t)(end - ph);
        ++ng;
        ph = end;
    }
    T.n_groups = ng;
    // classes and items per group
    int nc = 0, ni = 0, rows_total = 0, span_max = 0;
    for (int g = 0; g < ng; ++g) {
        struct PairRec { int ph, e0, e1, e2; };
        std::vector<PairRec> pairs;
        for (int ph = T.g_phase0[g]; ph < T.g_phase0[g] + T.g_nphase[g]; ++ph) {
            const int r0 = T.phase_r[ph][0], r1 = T.phase_r[ph][1], r2 = T.phase_r[ph][2];
            for (const Tap &a : p.taps[0][r0])
                for (const Tap &b : p.taps[1][r1])
                    for (const Tap &c : p.taps[2][r2]) pairs.push_back({ph, a.e, b.e, c.e});
        }
        // distinct (ez, ex) classes
        std::vector<std::pair<int, int>> keys;
        for (auto &q : pairs) keys.push_back({q.e0, q.e2});
        std::sort(keys.begin(), keys.end());
        keys.erase(std::unique(keys.begin(), keys.end()), keys.end());
        T.g_cls0[g] = (int16_t)nc;
        T.g_ncls[g] = (int16_t)keys.size();
        std::vector<char> touched(np, 0);
        int brow = 0;
        for (auto &kx : keys) {
            if (nc >= kMaxClasses) return false;
            Class &C = T.cls[nc];
            C.ez = (int16_t)kx.first;
            C.ex = (int16_t)kx.second;
            std::vector<int> eys;
            for (auto &q : pairs)
                if (q.e0 == kx.first && q.e2 == kx.second) eys.push_back(q.e1);
            std::sort(eys.begin(), eys.end());
            eys.erase(std::unique(eys.begin(), eys.end()), eys.end());
            C.ey_min = (int16_t)eys.front();
            span_max = std::max(span_max, eys.back() - eys.front());
            C.item0 = (int16_t)ni;
            for (int ey : eys) {
                std::vector<int> phs;
                for (auto &q : pairs)
                    if (q.e0 == kx.first && q.e2 == kx.second && q.e1 == ey) phs.push_back(q.ph);
                std::sort(phs.begin(), phs.end());
                // runs of consecutive phases with the same first-touch state, N <= 256
                size_t i = 0;
                while (i < phs.size()) {
                    size_t j = i + 1;
                    while (j < phs.size() && phs[j] == phs[j - 1] + 1 && touched[phs[j]] == touched[phs[i]] &&
                           (int)(j - i + 1) * T.Np <= 256)
                        ++j;
                    if (ni >= kMaxItems) return false;
                    Item &I = T.item[ni];
                    I.e[0] = (int16_t)kx.first;
                    I.e[1] = (int16_t)ey;
                    I.e[2] = (int16_t)kx.second;
                    I.row_shift = 0;   // set once BX is known
                    I.n = (int16_t)((j - i) * T.Np);
                    I.tcol = (int16_t)((phs[i] - T.g_phase0[g]) * T.Np);
                    I.phase0 = (int16_t)phs[i];
                    I.first = touched[phs[i]] ? 0 : 1;
                    I.brow = brow;
                    brow += I.n;
                    for (size_t q = i; q < j; ++q) touched[phs[q]] = 1;
                    ++ni;
                    i = j;
                }
            }
            C.nitems = (int16_t)(ni - C.item0);
            ++nc;
        }
        T.g_brow[g] = rows_total;
        T.g_rows_kb[g] = brow;
        rows_total += brow * T.KB;
    }
    T.n_classes = nc;
    T.n_items = ni;
    T.total_rows = rows_total;
    // tile geometry: BX J-columns (power of two, >= 8), R = 128 / BX J-rows per M-tile
    int bx = 8;
    while (bx < T.nJ[2] && bx < 128) bx *= 2;
    T.BX = bx;
    T.R = 128 / bx;
    int mt = Mt_pref;
    while (mt > 1 && (mt - 1) * T.R >= T.nJ[1]) --mt;   // no M-tile entirely past the rows
    T.Mt = mt;
    T.BYh = mt * T.R + span_max;
    if (T.BYh > 256) return false;
    for (int i = 0; i < ni; ++i) {
        const Class *Cp = nullptr;
        for (int c = 0; c < nc; ++c)
            if (i >= T.cls[c].item0 && i < T.cls[c].item0 + T.cls[c].nitems) Cp = &T.cls[c];
        T.item[i].row_shift = (int16_t)((T.item[i].e[1] - Cp->ey_min) * bx);
    }
    T.TX = (int32_t)ceil_div(T.nJ[2], bx);
    T.TY = (int32_t)ceil_div(T.nJ[1], (int64_t)mt * T.R);
    T.TZ = T.nJ[0];
    const long long units = (long long)T.N * T.TZ * T.TY * T.TX * T.n_groups;
    if (units > (1LL << 30)) return false;
    T.n_units = (int32_t)units;
    // TMEM: Mt x group columns per buffer, double-buffered when that fits
    int gmax = 0;
    for (int g = 0; g < ng; ++g) gmax = std::max(gmax, (int)T.g_nphase[g] * T.Np);
    T.bufcols = mt * gmax;
    if (T.bufcols > 512) return false;
    T.nbuf = T.bufcols <= 256 ? 2 : 1;
    // weight box rows: largest power of two dividing every item N (<= 256)
    int br = 256;
    for (int i = 0; i < ni; ++i)
        while (T.item[i].n % br) br /= 2;
    T.BR = br;
    int nmax = 0;
    for (int i = 0; i < ni; ++i) nmax = std::max(nmax, (int)T.item[i].n);
    T.b_slot_bytes = nmax * 128;
    T.a_bytes = bx * T.BYh * 128;
    // shared memory: resident weights if the single group's packed rows fit
    const int fixed = 1024 + T.Np * 4 + 64 * 8 + 64;
    T.resident = 0;
    T.res_rows = 0;
    if (ng == 1 && (long long)rows_total * 128 + 3LL * T.a_bytes + fixed <= kSmemBudget) {
        T.resident = 1;
        T.res_rows = rows_total;
        T.SA = (int)std::min<long long>(6, (kSmemBudget - fixed - (long long)rows_total * 128) / T.a_bytes);
        T.SB = 1;
    } else {
        // input slots first (most that still leave >= 3 weight slots), else 2 + 2
        int best_sa = 0, best_sb = 0;
        for (int sa = 6; sa >= 2 && !best_sa; --sa) {
            const long long rest = kSmemBudget - fixed - (long long)sa * T.a_bytes;
            const long long sb = rest / T.b_slot_bytes;
            if (sb >= 3) {
                best_sa = sa;
                best_sb = (int)std::min<long long>(sb, 8);
            }
        }
        if (!best_sa && 2LL * T.a_bytes + 2LL * T.b_slot_bytes + fixed <= kSmemBudget) {
            best_sa = 2;
            best_sb = 2;
        }
        if (best_sa == 0) return false;
        T.SA = best_sa;
        T.SB = best_sb;
    }
    return smem_bytes(T) <= (size_t)kSmemBudget;
}

}  // namespace

bool dense_tc_supports(const Plan &p) {
    if (p.dtype != CT_F16 || p.G != 1 || !p.tabled) return false;
    if (p.C < 1 || p.C % 8 != 0 || p.M < 1 || p.M > 256 || p.N < 1 || p.N > 65535) return false;
    for (int a = 0; a < 3; ++a)
        if (p.in[a] < 1 || p.in[a] > (1 << 24) || p.out[a] > (1 << 24)) return false;
    for (int a = 0; a < 3; ++a)
        for (int r = 0; r < p.s[a]; ++r)
            for (const Tap &t : p.taps[a][r])
                if (t.e < -30000 || t.e > 30000) return false;
    if (ceil_div(p.out[2], p.s[2]) < 8) return false;   // narrow rows: the per-tap kernel
    HaloTables *T = new HaloTables();
    const bool ok = build_tables(p, *T, 2, false);
    delete T;
    return ok;
}

void dense_tc_setup(Plan &p) {
    p.aux.assign((sizeof(HaloTables) + 7) / 8, 0);
    HaloTables &T = *reinterpret_cast<HaloTables *>(p.aux.data());
    // Mt = 2 (weights feed two pixel tiles) unless the weights are resident
    // and a single M-tile double-buffers TMEM.
    build_tables(p, T, 2, false);
    if (T.resident && T.Mt > 1) {
        HaloTables *T1 = new HaloTables();
        if (build_tables(p, *T1, 1, false) && T1->resident) T = *T1;
        delete T1;
    }
    p.launches = 1 + (p.layout == CT_NCHW ? 1 : 0) + (T.dead ? 1 : 0);
}

size_t dense_tc_packed_bytes(const Plan &p) { return (size_t)tables(p).total_rows * 128; }

size_t dense_tc_ws_bytes(const Plan &p) {
    if (p.layout == CT_NHWC) return 0;
    return (size_t)p.N * numel_in(p) * p.C * 2;
}

ct_status dense_tc_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const HaloTables &T = tables(p);
    const long long total = (long long)T.total_rows * 64;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    halo_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(T, (const __half *)w, (__half *)wp,
                                                         p.layout == CT_NHWC);
    return launch_status();
}

ct_status dense_tc_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                       void *ws, cudaStream_t st) {
    const HaloTables &T = tables(p);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CT_ERR_DEVICE;
    const void *xa = x;
    if (p.layout == CT_NCHW) {
        ct_status s1 = launch_nchw_to_nhwc_f16(p, x, ws, st);
        if (s1 != CT_OK) return s1;
        xa = ws;
    }
    CUtensorMap tmA, tmB;
    {
        const cuuint64_t dims[5] = {(cuuint64_t)p.C, (cuuint64_t)p.in[2], (cuuint64_t)p.in[1],
                                    (cuuint64_t)p.in[0], (cuuint64_t)p.N};
        const cuuint64_t c2 = (cuuint64_t)p.C * 2;
        const cuuint64_t strides[4] = {c2, c2 * p.in[2], c2 * p.in[2] * p.in[1],
                                       c2 * p.in[2] * p.in[1] * p.in[0]};
        const cuuint32_t box[5] = {64, (cuuint32_t)T.BX, (cuuint32_t)T.BYh, 1, 1};
        const cuuint32_t es[5] = {1, 1, 1, 1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void *>(xa), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    {
        const cuuint64_t dims[2] = {64, (cuuint64_t)T.total_rows};
        const cuuint64_t strides[1] = {128};
        const cuuint32_t box[2] = {64, (cuuint32_t)T.BR};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(wp), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    if (T.dead) {
        ct_status s2 = launch_dead_fill(p, bias, y, st);
        if (s2 != CT_OK) return s2;
    }
    static std::atomic<int> attr_set[64];
    if (!allow_smem(dense_halo_kernel, attr_set, kSmemBudget)) return CT_ERR_DEVICE;
    int grid = sm_count();
    if (grid > T.n_units) grid = T.n_units;
    dense_halo_kernel<<<grid, kThreads, smem_bytes(T), st>>>(tmA, tmB, T, (const __half *)bias, (__half *)y);
    return launch_status();
}

}  // namespace ct
