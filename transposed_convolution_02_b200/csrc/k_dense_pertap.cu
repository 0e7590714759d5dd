// Dense fp16 ConvTranspose (group 1) as stride-phase implicit GEMMs on the
// sm_100a tensor cores (tcgen05, fp32 accumulators in TMEM): the general
// per-tap variant, one TMA load of the input window per (tap, channel block).
// It serves every dense fp16 shape; the halo variant (k_dense_halo.cu) is
// faster where its tile geometry applies.
//
// Every output position o = s*J + r (per axis: r the stride phase, J the
// position inside the phase) receives exactly the taps k of its phase, and
// tap k reads input position i = J + e with e = (r + pad_begin - k*d) / s.
// So each phase is a stride-1 correlation of the input with the phase's
// taps, in reversed tap order (ai.onnx.ConvTranspose README, implementation
// notes: the stride-1 case is a forward convolution with tap-reversed
// weights; the grouped stride-phase variant generalises it per phase).
// Per phase it is a GEMM over pixels (J) x output channels (m) with the
// reduction over (tap, input channel):
//
//     D[J, m] = sum_{tap, c} X[c, J + e_tap] * W[c, m, k_tap]
//
// Here the pixels sit on the MMA's M side (128 TMEM lanes) and the output
// channels on its N side.  The A operand (128 pixels x 64 channels) is one
// TMA tile load of the channels-last input at the tap's signed offset, so
// padding and borders come from TMA's zero fill and no column matrix
// exists.  The B operand is the pre-packed weight of (phase, tap, channel
// block).  A CTA owns a tile of 128 J positions for a group of phases whose
// accumulators fit in half of TMEM, so the epilogue of one tile overlaps the
// MMAs of the next.  Warp roles: warp 0 issues TMA, warp 1 issues MMAs,
// warps 2-5 drain TMEM, add the bias, round to fp16 and store.
//
// Channels-first input is first re-laid channels-last into the workspace.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "ct_cuda_util.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

constexpr int kMaxPairs = 256;
constexpr int kMaxPhases = 64;
constexpr int kMaxGroups = 64;
constexpr int kThreads = 192;
constexpr int kATileBytes = 128 * 64 * 2;   // 128 pixels x 64 fp16 channels

struct DenseTables {
    int32_t n_pairs, n_phases, n_groups, n_units;
    int32_t BX, BY, BZ, lbx, lby;   // tile extents in J (powers of 2), product 128
    int32_t TX, TY, TZ;             // tiles per axis
    int32_t KB, Np, stages;
    int32_t nhwc, has_bias, dead, act;
    int32_t N, C, M;
    int32_t out[3], s[3], nJ[3];
    int16_t pair_e[kMaxPairs][3];
    int16_t pair_k[kMaxPairs][3];
    int16_t phase_r[kMaxPhases][3];
    int16_t phase_pair0[kMaxPhases], phase_npair[kMaxPhases];
    int16_t group_phase0[kMaxGroups], group_nphase[kMaxGroups];
};

__device__ int g_dense_pertap_err;   // non-zero after a bounded wait ran out

const DenseTables &tables(const Plan &p) {
    return *reinterpret_cast<const DenseTables *>(p.aux.data());
}

// ---------------------------------------------------------------------------
// weight pre-pack: Wp[pair][kb][m < Np][cc < 64] = W[kb*64 + cc][m][k_pair]
// (zero outside C and M); W channels-first [C][M][k..] or channels-last
// [C][k..][M].

__global__ void __launch_bounds__(256) dense_prepack_kernel(const DenseTables T,
                                                            const __half *__restrict__ w,
                                                            __half *__restrict__ wp, int k0,
                                                            int k1, int k2, int w_nhwc) {
    const long long total = (long long)T.n_pairs * T.KB * T.Np * 64;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int cc = (int)(i & 63);
        long long r = i >> 6;
        const int m = (int)(r % T.Np);
        r /= T.Np;
        const int kb = (int)(r % T.KB);
        const int pair = (int)(r / T.KB);
        const int c = kb * 64 + cc;
        __half v = __float2half(0.f);
        if (c < T.C && m < T.M) {
            const long long kpos =
                ((long long)T.pair_k[pair][0] * k1 + T.pair_k[pair][1]) * k2 + T.pair_k[pair][2];
            const long long ksz = (long long)k0 * k1 * k2;
            v = w_nhwc ? w[((long long)c * ksz + kpos) * T.M + m]
                       : w[((long long)c * T.M + m) * ksz + kpos];
        }
        wp[i] = v;
    }
}

// ---------------------------------------------------------------------------
// the phase-GEMM kernel

__global__ void __launch_bounds__(kThreads, 1)
    dense_pertap_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ DenseTables T, const __half *__restrict__ bias,
                    __half *__restrict__ y) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stages = T.stages;
    const uint32_t b_bytes = (uint32_t)T.Np * 128;
    const uint32_t b_stride = (b_bytes + 1023) & ~1023u;
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)stages * kATileBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + (size_t)stages * b_stride);
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = smem_u32(bars + stages);
    const uint32_t tfull0 = smem_u32(bars + 2 * stages);
    const uint32_t tempty0 = smem_u32(bars + 2 * stages + 2);
    const uint32_t mdone = smem_u32(bars + 2 * stages + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * stages + 5);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, 128);
        }
        mbar_init(mdone, 1);
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    int *err = &g_dense_pertap_err;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        int it = 0;
        bool ok = true;
        for (int unit = blockIdx.x; unit < T.n_units && ok; unit += gridDim.x) {
            const int g = unit % T.n_groups;
            int tile = unit / T.n_groups;
            const int tx = tile % T.TX; tile /= T.TX;
            const int ty = tile % T.TY; tile /= T.TY;
            const int tz = tile % T.TZ;
            const int n = tile / T.TZ;
            const int J0x = tx * T.BX, J0y = ty * T.BY, J0z = tz * T.BZ;
            const int ph0 = T.group_phase0[g], ph1 = ph0 + T.group_nphase[g];
            for (int ph = ph0; ph < ph1 && ok; ++ph) {
                const int q0 = T.phase_pair0[ph], q1 = q0 + T.phase_npair[ph];
                for (int q = q0; q < q1 && ok; ++q) {
                    for (int kb = 0; kb < T.KB; ++kb, ++it) {
                        const int s = it % stages;
                        const int round = it / stages;
                        if (round > 0 && !mbar_wait(empty0 + 8 * s, (round - 1) & 1, err, 1)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(full0 + 8 * s, kATileBytes + b_bytes);
                        tma_load_5d(smem_u32(sA + (size_t)s * kATileBytes), &tmA, full0 + 8 * s,
                                    kb * 64, J0x + T.pair_e[q][2], J0y + T.pair_e[q][1],
                                    J0z + T.pair_e[q][0], n);
                        tma_load_2d(smem_u32(sB + (size_t)s * b_stride), &tmB, full0 + 8 * s, 0,
                                    (q * T.KB + kb) * T.Np);
                    }
                }
            }
        }
        // the copies this thread issued must have landed before the CTA exits
        const int first = it > stages ? it - stages : 0;
        for (int j = first; j < it; ++j)
            mbar_wait(full0 + 8 * (j % stages), (j / stages) & 1, err, 2);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        const uint32_t idesc = idesc_f16_f32(128, T.Np);
        int it = 0, local = 0;
        bool ok = true;
        for (int unit = blockIdx.x; unit < T.n_units && ok; unit += gridDim.x, ++local) {
            const int g = unit % T.n_groups;
            const int buf = local & 1, use = local >> 1;
            if (use > 0 && !mbar_wait(tempty0 + 8 * buf, (use - 1) & 1, err, 3)) break;
            tc_fence_after();
            const int ph0 = T.group_phase0[g], ph1 = ph0 + T.group_nphase[g];
            for (int ph = ph0; ph < ph1 && ok; ++ph) {
                const uint32_t dcol = tmem_base + buf * 256 + (ph - ph0) * T.Np;
                const int q0 = T.phase_pair0[ph], q1 = q0 + T.phase_npair[ph];
                bool first = true;
                for (int q = q0; q < q1 && ok; ++q) {
                    for (int kb = 0; kb < T.KB; ++kb, ++it) {
                        const int s = it % stages;
                        if (!mbar_wait(full0 + 8 * s, (it / stages) & 1, err, 4)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + (size_t)s * kATileBytes));
                        const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + (size_t)s * b_stride));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16(dcol, ad + 2 * kk, bd + 2 * kk, idesc, (first && kk == 0) ? 0u : 1u);
                        first = false;
                        mma_commit(empty0 + 8 * s);
                    }
                }
            }
            mma_commit(tfull0 + 8 * buf);
        }
        // every MMA issued here is complete before TMEM is released
        mma_commit(mdone);
        mbar_wait(mdone, 0, err, 5);
    } else if (warp >= 2) {
        // ---------------- epilogue ----------------
        const int lane_base = 32 * (warp & 3);
        const int p = lane_base + lane;
        const int jx = p & (T.BX - 1);
        const int jy = (p >> T.lbx) & (T.BY - 1);
        const int jz = p >> (T.lbx + T.lby);
        int local = 0;
        for (int unit = blockIdx.x; unit < T.n_units; unit += gridDim.x, ++local) {
            const int g = unit % T.n_groups;
            int tile = unit / T.n_groups;
            const int tx = tile % T.TX; tile /= T.TX;
            const int ty = tile % T.TY; tile /= T.TY;
            const int tz = tile % T.TZ;
            const int n = tile / T.TZ;
            const int Jx = tx * T.BX + jx, Jy = ty * T.BY + jy, Jz = tz * T.BZ + jz;
            const int buf = local & 1, use = local >> 1;
            if (!mbar_wait(tfull0 + 8 * buf, use & 1, err, 6)) break;
            tc_fence_after();
            const int ph0 = T.group_phase0[g], ph1 = ph0 + T.group_nphase[g];
            for (int ph = ph0; ph < ph1; ++ph) {
                const int oz = T.s[0] * Jz + T.phase_r[ph][0];
                const int oy = T.s[1] * Jy + T.phase_r[ph][1];
                const int ox = T.s[2] * Jx + T.phase_r[ph][2];
                const bool valid = oz < T.out[0] && oy < T.out[1] && ox < T.out[2];
                const long long opos = ((long long)oz * T.out[1] + oy) * T.out[2] + ox;
                const long long plane = (long long)T.out[0] * T.out[1] * T.out[2];
                for (int m0 = 0; m0 < T.Np; m0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem_base + ((uint32_t)lane_base << 16) + buf * 256 +
                                  (ph - ph0) * T.Np + m0,
                              v);
                    tmem_ld_wait();
                    if (!valid) continue;
                    if (T.nhwc) {
                        __half *dst = y + ((long long)n * plane + opos) * T.M;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = m0 + j;
                            if (m < T.M) {
                                float a = __uint_as_float(v[j]);
                                if (T.has_bias) a += __half2float(bias[m]);
                                dst[m] = __float2half_rn(apply_act(a, T.act));
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = m0 + j;
                            if (m < T.M) {
                                float a = __uint_as_float(v[j]);
                                if (T.has_bias) a += __half2float(bias[m]);
                                y[((long long)n * T.M + m) * plane + opos] = __float2half_rn(apply_act(a, T.act));
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty0 + 8 * buf);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------------------
// host side

size_t smem_bytes(const DenseTables &T) {
    const size_t b_stride = ((size_t)T.Np * 128 + 1023) & ~(size_t)1023;
    return 1024 + (size_t)T.stages * (kATileBytes + b_stride) + (2 * T.stages + 6) * 8 + 16;
}

int ilog2(int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

}  // namespace

bool dense_pertap_supports(const Plan &p) {
    if (p.dtype != CT_F16 || p.G != 1 || !p.tabled) return false;
    if (p.C < 1 || p.C % 8 != 0 || p.M < 1 || p.M > 256 || p.N < 1) return false;
    if (p.N > 65535 || p.C > (1 << 24) || p.M * 1LL * numel_out(p) > (1LL << 40)) return false;
    for (int a = 0; a < 3; ++a)
        if (p.in[a] < 1 || p.in[a] > (1 << 24) || p.out[a] > (1 << 24) || p.s[a] > 64) return false;
    // count live phases and pairs
    int live = 0, pairs = 0;
    for (int r0 = 0; r0 < p.s[0]; ++r0)
        for (int r1 = 0; r1 < p.s[1]; ++r1)
            for (int r2 = 0; r2 < p.s[2]; ++r2) {
                const size_t t = p.taps[0][r0].size() * p.taps[1][r1].size() * p.taps[2][r2].size();
                if (t) {
                    ++live;
                    pairs += (int)t;
                }
            }
    if (live == 0 || live > kMaxPhases || pairs > kMaxPairs) return false;
    for (int a = 0; a < 3; ++a)
        for (int r = 0; r < p.s[a]; ++r)
            for (const Tap &t : p.taps[a][r])
                if (t.e < -30000 || t.e > 30000) return false;
    return true;
}

void dense_pertap_setup(Plan &p) {
    p.aux.assign((sizeof(DenseTables) + 7) / 8, 0);
    DenseTables &T = *reinterpret_cast<DenseTables *>(p.aux.data());
    T.N = (int32_t)p.N;
    T.C = (int32_t)p.C;
    T.M = (int32_t)p.M;
    T.Np = (int32_t)((p.M + 15) / 16 * 16);
    T.KB = (int32_t)ceil_div(p.C, 64);
    T.nhwc = p.layout == CT_NHWC;
    T.has_bias = p.has_bias;
    T.act = p.act;
    for (int a = 0; a < 3; ++a) {
        T.out[a] = (int32_t)p.out[a];
        T.s[a] = (int32_t)p.s[a];
        T.nJ[a] = (int32_t)ceil_div(p.out[a], p.s[a]);
    }
    // live phases in (r0, r1, r2) order, their tap pairs in reversed-tap order
    int np = 0, nq = 0, dead = 0;
    for (int r0 = 0; r0 < p.s[0]; ++r0)
        for (int r1 = 0; r1 < p.s[1]; ++r1)
            for (int r2 = 0; r2 < p.s[2]; ++r2) {
                const auto &t0 = p.taps[0][r0], &t1 = p.taps[1][r1], &t2 = p.taps[2][r2];
                if (t0.empty() || t1.empty() || t2.empty()) {
                    dead = 1;
                    continue;
                }
                T.phase_r[np][0] = (int16_t)r0;
                T.phase_r[np][1] = (int16_t)r1;
                T.phase_r[np][2] = (int16_t)r2;
                T.phase_pair0[np] = (int16_t)nq;
                for (const Tap &a : t0)
                    for (const Tap &b : t1)
                        for (const Tap &c : t2) {
                            T.pair_e[nq][0] = (int16_t)a.e;
                            T.pair_e[nq][1] = (int16_t)b.e;
                            T.pair_e[nq][2] = (int16_t)c.e;
                            T.pair_k[nq][0] = (int16_t)a.k;
                            T.pair_k[nq][1] = (int16_t)b.k;
                            T.pair_k[nq][2] = (int16_t)c.k;
                            ++nq;
                        }
                T.phase_npair[np] = (int16_t)(nq - T.phase_pair0[np]);
                ++np;
            }
    T.n_phases = np;
    T.n_pairs = nq;
    T.dead = dead;
    // groups: consecutive live phases whose accumulators fit in 256 TMEM columns,
    // kept within one (r0, r1) row of phases where possible
    const int per = 256 / T.Np;
    auto same_row = [&](int a, int b) {
        return T.phase_r[a][0] == T.phase_r[b][0] && T.phase_r[a][1] == T.phase_r[b][1];
    };
    int ng = 0;
    for (int ph = 0; ph < np;) {
        int end = ph;
        // whole rows of phases sharing (r0, r1) while they fit
        while (end < np) {
            int row_end = end + 1;
            while (row_end < np && same_row(row_end, end)) ++row_end;
            if (row_end - ph <= per)
                end = row_end;
            else
                break;
        }
        if (end == ph) {   // one row wider than a group: split it
            end = ph + 1;
            while (end < np && end - ph < per && same_row(end, ph)) ++end;
        }
        T.group_phase0[ng] = (int16_t)ph;
        T.group_nphase[ng] = (int16_t)(end - ph);
        ++ng;
        ph = end;
    }
    T.n_groups = ng;
    // tile of 128 J positions: x first, then y, then z, powers of two
    int bx = 1;
    while (bx < T.nJ[2] && bx < 128) bx *= 2;
    int rem = 128 / bx;
    int by = 1;
    while (by < T.nJ[1] && by < rem) by *= 2;
    int bz = rem / by;
    T.BX = bx; T.BY = by; T.BZ = bz;
    T.lbx = ilog2(bx); T.lby = ilog2(by);
    T.TX = (int32_t)ceil_div(T.nJ[2], bx);
    T.TY = (int32_t)ceil_div(T.nJ[1], by);
    T.TZ = (int32_t)ceil_div(T.nJ[0], bz);
    T.n_units = T.N * T.TZ * T.TY * T.TX * T.n_groups;
    const size_t b_stride = ((size_t)T.Np * 128 + 1023) & ~(size_t)1023;
    int st = (int)((227 * 1024 - 4096) / (kATileBytes + b_stride));
    T.stages = st > 6 ? 6 : st;
    p.launches = 1 + (p.layout == CT_NCHW ? 1 : 0) + (dead ? 1 : 0);
}

size_t dense_pertap_packed_bytes(const Plan &p) {
    const DenseTables &T = tables(p);
    return (size_t)T.n_pairs * T.KB * T.Np * 64 * 2;
}

size_t dense_pertap_ws_bytes(const Plan &p) {
    if (p.layout == CT_NHWC) return 0;
    return (size_t)p.N * numel_in(p) * p.C * 2;
}

ct_status dense_pertap_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const DenseTables &T = tables(p);
    const long long total = (long long)T.n_pairs * T.KB * T.Np * 64;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    dense_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(T, (const __half *)w, (__half *)wp,
                                                          (int)p.k[0], (int)p.k[1], (int)p.k[2],
                                                          p.layout == CT_NHWC);
    return launch_status();
}

ct_status dense_pertap_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                       void *ws, cudaStream_t st, int parts) {
    const DenseTables &T = tables(p);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CT_ERR_DEVICE;
    const void *xa = x;
    if (p.layout == CT_NCHW) {
        if (parts & CT_PART_PREPARE) {
            ct_status s1 = launch_nchw_to_nhwc_f16(p, x, ws, st);
            if (s1 != CT_OK) return s1;
        }
        xa = ws;
    }
    CUtensorMap tmA, tmB;
    {
        const cuuint64_t dims[5] = {(cuuint64_t)p.C, (cuuint64_t)p.in[2], (cuuint64_t)p.in[1],
                                    (cuuint64_t)p.in[0], (cuuint64_t)p.N};
        const cuuint64_t c2 = (cuuint64_t)p.C * 2;
        const cuuint64_t strides[4] = {c2, c2 * p.in[2], c2 * p.in[2] * p.in[1],
                                       c2 * p.in[2] * p.in[1] * p.in[0]};
        const cuuint32_t box[5] = {64, (cuuint32_t)T.BX, (cuuint32_t)T.BY, (cuuint32_t)T.BZ, 1};
        const cuuint32_t es[5] = {1, 1, 1, 1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void *>(xa), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    {
        const cuuint64_t rows = (cuuint64_t)T.n_pairs * T.KB * T.Np;
        const cuuint64_t dims[2] = {64, rows};
        const cuuint64_t strides[1] = {128};
        const cuuint32_t box[2] = {64, (cuuint32_t)T.Np};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(wp), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    if (T.dead && (parts & CT_PART_PREPARE)) {
        ct_status s2 = launch_dead_fill(p, bias, y, st);
        if (s2 != CT_OK) return s2;
    }
    if (!(parts & CT_PART_MAIN)) return CT_OK;
    const size_t sm = smem_bytes(T);
    static std::atomic<int> attr_set[64];
    if (!allow_smem(dense_pertap_kernel, attr_set, 227 * 1024)) return CT_ERR_DEVICE;
    int grid = sm_count();
    if (grid > T.n_units) grid = T.n_units;
    dense_pertap_kernel<<<grid, kThreads, sm, st>>>(tmA, tmB, T, (const __half *)bias, (__half *)y);
    return launch_status();
}

int dense_pertap_take_error(cudaStream_t st) { return take_error_word(g_dense_pertap_err, st); }

}  // namespace ct
