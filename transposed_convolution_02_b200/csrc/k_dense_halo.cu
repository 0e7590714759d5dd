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
//  * A unit's input is ONE TMA tile per 64-channel block: a box of HX x HYb x
//    HZb input pixels (the unit's pixels plus the halo every tap needs), each
//    pixel a 128-byte row of 64 channels in the 128-byte-swizzled K-major
//    layout.  The unit's output pixels are numbered in the same pitch (HX
//    per row), so every tap is the same 128 rows shifted by a constant; the
//    MMA descriptor simply starts at that row (the swizzle follows the
//    absolute shared address, so any 128-byte row start is valid).  Lanes
//    that fall on halo columns compute values that are never stored.
//  * (phase, tap) pairs with the same input offset whose phases own adjacent
//    TMEM accumulators run as one MMA with a wider N.
//  * A unit covers Mt tiles of 128 positions, so each weight tile feeds Mt
//    MMAs; weights stay resident in shared memory when they all fit.
// Warps: 0 loads input tiles, 1 issues MMAs, 2-3 load weights, 4-7 drain TMEM
// (bias, fp16 rounding; paired x phases stored as half2 channels-first, 16
// channels as two 16-byte vectors channels-last).  More epilogue warps were
// measured slower here: the register cap of a larger block costs the 3-D
// upsample more than the extra store parallelism gains.
//
// Row mode (channels-first output with s_x = 1 or paired x phases, every
// phase live, out_x a multiple of 8): positions are numbered without halo
// columns (pitch BXt = 32, 64 or 128), one TMA box per x offset, and a unit
// is R = Mt*128/BXt whole rows.  Each epilogue warp then owns 32 consecutive
// J_x of one row: it writes the outputs of one (z phase, y phase, 32-channel
// block) as a [32 channels][s_x*32 x] tile to shared memory and one lane
// stores the tile with a TMA tensor store (parts outside Y are clipped), so
// the output leaves the SM as whole lines from the bulk-copy engine.
#include <cuda.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <cstring>
#include <vector>

#include "ct_cuda_util.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

constexpr int kMaxPhases = 64;
constexpr int kMaxGroups = 64;
constexpr int kMaxItems = 512;
constexpr int kMaxZ = 8;   // row mode: z slices of one unit's input
constexpr int kThreads = 256;
constexpr int kEpiSets = (kThreads / 32 - 4) / 4;   // epilogue warps per TMEM lane quarter
constexpr int kSmemBudget = 227 * 1024;
// row mode: per epilogue warp two output tiles of 32 channels x 64 halves
constexpr int kStageTile = 32 * 64 * 2;
constexpr int kStageBytes = (kThreads / 32 - 4) * 2 * kStageTile;

struct Item {
    int16_t e[3];       // input offset (z, y, x)
    int16_t n;          // MMA N: run length x Np
    int32_t shift;      // rows from a position to its input under this offset
    int16_t tcol;       // first TMEM column of the run inside the group
    int16_t phase0;     // first phase of the run (global live-phase index)
    int16_t first;      // first write of these columns (at channel block 0)
    int16_t pad;
    int32_t brow;       // row offset of this item's weights inside one channel block
};

struct HaloTables {
    int32_t N, C, M, Np, KB;
    int32_t out[3], s[3], nJ[3], pb[3], d[3], k[3];
    int32_t emin[3], span[3];
    int32_t BXt, HX, HYb, HZb, Mt;      // x-tile width, input-tile box, M-tiles per unit
    int32_t TX, PU, n_units, n_groups;  // x tiles, units per (n, z, x-tile) plane
    int32_t nbuf, bufcols, SA, SB, a_bytes, a_stride, b_slot_bytes, BR;
    int32_t resident, res_rows;
    int32_t rowmode, n_ex, box_rows, R;  // row mode: x-offset boxes, rows per unit
    int32_t zslices;                     // A ring entries per channel block (row mode: z slices)
    int32_t nhwc, has_bias, dead, pair_x, act;
    int32_t n_phases, n_items, total_rows;
    int16_t phase_r[kMaxPhases][3];
    int16_t g_phase0[kMaxGroups], g_nphase[kMaxGroups], g_item0[kMaxGroups], g_nitem[kMaxGroups];
    int16_t g_emin[kMaxGroups][3];      // smallest input offset of the group's taps
    // row mode: the input comes in z slices (zslices per channel block), and
    // a group's items are ordered by z offset; its items of slice z are
    // [g_zitem[g][z], g_zitem[g][z + 1]) relative to g_item0
    int16_t g_zitem[kMaxGroups][kMaxZ + 1];
    int32_t g_brow[kMaxGroups], g_rows_kb[kMaxGroups];
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
        int g = 0;
        while (g + 1 < T.n_groups && row >= T.g_brow[g + 1]) ++g;
        const int rg = row - T.g_brow[g];
        const int kb = rg / T.g_rows_kb[g];
        const int rk = rg % T.g_rows_kb[g];
        int it = T.g_item0[g];
        const int i1 = T.g_item0[g] + T.g_nitem[g];
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
// A unit: image n, output z-slice jz, x-tile tx, positions [F0, F0 + Mt*128)
// of the (y, x) plane numbered f = jy * HX + jx (jx < BXt valid), group g.
// The kernel copies every table it walks into shared memory and every scalar
// into registers at start: the parameter block is large, and re-reading it
// between the tcgen05 instructions costs constant-cache misses.

struct SItem {
    int32_t shift;
    int32_t brow;
    int16_t n, tcol, first, pad;
};
// An item as the MMA loop consumes it: descriptor offsets in 16-byte units
// (A rows from the tile start, B rows from the channel block's weights), the
// instruction descriptor, and the accumulator column with the first-write
// flag in bit 16.
struct MItem {
    uint32_t a16, b16, idesc, col_first;
};
struct SGroup {
    int32_t brow, rows_kb;
    int16_t item0, nitem, phase0, nphase;
    int16_t emin[3], pad;
};

struct Geo {
    int n_groups, PU, TX, nJz, Mt, HX;
};

struct Unit {
    int g, n, jz, tx, F0, y0;
};

__device__ __forceinline__ Unit decode_unit(const Geo &G, int u) {
    Unit r;
    r.g = u % G.n_groups;
    int t = u / G.n_groups;
    const int pu = t % G.PU;
    t /= G.PU;
    r.tx = t % G.TX;
    t /= G.TX;
    r.jz = t % G.nJz;
    r.n = t / G.nJz;
    r.F0 = pu * G.Mt * 128;
    r.y0 = r.F0 / G.HX;
    return r;
}

// The four K = 16 steps of one 64-channel block (descriptor start + 32 bytes each).
__device__ __forceinline__ void issue4(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc0) {
    sm100::mma_f16(d, ad, bd, idesc, acc0);
    sm100::mma_f16(d, ad + 2, bd + 2, idesc, 1u);
    sm100::mma_f16(d, ad + 4, bd + 4, idesc, 1u);
    sm100::mma_f16(d, ad + 6, bd + 6, idesc, 1u);
}

// 16 consecutive channels of one channels-last position: two 16-byte stores
// when the row is whole and aligned, else element by element.
template <int ACT>
__device__ __forceinline__ void store_row16(__half *dst, const uint32_t (&v)[16], const float *b, int mcount) {
    if (mcount == 16 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
        uint4 q[2];
        __half2 *h = reinterpret_cast<__half2 *>(q);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            h[j] = __floats2half2_rn(apply_act(__uint_as_float(v[2 * j]) + b[2 * j], ACT),
                                     apply_act(__uint_as_float(v[2 * j + 1]) + b[2 * j + 1], ACT));
        reinterpret_cast<uint4 *>(dst)[0] = q[0];
        reinterpret_cast<uint4 *>(dst)[1] = q[1];
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < mcount) dst[j] = __float2half_rn(apply_act(__uint_as_float(v[j]) + b[j], ACT));
    }
}

template <int ACT>
__device__ __forceinline__ void store_chunk16(__half *dst, long long stride, const uint32_t (&v)[16],
                                              const float *b, int mcount) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < mcount) dst[j * stride] = __float2half_rn(apply_act(__uint_as_float(v[j]) + b[j], ACT));
}

// ACT: the output activation (ct_activation), fixed at compile time so that
// the identity epilogue carries no per-element test.
template <int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    dense_halo_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmY, const __grid_constant__ HaloTables T,
                      const __half *__restrict__ bias, __half *__restrict__ y) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // scalars in registers
    const int SA = T.SA, SB = T.SB, KB = T.KB, Np = T.Np, M = T.M, Mt = T.Mt;
    const int n_units = T.n_units, resident = T.resident, nbuf = T.nbuf, bufcols = T.bufcols;
    const int a_stride = T.a_stride, a_bytes = T.a_bytes, b_slot = T.b_slot_bytes, BR = T.BR;
    const int res_rows = T.res_rows, BXt = T.BXt, HX = T.HX, nhwc = T.nhwc, pair_x = T.pair_x;
    const int n_items = T.n_items, n_groups = T.n_groups, n_phases = T.n_phases;
    const Geo G{T.n_groups, T.PU, T.TX, T.nJ[0], T.Mt, T.HX};
    const int rowmode = T.rowmode, n_ex = T.n_ex, box_rows = T.box_rows, zslices = T.zslices;
    // shared-memory layout
    uint8_t *sA = smem;
    uint8_t *sStage = sA + (size_t)SA * a_stride;   // row mode: output tiles, two per epilogue warp
    uint8_t *sB = sStage + (rowmode ? (size_t)kStageBytes : 0);   // ring slots, or the resident weights
    const size_t b_region = resident ? (size_t)res_rows * 128 : (size_t)SB * b_slot;
    float *bias_s = reinterpret_cast<float *>(sB + b_region);
    SItem *items_s = reinterpret_cast<SItem *>(bias_s + ((Np + 31) & ~31));   // bias padded to 32
    MItem *mitems_s = reinterpret_cast<MItem *>(items_s + n_items);
    SGroup *groups_s = reinterpret_cast<SGroup *>(mitems_s + n_items);
    int16_t *phr_s = reinterpret_cast<int16_t *>(groups_s + n_groups);
    uint64_t *bars = reinterpret_cast<uint64_t *>(((uintptr_t)(phr_s + 3 * n_phases) + 7) & ~(uintptr_t)7);
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
            mbar_init(tempty + 8 * b, kThreads / 32 - 4);   // one arrival per epilogue warp
        }
        mbar_init(bres, 1);
        mbar_init(mdone, 1);
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (rowmode) prefetch_tmap(&tmY);
        // Start the first loads before the table copies and the TMEM
        // allocation: the resident weights (the grid this one may overlap
        // with, under programmatic launch, is the call's own re-layout or
        // bias fill, which does not write them; see the launch), then, once
        // that grid's output is visible, the first unit's input ring entries.
        if (resident) {
            mbar_arrive_expect_tx(bres, (uint32_t)res_rows * 128);
            for (int r = 0; r < res_rows; r += BR) tma_load_2d(smem_u32(sB + (size_t)r * 128), &tmB, bres, 0, r);
        }
        griddep_wait();
        if ((int)blockIdx.x < n_units) {
            const Unit U = decode_unit(G, blockIdx.x);
            const int x0 = U.tx * BXt + T.g_emin[U.g][2];
            const int y0 = U.y0 + T.g_emin[U.g][1];
            const int z0 = U.jz + T.g_emin[U.g][0];
            const int pre = min(SA, KB * zslices);
            for (int q = 0; q < pre; ++q) {
                const int kb = q / zslices, z = q - kb * zslices;
                mbar_arrive_expect_tx(fullA + 8 * q, a_bytes);
                if (rowmode) {
                    for (int e = 0; e < n_ex; ++e)
                        tma_load_5d(smem_u32(sA + (size_t)q * a_stride + (size_t)e * box_rows * 128), &tmA,
                                    fullA + 8 * q, kb * 64, x0 + e, y0, z0 + z, U.n);
                } else {
                    tma_load_5d(smem_u32(sA + (size_t)q * a_stride), &tmA, fullA + 8 * q, kb * 64, x0, y0, z0, U.n);
                }
            }
        }
    }
    for (int i = threadIdx.x; i < n_items; i += kThreads) {
        SItem it;
        it.shift = T.item[i].shift;
        it.brow = T.item[i].brow;
        it.n = T.item[i].n;
        it.tcol = T.item[i].tcol;
        it.first = T.item[i].first;
        it.pad = 0;
        items_s[i] = it;
        MItem mi;
        mi.a16 = (uint32_t)it.shift * 8u;
        mi.b16 = (uint32_t)it.brow * 8u;
        mi.idesc = idesc_f16_f32(128, it.n);
        mi.col_first = (uint32_t)it.tcol | ((uint32_t)(it.first ? 1 : 0) << 16);
        mitems_s[i] = mi;
    }
    for (int g = threadIdx.x; g < n_groups; g += kThreads) {
        SGroup gr;
        gr.brow = T.g_brow[g];
        gr.rows_kb = T.g_rows_kb[g];
        gr.item0 = T.g_item0[g];
        gr.nitem = T.g_nitem[g];
        gr.phase0 = T.g_phase0[g];
        gr.nphase = T.g_nphase[g];
        gr.emin[0] = T.g_emin[g][0];
        gr.emin[1] = T.g_emin[g][1];
        gr.emin[2] = T.g_emin[g][2];
        gr.pad = 0;
        groups_s[g] = gr;
    }
    for (int i = threadIdx.x; i < 3 * n_phases; i += kThreads) phr_s[i] = T.phase_r[i / 3][i % 3];
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
        // (this thread issued the first unit's first ring entries above,
        // after waiting for the grid whose output it reads)
        const int pre = min(SA, KB * zslices);
        int ia = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            const Unit U = decode_unit(G, u);
            const SGroup gr = groups_s[U.g];
            const int x0 = U.tx * BXt + gr.emin[2];
            const int y0 = U.y0 + gr.emin[1];
            const int z0 = U.jz + gr.emin[0];
            for (int q = 0; q < KB * zslices && ok; ++q, ++ia) {
                if (u == (int)blockIdx.x && q < pre) continue;   // issued in the set-up
                const int kb = q / zslices, z = q - kb * zslices;
                const int s = ia % SA;
                if (ia >= SA && !mbar_wait(emptyA + 8 * s, ((ia / SA) - 1) & 1, err, 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(fullA + 8 * s, a_bytes);
                if (rowmode) {
                    // one z slice: one box per x offset, the unit's rows at pitch BXt
                    for (int e = 0; e < n_ex; ++e)
                        tma_load_5d(smem_u32(sA + (size_t)s * a_stride + (size_t)e * box_rows * 128), &tmA,
                                    fullA + 8 * s, kb * 64, x0 + e, y0, z0 + z, U.n);
                } else {
                    tma_load_5d(smem_u32(sA + (size_t)s * a_stride), &tmA, fullA + 8 * s, kb * 64, x0, y0, z0, U.n);
                }
            }
        }
        const int first = ia > SA ? ia - SA : 0;
        for (int j = first; j < ia; ++j) mbar_wait(fullA + 8 * (j % SA), (j / SA) & 1, err, 2);
    } else if ((warp == 2 || warp == 3) && lane == 0) {
        // ---------------- weight tiles: two issuing warps, alternate ring items ----------------
        const int me = warp - 2;
        // resident weights: loaded in the set-up (the MMA warp waits for them)
        if (!resident) {
            griddep_wait();
            int ib = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const Unit U = decode_unit(G, u);
                const SGroup gr = groups_s[U.g];
                for (int kb = 0; kb < KB && ok; ++kb) {
                    const int rowbase = gr.brow + kb * gr.rows_kb;
                    for (int it = gr.item0; it < gr.item0 + gr.nitem; ++it, ++ib) {
                        if ((ib & 1) != me) continue;
                        const int s = ib % SB;
                        if (ib >= SB && !mbar_wait(emptyB + 8 * s, ((ib / SB) - 1) & 1, err, 4)) {
                            ok = false;
                            break;
                        }
                        const SItem I = items_s[it];
                        mbar_arrive_expect_tx(fullB + 8 * s, (uint32_t)I.n * 128);
                        for (int r = 0; r < I.n; r += BR)
                            tma_load_2d(smem_u32(sB + (size_t)s * b_slot + (size_t)r * 128), &tmB, fullB + 8 * s, 0,
                                        rowbase + I.brow + r);
                    }
                }
            }
            // this warp's copies in flight must land before the CTA exits
            const int first = ib > SB ? ib - SB : 0;
            for (int j = first; j < ib; ++j)
                if ((j & 1) == me) mbar_wait(fullB + 8 * (j % SB), (j / SB) & 1, err, 5);
        }
    } else if (warp == 1) {
        // ---------------- MMA issue ----------------
        // One elected lane walks the items and issues (the rest of the warp
        // waits at the end of each channel block).  The items are narrow
        // (down to N = 32, four K steps each): a whole-warp loop, with its
        // reconvergence between items, measured twice as long per unit here.
        // Each item's descriptor offsets are precomputed in shared memory;
        // the lane adds them to the descriptors of the tile and the weights.
        const bool issuer = elect_one();
        bool ok = true;
        if (resident) ok = __all_sync(0xffffffffu, mbar_wait(bres, 0, err, 6));
        int local = 0;
        uint32_t sa_slot = 0, sa_phase = 0, sb_slot = 0, sb_phase = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++local) {
            const Unit U = decode_unit(G, u);
            const int i0 = T.g_item0[U.g], i1 = i0 + T.g_nitem[U.g];
            const int gbrow = T.g_brow[U.g], grows = T.g_rows_kb[U.g];
            const int buf = nbuf == 2 ? (local & 1) : 0;
            const int use = nbuf == 2 ? (local >> 1) : local;
            if (use > 0) ok = __all_sync(0xffffffffu, mbar_wait(tempty + 8 * buf, (use - 1) & 1, err, 7));
            if (!ok) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + buf * bufcols;
            const uint32_t mstep = (uint32_t)(T.g_nphase[U.g] * Np);
            const int rel = U.F0 - U.y0 * HX;   // row of the unit's first position in the tile
            for (int q = 0; q < KB * zslices && ok; ++q) {
                const int kb = q / zslices, z = q - kb * zslices;
                // the items that read this ring entry: all of the group's, or
                // (row mode) those of z slice z
                const int j0 = rowmode ? i0 + T.g_zitem[U.g][z] : i0;
                const int j1 = rowmode ? i0 + T.g_zitem[U.g][z + 1] : i1;
                if (issuer) {
                    ok = mbar_wait(fullA + 8 * sa_slot, sa_phase, err, 8);
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA) + sa_slot * (uint32_t)a_stride + (uint32_t)rel * 128;
                    const uint64_t adesc0 = desc_kmajor_sw128(a_addr);
                    const uint64_t bdesc0 = desc_kmajor_sw128(smem_u32(sB) + (uint32_t)((gbrow + kb * grows) * 128));
                    if (resident && ok) {
                        // weights resident: nothing to wait for between the items
                        for (int it = j0; it < j1; ++it) {
                            const MItem mi = mitems_s[it];
                            const uint64_t ad = adesc0 + mi.a16;
                            const uint64_t bd = bdesc0 + mi.b16;
                            const uint32_t d = dbase + (mi.col_first & 0xffffu);
                            const uint32_t acc0 = (kb == 0 && (mi.col_first >> 16)) ? 0u : 1u;
                            issue4(d, ad, bd, mi.idesc, acc0);
                            if (Mt > 1) issue4(d + mstep, ad + 1024, bd, mi.idesc, acc0);   // +128 rows
                        }
                    } else {
                        for (int it = j0; it < j1 && ok; ++it) {
                            const MItem mi = mitems_s[it];
                            ok = mbar_wait(fullB + 8 * sb_slot, sb_phase, err, 9);
                            if (!ok) break;
                            tc_fence_after();
                            const uint64_t bd = desc_kmajor_sw128(smem_u32(sB) + sb_slot * (uint32_t)b_slot);
                            const uint64_t ad = adesc0 + mi.a16;
                            const uint32_t d = dbase + (mi.col_first & 0xffffu);
                            const uint32_t acc0 = (kb == 0 && (mi.col_first >> 16)) ? 0u : 1u;
                            issue4(d, ad, bd, mi.idesc, acc0);
                            if (Mt > 1) issue4(d + mstep, ad + 1024, bd, mi.idesc, acc0);   // +128 rows
                            mma_commit(emptyB + 8 * sb_slot);
                            if (++sb_slot == (uint32_t)SB) {
                                sb_slot = 0;
                                sb_phase ^= 1u;
                            }
                        }
                    }
                    if (ok) mma_commit(emptyA + 8 * sa_slot);
                }
                __syncwarp();
                ok = __all_sync(0xffffffffu, ok);
                if (++sa_slot == (uint32_t)SA) {
                    sa_slot = 0;
                    sa_phase ^= 1u;
                }
            }
            if (!ok) break;
            if (issuer) mma_commit(tfull + 8 * buf);
            __syncwarp();
        }
        if (issuer) mma_commit(mdone);
        __syncwarp();
        mbar_wait(mdone, 0, err, 10);
    } else if (warp >= 4 && rowmode) {
        // ---------------- epilogue, row mode: tiles to shared memory, TMA stores ----------------
        const int q = warp & 3;                  // the TMEM lane quarter this warp may read
        const int sx = T.s[2];
        const bool has_bias = T.has_bias;
        const bool bias_vec = has_bias && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
        uint8_t *stage = sStage + (size_t)(warp - 4) * 2 * kStageTile;
        int sbuf = 0;
        int local = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
            const Unit U = decode_unit(G, u);
            const int buf = nbuf == 2 ? (local & 1) : 0;
            const int use = nbuf == 2 ? (local >> 1) : local;
            if (!mbar_wait(tfull + 8 * buf, use & 1, err, 12)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + ((uint32_t)(32 * q) << 16) + buf * bufcols;
            const int gcols = T.g_nphase[U.g] * Np;
            const int ph0 = T.g_phase0[U.g], ph1 = ph0 + T.g_nphase[U.g];
            for (int mt = 0; mt < Mt; ++mt) {
                const int p0 = mt * 128 + 32 * q;          // this warp's first position in the unit
                const int jy = U.y0 + p0 / BXt;
                const int jx0 = U.tx * BXt + p0 % BXt;
                for (int ph = ph0; ph < ph1; ph += sx) {   // s_x = 2: (ph, ph + 1) have r_x = 0, 1
                    const int oz = T.s[0] * U.jz + T.phase_r[ph][0];
                    const int oy = T.s[1] * jy + T.phase_r[ph][1];
                    const uint32_t col0 = dbase + mt * gcols + (ph - ph0) * Np;
                    for (int m0 = 0; m0 < Np; m0 += 32) {
                        uint32_t v0[16], v1[16], w0[16], w1[16];
                        const bool two = m0 + 16 < Np;
                        tmem_ld16(col0 + m0, v0);
                        if (two) tmem_ld16(col0 + m0 + 16, v1);
                        if (sx == 2) {
                            tmem_ld16(col0 + Np + m0, w0);
                            if (two) tmem_ld16(col0 + Np + m0 + 16, w1);
                        }
                        tmem_ld_wait();
                        // the bias from global memory (read-only path): shared-memory
                        // reads here would queue behind the tile loads and stores
                        float bb[32];
                        if (bias_vec && m0 + 32 <= M) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint4 h = __ldg(reinterpret_cast<const uint4 *>(bias + m0) + j);
                                const __half2 *h2 = reinterpret_cast<const __half2 *>(&h);
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const float2 f = __half22float2(h2[c]);
                                    bb[8 * j + 2 * c] = f.x;
                                    bb[8 * j + 2 * c + 1] = f.y;
                                }
                            }
                        } else if (!has_bias) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) bb[j] = 0.f;
                        } else {   // the last, partial block of channels, or an unaligned bias
#pragma unroll
                            for (int j = 0; j < 32; ++j) bb[j] = m0 + j < M ? __half2float(__ldg(bias + m0 + j)) : 0.f;
                        }
                        // the tile written two stores ago must have been read out
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        uint8_t *tile = stage + (size_t)sbuf * kStageTile;
                        if (sx == 2) {
                            // [32 channels][64 x]: lane = J_x, its two x phases side by side
                            uint32_t *t32 = reinterpret_cast<uint32_t *>(tile) + lane;
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const __half2 h = __floats2half2_rn(apply_act(__uint_as_float(v0[j]) + bb[j], ACT),
                                                                    apply_act(__uint_as_float(w0[j]) + bb[j], ACT));
                                t32[32 * j] = *reinterpret_cast<const uint32_t *>(&h);
                            }
                            if (two) {
#pragma unroll
                                for (int j = 0; j < 16; ++j) {
                                    const __half2 h =
                                        __floats2half2_rn(apply_act(__uint_as_float(v1[j]) + bb[16 + j], ACT),
                                                          apply_act(__uint_as_float(w1[j]) + bb[16 + j], ACT));
                                    t32[32 * (16 + j)] = *reinterpret_cast<const uint32_t *>(&h);
                                }
                            }
                        } else {
                            // [32 channels][32 x]
                            __half *t16 = reinterpret_cast<__half *>(tile) + lane;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                t16[32 * j] = __float2half_rn(apply_act(__uint_as_float(v0[j]) + bb[j], ACT));
                            if (two) {
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    t16[32 * (16 + j)] =
                                        __float2half_rn(apply_act(__uint_as_float(v1[j]) + bb[16 + j], ACT));
                            }
                        }
                        fence_proxy_async();   // the tile, written by this warp, before the bulk store reads it
                        __syncwarp();
                        if (lane == 0) {
                            // channels m0 + 16.. of a one-chunk piece hold no data: they lie at or
                            // beyond M, where the store writes nothing
                            tma_store_5d(&tmY, smem_u32(tile), sx * jx0, oy, oz, m0, U.n);
                            bulk_commit_group();
                        }
                        sbuf ^= 1;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + 8 * buf);
        }
        if (lane == 0) bulk_wait_group_all();   // every store has left this CTA's shared memory
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- epilogue ----------------
        // the bias, staged by the epilogue warps themselves (its global reads
        // stay off the set-up's path to the first loads)
        for (int m = (int)threadIdx.x - 128; m < ((Np + 31) & ~31); m += kThreads - 128)
            bias_s[m] = (T.has_bias && m < M) ? __half2float(bias[m]) : 0.f;
        named_bar_sync(1, kThreads - 128);
        const int lane_base = 32 * (warp & 3);   // the TMEM lane quarter this warp may read
        const int eh = (warp - 4) >> 2;           // first 32-channel chunk of this warp's set
        const int p = lane_base + lane;
        const int out0 = T.out[0], out1 = T.out[1], out2 = T.out[2];
        const int s0 = T.s[0], s1 = T.s[1], s2 = T.s[2];
        const int nJ1 = T.nJ[1], nJ2 = T.nJ[2];
        const bool has_bias = T.has_bias;
        const bool bias_vec = has_bias && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
        const long long plane = (long long)out0 * out1 * out2;
        const long long cstride = nhwc ? 1 : plane;        // between channels
        const long long xstep = nhwc ? (long long)M : 1;   // between x positions
        int local = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
            const Unit U = decode_unit(G, u);
            const int buf = nbuf == 2 ? (local & 1) : 0;
            const int use = nbuf == 2 ? (local >> 1) : local;
            if (!mbar_wait(tfull + 8 * buf, use & 1, err, 11)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + ((uint32_t)lane_base << 16) + buf * bufcols;
            const int gcols = T.g_nphase[U.g] * Np;
            const int ph0 = T.g_phase0[U.g], ph1 = ph0 + T.g_nphase[U.g];
            for (int mt = 0; mt < Mt; ++mt) {
                const int F = U.F0 + mt * 128 + p;
                const int jxl = F % HX;
                const int Jy = F / HX;
                const int Jx = U.tx * BXt + jxl;
                const bool pos_ok = jxl < BXt && Jx < nJ2 && Jy < nJ1;
                for (int ph = ph0; ph < ph1;) {
                    const int r0 = T.phase_r[ph][0], r1 = T.phase_r[ph][1], r2 = T.phase_r[ph][2];
                    const int oz = s0 * U.jz + r0;
                    const int oy = s1 * Jy + r1;
                    const int ox = s2 * Jx + r2;
                    const bool valid = pos_ok && oz < out0 && oy < out1 && ox < out2;
                    const bool pair = pair_x && ph + 1 < ph1 && (r2 & 1) == 0 && T.phase_r[ph + 1][2] == r2 + 1 &&
                                      T.phase_r[ph + 1][1] == r1 && T.phase_r[ph + 1][0] == r0;
                    const long long opos = ((long long)oz * out1 + oy) * out2 + ox;
                    const uint32_t col0 = dbase + mt * gcols + (ph - ph0) * Np;
                    __half *base = nhwc ? y + ((long long)U.n * plane + opos) * M : y + (long long)U.n * M * plane + opos;
                    for (int m0 = 32 * eh; m0 < Np; m0 += 32 * kEpiSets) {
                        uint32_t v0[16], v1[16], w0[16], w1[16];
                        const bool two = m0 + 16 < Np;
                        tmem_ld16(col0 + m0, v0);
                        if (two) tmem_ld16(col0 + m0 + 16, v1);
                        if (pair) {
                            tmem_ld16(col0 + Np + m0, w0);
                            if (two) tmem_ld16(col0 + Np + m0 + 16, w1);
                        }
                        tmem_ld_wait();
                        if (!valid) continue;
                        const int mc0 = min(16, M - m0), mc1 = min(16, M - m0 - 16);
                        __half *dst = base + (long long)m0 * cstride;
                        if (!nhwc && pair) {
                            // both x phases of a channel are adjacent: one half2 per channel
                            // bias through the read-only global path: shared-memory
                            // reads here wait behind the next unit's tile loads
                            float bb[32];
                            if (bias_vec && m0 + 32 <= M) {
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const uint4 h = __ldg(reinterpret_cast<const uint4 *>(bias + m0) + j);
                                    const __half2 *h2 = reinterpret_cast<const __half2 *>(&h);
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        const float2 f = __half22float2(h2[q]);
                                        bb[8 * j + 2 * q] = f.x;
                                        bb[8 * j + 2 * q + 1] = f.y;
                                    }
                                }
                            } else if (!has_bias) {
#pragma unroll
                                for (int j = 0; j < 32; ++j) bb[j] = 0.f;
                            } else {   // the last, partial chunk of channels, or an unaligned bias
#pragma unroll
                                for (int j = 0; j < 32; ++j) bb[j] = bias_s[m0 + j];
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (j < mc0)
                                    *reinterpret_cast<__half2 *>(dst + j * plane) =
                                        __floats2half2_rn(apply_act(__uint_as_float(v0[j]) + bb[j], ACT),
                                                          apply_act(__uint_as_float(w0[j]) + bb[j], ACT));
                            if (two) {
                                __half *d1 = dst + 16 * plane;
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    if (j < mc1)
                                        *reinterpret_cast<__half2 *>(d1 + j * plane) =
                                            __floats2half2_rn(apply_act(__uint_as_float(v1[j]) + bb[16 + j], ACT),
                                                              apply_act(__uint_as_float(w1[j]) + bb[16 + j], ACT));
                            }
                        } else if (nhwc) {
                            float bb[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) bb[j] = bias_s[m0 + j];
                            store_row16<ACT>(dst, v0, bb, mc0);
                            if (two) store_row16<ACT>(dst + 16, v1, bb + 16, mc1);
                            if (pair) {
                                __half *dx = dst + xstep;   // x + 1
                                store_row16<ACT>(dx, w0, bb, mc0);
                                if (two) store_row16<ACT>(dx + 16, w1, bb + 16, mc1);
                            }
                        } else {
                            store_chunk16<ACT>(dst, cstride, v0, bias_s + m0, mc0);
                            if (two) store_chunk16<ACT>(dst + 16 * cstride, cstride, v1, bias_s + m0 + 16, mc1);
                            if (pair) {
                                __half *dx = dst + xstep;   // x + 1
                                store_chunk16<ACT>(dx, cstride, w0, bias_s + m0, mc0);
                                if (two) store_chunk16<ACT>(dx + 16 * cstride, cstride, w1, bias_s + m0 + 16, mc1);
                            }
                        }
                    }
                    ph += pair ? 2 : 1;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + 8 * buf);
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
    const size_t tables = (size_t)T.n_items * (sizeof(SItem) + sizeof(MItem)) + (size_t)T.n_groups * sizeof(SGroup) +
                          (size_t)T.n_phases * 6 + 8;
    return 1024 + (size_t)T.SA * T.a_stride + (T.rowmode ? (size_t)kStageBytes : 0) + b_region +
           (size_t)((T.Np + 31) & ~31) * 4 + tables + (size_t)(2 * T.SA + 2 * T.SB + 6) * 8 + 16;
}

// Row mode applies to channels-first output whose x phases the epilogue can
// store as contiguous runs: s_x = 1, or s_x = 2 with both x phases live;
// every phase live (the stores cover whole rows); out_x a multiple of 8 (the
// output rows are 16-byte multiples, as TMA needs).
bool rowmode_ok(const Plan &p) {
    if (p.layout != CT_NCHW || has_dead_phases(p)) return false;
    if (!(p.s[2] == 1 || (p.s[2] == 2 && p.out[2] % 2 == 0))) return false;
    if (p.out[2] % 8 != 0) return false;
    for (int a = 0; a < 3; ++a)
        if (p.out[a] > (1 << 30) / 2) return false;
    return true;
}

// Build the tables for one policy: Mt M-tiles per unit and groups of at
// most `gmax_cols` accumulator columns.  Returns false when a limit or the
// shared-memory budget is exceeded.
bool build_tables(const Plan &p, HaloTables &T, int Mt, int gmax_cols, bool rowmode) {
    T.N = (int32_t)p.N;
    T.C = (int32_t)p.C;
    T.M = (int32_t)p.M;
    T.Np = (int32_t)((p.M + 15) / 16 * 16);
    T.KB = (int32_t)ceil_div(p.C, 64);
    T.nhwc = p.layout == CT_NHWC;
    T.has_bias = p.has_bias;
    T.act = p.act;
    T.Mt = Mt;
    if (T.Np > gmax_cols) return false;
    // row mode stores the x phases of a (z, y) phase pair together: both must
    // fall in one group
    if (rowmode && p.s[2] * T.Np > gmax_cols) return false;
    for (int a = 0; a < 3; ++a) {
        T.out[a] = (int32_t)p.out[a];
        T.s[a] = (int32_t)p.s[a];
        T.nJ[a] = (int32_t)ceil_div(p.out[a], p.s[a]);
        T.pb[a] = (int32_t)p.pb[a];
        T.d[a] = (int32_t)p.d[a];
        T.k[a] = (int32_t)p.k[a];
    }
    T.pair_x = (p.s[2] % 2 == 0) && (p.out[2] % 2 == 0);
    T.dead = has_dead_phases(p);
    // live phases
    int np = 0;
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
    // groups: whole (r0, r1) rows of phases, merged while within gmax_cols
    const int per = gmax_cols / T.Np;
    auto same_row = [&](int a, int b) {
        return T.phase_r[a][0] == T.phase_r[b][0] && T.phase_r[a][1] == T.phase_r[b][1];
    };
    int ng = 0;
    for (int ph = 0; ph < np;) {
        int end = ph;
        while (end < np) {
            int row_end = end + 1;
            while (row_end < np && same_row(row_end, end)) ++row_end;
            if (row_end - ph <= per)
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
    // offset range of every group; the input tile is sized by the widest
    for (int a = 0; a < 3; ++a) {
        T.emin[a] = 0;
        T.span[a] = 0;
    }
    for (int g = 0; g < ng; ++g) {
        int lo[3] = {1 << 20, 1 << 20, 1 << 20}, hi[3] = {-(1 << 20), -(1 << 20), -(1 << 20)};
        for (int ph = T.g_phase0[g]; ph < T.g_phase0[g] + T.g_nphase[g]; ++ph)
            for (int a = 0; a < 3; ++a)
                for (const Tap &t : p.taps[a][T.phase_r[ph][a]]) {
                    lo[a] = std::min(lo[a], (int)t.e);
                    hi[a] = std::max(hi[a], (int)t.e);
                }
        for (int a = 0; a < 3; ++a) {
            T.g_emin[g][a] = (int16_t)lo[a];
            T.span[a] = std::max(T.span[a], hi[a] - lo[a]);
        }
    }
    // input tile geometry
    T.rowmode = rowmode ? 1 : 0;
    if (rowmode) {
        // pitch BXt (no halo columns): 32, 64 or 128 J_x per row segment, x
        // tiles of 128 beyond that; R whole rows per unit
        T.BXt = T.nJ[2] <= 32 ? 32 : T.nJ[2] <= 64 ? 64 : 128;
        T.HX = T.BXt;
        T.R = Mt * 128 / T.BXt;
        T.HYb = T.R + T.span[1];
        T.n_ex = 1 + T.span[2];
    } else {
        if (T.nJ[2] + T.span[2] <= 256) {
            T.BXt = T.nJ[2];
        } else {
            T.BXt = 256 - T.span[2];
            if (T.BXt < 64) return false;
        }
        T.HX = T.BXt + T.span[2];
        T.HYb = (int32_t)ceil_div((int64_t)Mt * 128 + T.HX + T.span[2], T.HX) + T.span[1];
        T.R = 0;
        T.n_ex = 1;
    }
    T.HZb = 1 + T.span[0];
    if (T.HYb > 256 || T.HZb > 256) return false;
    if (rowmode) {
        // one ring entry per z slice: n_ex boxes of HX x HYb positions
        if (T.HZb > kMaxZ) return false;
        T.zslices = T.HZb;
        T.box_rows = T.HX * T.HYb;
    } else {
        T.zslices = 1;
        T.box_rows = T.HX * T.HYb * T.HZb;
    }
    T.a_bytes = T.n_ex * T.box_rows * 128;
    T.a_stride = (T.a_bytes + 1023) & ~1023;
    T.TX = (int32_t)ceil_div(T.nJ[2], T.BXt);
    const long long plane_pos = (long long)T.nJ[1] * T.HX;
    T.PU = (int32_t)ceil_div(plane_pos, (long long)Mt * 128);
    const long long units = (long long)T.N * T.nJ[0] * T.TX * T.PU * ng;
    if (units > (1LL << 30)) return false;
    T.n_units = (int32_t)units;
    // items per group: pairs grouped by input offset, merged over adjacent phases
    int ni = 0, rows_total = 0;
    // row mode: a slice holds one z offset (slice_pitch unused), x offsets are boxes
    const int row_pitch = T.HX, slice_pitch = rowmode ? 0 : T.HX * T.HYb, ex_pitch = rowmode ? T.box_rows : 1;
    for (int g = 0; g < ng; ++g) {
        struct PairRec { int ph, e0, e1, e2; };
        std::vector<PairRec> pairs;
        for (int ph = T.g_phase0[g]; ph < T.g_phase0[g] + T.g_nphase[g]; ++ph) {
            const int r0 = T.phase_r[ph][0], r1 = T.phase_r[ph][1], r2 = T.phase_r[ph][2];
            for (const Tap &a : p.taps[0][r0])
                for (const Tap &b : p.taps[1][r1])
                    for (const Tap &c : p.taps[2][r2]) pairs.push_back({ph, a.e, b.e, c.e});
        }
        std::vector<std::array<int, 3>> offs;
        for (auto &q : pairs) offs.push_back({q.e0, q.e1, q.e2});
        std::sort(offs.begin(), offs.end());
        offs.erase(std::unique(offs.begin(), offs.end()), offs.end());
        // offsets shared by more phases first: their phases are then all
        // untouched and merge into one wide item instead of several narrow ones
        auto nph = [&](const std::array<int, 3> &e) {
            int c = 0;
            for (auto &q : pairs) c += (q.e0 == e[0] && q.e1 == e[1] && q.e2 == e[2]);
            return c;
        };
        std::stable_sort(offs.begin(), offs.end(),
                         [&](const std::array<int, 3> &a, const std::array<int, 3> &b) { return nph(a) > nph(b); });
        if (rowmode)   // row mode consumes the input z slice by z slice
            std::stable_sort(offs.begin(), offs.end(),
                             [&](const std::array<int, 3> &a, const std::array<int, 3> &b) { return a[0] < b[0]; });
        std::vector<char> touched(np, 0);
        T.g_item0[g] = (int16_t)ni;
        int brow = 0;
        for (auto &e : offs) {
            std::vector<int> phs;
            for (auto &q : pairs)
                if (q.e0 == e[0] && q.e1 == e[1] && q.e2 == e[2]) phs.push_back(q.ph);
            std::sort(phs.begin(), phs.end());
            size_t i = 0;
            while (i < phs.size()) {
                size_t j = i + 1;
                while (j < phs.size() && phs[j] == phs[j - 1] + 1 && touched[phs[j]] == touched[phs[i]] &&
                       (int)(j - i + 1) * T.Np <= 256)
                    ++j;
                if (ni >= kMaxItems) return false;
                Item &I = T.item[ni];
                I.e[0] = (int16_t)e[0];
                I.e[1] = (int16_t)e[1];
                I.e[2] = (int16_t)e[2];
                I.n = (int16_t)((j - i) * T.Np);
                I.shift = (e[0] - T.g_emin[g][0]) * slice_pitch + (e[1] - T.g_emin[g][1]) * row_pitch +
                          (e[2] - T.g_emin[g][2]) * ex_pitch;
                I.tcol = (int16_t)((phs[i] - T.g_phase0[g]) * T.Np);
                I.phase0 = (int16_t)phs[i];
                I.first = touched[phs[i]] ? 0 : 1;
                I.pad = 0;
                I.brow = brow;
                brow += I.n;
                for (size_t q = i; q < j; ++q) touched[phs[q]] = 1;
                ++ni;
                i = j;
            }
        }
        T.g_nitem[g] = (int16_t)(ni - T.g_item0[g]);
        if (rowmode) {
            for (int z = 0; z <= T.zslices; ++z) {
                int c = 0;
                while (c < T.g_nitem[g] && T.item[T.g_item0[g] + c].e[0] - T.g_emin[g][0] < z) ++c;
                T.g_zitem[g][z] = (int16_t)c;
            }
        }
        T.g_brow[g] = rows_total;
        T.g_rows_kb[g] = brow;
        rows_total += brow * T.KB;
    }
    T.n_items = ni;
    T.total_rows = rows_total;
    // TMEM: Mt x group columns per buffer, double-buffered when that fits
    int gcols = 0;
    for (int g = 0; g < ng; ++g) gcols = std::max(gcols, (int)T.g_nphase[g] * T.Np);
    T.bufcols = Mt * gcols;
    if (T.bufcols > 512) return false;
    T.nbuf = T.bufcols <= 256 ? 2 : 1;
    int br = 256;
    for (int i = 0; i < ni; ++i)
        while (T.item[i].n % br) br /= 2;
    T.BR = br;
    int nmax = 0;
    for (int i = 0; i < ni; ++i) nmax = std::max(nmax, (int)T.item[i].n);
    T.b_slot_bytes = nmax * 128;
    // shared memory: resident weights if they fit next to two input slots
    const int fixed = 1024 + ((T.Np + 31) & ~31) * 4 + 64 * 8 + 64 + ni * (int)(sizeof(SItem) + sizeof(MItem)) + ng * (int)sizeof(SGroup) +
                      np * 6 + 8 + (rowmode ? kStageBytes : 0);
    T.resident = 0;
    T.res_rows = 0;
    // row mode keeps the weights resident with a single input slot too: its
    // input is re-read from L2 and the output stores run under the next unit
    const long long min_sa = rowmode ? 1 : 2;
    if ((long long)rows_total * 128 + min_sa * T.a_stride + fixed <= kSmemBudget) {
        T.resident = 1;
        T.res_rows = rows_total;
        T.SA = (int)std::min<long long>(4, (kSmemBudget - fixed - (long long)rows_total * 128) / T.a_stride);
        T.SB = 1;
    } else {
        int best_sa = 0, best_sb = 0;
        for (int sa = 4; sa >= 2 && !best_sa; --sa) {
            const long long rest = kSmemBudget - fixed - (long long)sa * T.a_stride;
            const long long sb = rest / T.b_slot_bytes;
            if (sb >= 4 || (sa == 2 && sb >= 2)) {
                best_sa = sa;
                best_sb = (int)std::min<long long>(sb, 12);
            }
        }
        if (best_sa == 0) return false;
        T.SA = best_sa;
        T.SB = best_sb;
    }
    return smem_bytes(T) <= (size_t)kSmemBudget;
}

// Pick the layout: Mt x group of accumulator columns.  Measured on a B200
// (2-D fp16 decoder and 3-D fp16 upsample workloads), two M-tiles with both x
// phases of a pair in one group (TMEM single-buffered, whole-line half2
// stores, half the weight traffic per pixel) is fastest, then one M-tile with
// paired phases (double-buffered), then two M-tiles of lone phases.
bool choose_tables(const Plan &p, HaloTables &T) {
    if (rowmode_ok(p)) {
        // row mode: one M-tile per unit, so the accumulators are double-buffered
        const int ropts[2][2] = {{1, 256}, {1, 128}};
        for (int o = 0; o < 2; ++o) {
            T = HaloTables();
            if (build_tables(p, T, ropts[o][0], ropts[o][1], true)) return true;
        }
    }
    const int opts[3][2] = {{2, 256}, {1, 256}, {2, 128}};
    for (int o = 0; o < 3; ++o) {
        T = HaloTables();
        if (build_tables(p, T, opts[o][0], opts[o][1], false)) return true;
    }
    return false;
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
    HaloTables *T = new HaloTables();
    const bool ok = choose_tables(p, *T);
    delete T;
    return ok;
}

void dense_tc_setup(Plan &p) {
    p.aux.assign((sizeof(HaloTables) + 7) / 8, 0);
    HaloTables &T = *reinterpret_cast<HaloTables *>(p.aux.data());
    choose_tables(p, T);
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
                       void *ws, cudaStream_t st, int parts) {
    const HaloTables &T = tables(p);
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
        // row mode loads one z slice per box
        const cuuint32_t box[5] = {64, (cuuint32_t)T.HX, (cuuint32_t)T.HYb, (cuuint32_t)(T.rowmode ? 1 : T.HZb), 1};
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
    CUtensorMap tmY;
    memset(&tmY, 0, sizeof(tmY));
    if (T.rowmode) {
        // Y[n][m][z][y][x] as a 5-D tensor; box: one row segment of s_x*32
        // outputs for 32 channels
        const cuuint64_t dims[5] = {(cuuint64_t)p.out[2], (cuuint64_t)p.out[1], (cuuint64_t)p.out[0],
                                    (cuuint64_t)p.M, (cuuint64_t)p.N};
        const cuuint64_t e2 = 2;
        const cuuint64_t strides[4] = {e2 * p.out[2], e2 * p.out[2] * p.out[1], e2 * p.out[2] * p.out[1] * p.out[0],
                                       e2 * p.out[2] * p.out[1] * p.out[0] * p.M};
        const cuuint32_t box[5] = {(cuuint32_t)(T.s[2] * 32), 1, 1, 32, 1};
        const cuuint32_t es[5] = {1, 1, 1, 1, 1};
        if (enc(&tmY, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    if (T.dead && (parts & CT_PART_PREPARE)) {
        ct_status s2 = launch_dead_fill(p, bias, y, st);
        if (s2 != CT_OK) return s2;
    }
    if (!(parts & CT_PART_MAIN)) return CT_OK;
    int grid = sm_count();
    if (grid > T.n_units) grid = T.n_units;
    // programmatic dependent launch when this call's own re-layout or bias
    // fill runs just before: the set-up overlaps that grid's tail, and the
    // kernel reads the packed weights before waiting for it (neither writes
    // them; the grid before it is complete, as it was launched normally).
    // Otherwise the kernel starts after all earlier work, like any launch.
    const bool pdl = (parts & CT_PART_PREPARE) && (p.layout == CT_NCHW || T.dead);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes(T);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const __half *b = (const __half *)bias;
    __half *yy = (__half *)y;
    cudaError_t e;
    if (T.act == CT_ACT_RELU) {
        static std::atomic<int> attr_set[64];
        if (!allow_smem(dense_halo_kernel<CT_ACT_RELU>, attr_set, kSmemBudget)) return CT_ERR_DEVICE;
        e = cudaLaunchKernelEx(&cfg, dense_halo_kernel<CT_ACT_RELU>, tmA, tmB, tmY, T, b, yy);
    } else {
        static std::atomic<int> attr_set[64];
        if (!allow_smem(dense_halo_kernel<CT_ACT_IDENTITY>, attr_set, kSmemBudget)) return CT_ERR_DEVICE;
        e = cudaLaunchKernelEx(&cfg, dense_halo_kernel<CT_ACT_IDENTITY>, tmA, tmB, tmY, T, b, yy);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return CT_ERR_DEVICE;
    }
    return launch_status();
}

int dense_tc_take_error(cudaStream_t st) { return take_error_word(g_dense_halo_err, st); }

}  // namespace ct
