// Dense fp16 ConvTranspose (group 1, one or two spatial axes, channels-first)
// on pairs of SMs: every tcgen05 MMA spans the two CTAs of a cluster
// (cta_group::2, M = 256 positions).  Each SM reads its own 128 positions of
// A and only HALF of every weight tile from its shared memory, and keeps the
// accumulators of its 128 positions in its TMEM, double-buffered, so a unit's
// epilogue runs under the next unit's MMAs.
//
// Phases as in the halo kernel: output o = s*J + r per axis; tap k of phase r
// reads input i = J + e, e = (r + pad_begin - k*d) / s (ai.onnx.ConvTranspose
// README, implementation notes on the tap-reversed stride-1 form and the
// grouped stride-phase variant).
//
// Input staging: X is re-laid into a zero-padded channels-last copy
// Xp[n][yp][xp][c], yp = iy - emin_y, xp = ix - emin_x (emin the smallest
// input offset of any tap), HX = nJx + span_x columns and HYp = nJy + span_y
// rows per image.  Output position (Jy, Jx) is numbered F = Jy*HX + Jx, and
// its input under offset e is padded row F + shift(e), shift(e) =
// (ey - emin_y)*HX + (ex - emin_x).  So a CTA's 128 positions need ONE
// contiguous run of 128 + max shift rows (plain 2-D TMA boxes), both CTAs of
// a pair place their runs at the same shared offset, and every tap of every
// phase is the same run shifted by a constant number of 128-byte rows.
//
// Warps: 0 loads input runs, 1 allocates TMEM (both CTAs) and issues MMAs
// (rank 0), 2-3 load weight chunks, 4-11 drain TMEM (both CTAs; two warps
// per TMEM lane quarter, alternate 32-channel chunks).
#include <cuda.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <vector>

#include "ct_cuda_util.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {
namespace {

constexpr int kPMaxPhases = 64;
constexpr int kPMaxGroups = 64;
constexpr int kPMaxItems = 256;
constexpr int kPMaxChunks = 256;
constexpr int kPThreads = 384;
constexpr int kPSmemBudget = 227 * 1024;
constexpr int kPMaxTileRows = 512;

struct PItem {
    int32_t shift;    // padded rows from a position to its input under this offset
    int16_t n;        // MMA N: phases of the run x Np (each CTA holds n/2 weight rows)
    int16_t tcol;     // first accumulator column of the run
    int16_t first;    // first write of these columns (at channel block 0)
    int16_t phase0;   // first phase of the run
    int16_t e[2];     // input offset (y, x)
    int16_t crow;     // first row of the item's half inside its chunk's half (either rank)
    int16_t pad;
};

struct PairTables {
    int32_t N, C, M, Np, KB;
    int32_t H, W, nJy, nJx, outy, outx, sy, sx, pby, pbx, dy, dx, ky, kx;
    int32_t emin_y, emin_x, HX, HYp;
    int32_t tile_rows, chunk_rows, n_chunks, a_bytes, a_stride;
    int32_t SA, SB, b_slot, BR;
    int32_t PU, n_units, n_groups, n_phases, n_items, total_rows;
    int32_t has_bias, dead, pair_x, act;
    int16_t phase_r[kPMaxPhases][2];   // (ry, rx) of every live phase
    int16_t g_phase0[kPMaxGroups], g_nphase[kPMaxGroups], g_item0[kPMaxGroups], g_nitem[kPMaxGroups];
    int32_t g_brow[kPMaxGroups], g_rows_kb[kPMaxGroups];
    int16_t g_chunk0[kPMaxGroups], g_nchunk[kPMaxGroups];
    // a chunk: consecutive items of a group whose weights one barrier covers;
    // inside one channel block its rows are [row0, row0 + half) for rank 0,
    // then [row0 + half, row0 + 2 half) for rank 1
    int16_t c_item0[kPMaxChunks], c_nitem[kPMaxChunks];
    int32_t c_row0[kPMaxChunks], c_half[kPMaxChunks];
    PItem item[kPMaxItems];
};

__device__ int g_dense_pair_err;

const PairTables &ptables(const Plan &p) { return *reinterpret_cast<const PairTables *>(p.aux.data()); }

// ---------------------------------------------------------------------------
// weight pre-pack: rows of every group, channel block, chunk and rank in the
// order the kernel loads them; a row holds 64 input channels of one output
// channel m of one phase, W[kb*64 + cc][m][ky][kx] at the phase's taps for the
// item's offset, zero outside C and M.  Rows [0, n/2) of an item's N columns
// feed the pair's rank 0, rows [n/2, n) rank 1.

__global__ void __launch_bounds__(256) pair_prepack_kernel(const __grid_constant__ PairTables T,
                                                           const __half *__restrict__ w,
                                                           __half *__restrict__ wp) {
    const long long total = (long long)T.total_rows * 64;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int cc = (int)(i & 63);
        const int row = (int)(i >> 6);
        int g = 0;
        while (g + 1 < T.n_groups && row >= T.g_brow[g + 1]) ++g;
        const int rg = row - T.g_brow[g];
        const int kb = rg / T.g_rows_kb[g];
        const int rk = rg % T.g_rows_kb[g];
        int c = T.g_chunk0[g];
        const int c1 = T.g_chunk0[g] + T.g_nchunk[g];
        while (c + 1 < c1 && rk >= T.c_row0[c + 1]) ++c;
        const int r2 = rk - T.c_row0[c];
        const int rank = r2 >= T.c_half[c] ? 1 : 0;
        const int r3 = r2 - rank * T.c_half[c];
        int it = T.c_item0[c];
        const int i1 = T.c_item0[c] + T.c_nitem[c];
        while (it + 1 < i1 && r3 >= T.item[it + 1].crow) ++it;
        const PItem &I = T.item[it];
        const int rr = rank * (I.n / 2) + (r3 - I.crow);
        const int ph = I.phase0 + rr / T.Np;
        const int m = rr % T.Np;
        const int ci = kb * 64 + cc;
        __half v = __float2half(0.f);
        if (ci < T.C && m < T.M) {
            const int nyy = T.phase_r[ph][0] + T.pby - I.e[0] * T.sy;
            const int nxx = T.phase_r[ph][1] + T.pbx - I.e[1] * T.sx;
            const int ka = nyy / T.dy, kc = nxx / T.dx;
            if (nyy % T.dy == 0 && nxx % T.dx == 0 && ka >= 0 && ka < T.ky && kc >= 0 && kc < T.kx)
                v = w[(((long long)ci * T.M + m) * T.ky + ka) * T.kx + kc];
        }
        wp[i] = v;
    }
}

// ---------------------------------------------------------------------------
// X[n][c][iy][ix] -> Xp[n][iy + oy][ix + ox][c] (positions outside the padded
// image dropped), plus zeros at every padded position no input lands on.
// Block x = 0 writes the zero halo of image blockIdx.z for the 64-channel
// block blockIdx.y; blocks x = 1..tiles move a tile of 64 channels x 128
// input positions (as the plain channels-last re-layout, XOR-swizzled
// exchange).

constexpr int kPadC = 64, kPadS = 128;

__global__ void __launch_bounds__(256) nchw_to_padded_kernel(const __half *__restrict__ x,
                                                             __half *__restrict__ xp, int C, int H,
                                                             int W, int HYp, int HX, int oy, int ox) {
    const int n = blockIdx.z;
    const long long S = (long long)H * W;
    const long long P = (long long)HYp * HX;
    const int t = threadIdx.x;
    if (blockIdx.x == 0) {
        // zero halo of image n, channels [c0, c0 + 64): full rows above and
        // below the input, and the columns left and right of it in between
        const int c0 = blockIdx.y * kPadC;
        const int c8 = (min(kPadC, C - c0)) >> 3;
        const int top = min(max(oy, 0), HYp);
        const int mid_end = min(max(oy + H, top), HYp);
        const int left = min(max(ox, 0), HX);
        const int right0 = min(max(ox + W, left), HX);
        const int lr = left + (HX - right0);
        const int n_top = top * HX, n_mid = (mid_end - top) * lr, n_all = n_top + n_mid + (HYp - mid_end) * HX;
        __half *img = xp + (long long)n * P * C + c0;
        for (int q = t; q < n_all * c8; q += blockDim.x) {
            const int k = q / c8;
            const int cc = q - k * c8;
            int yp, xq;
            if (k < n_top) {
                yp = k / HX;
                xq = k - yp * HX;
            } else if (k < n_top + n_mid) {
                const int r = (k - n_top) / lr, j = (k - n_top) - r * lr;
                yp = top + r;
                xq = j < left ? j : right0 + (j - left);
            } else {
                const int k3 = k - n_top - n_mid;
                yp = mid_end + k3 / HX;
                xq = k3 - (k3 / HX) * HX;
            }
            *reinterpret_cast<uint4 *>(img + ((long long)yp * HX + xq) * C + cc * 8) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    __shared__ __align__(16) __half tile[kPadC][kPadS];
    const int c0 = blockIdx.y * kPadC;
    const long long s0 = (long long)(blockIdx.x - 1) * kPadS;
    const bool vec = (S & 7) == 0;
    {
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
            *reinterpret_cast<uint4 *>(&tile[row][(sv ^ ((row >> 3) & 7)) * 8]) = v[r];
        }
    }
    __syncthreads();
    {
        const int sl = t >> 3, cv = t & 7;
        const int c = c0 + cv * 8;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int sp = sl + 32 * r;
            const long long s = s0 + sp;
            if (s >= S || c >= C) continue;
            const int iy = (int)s / W, ix = (int)s - iy * W;   // S < 2^31
            const int yp = iy + oy, xq = ix + ox;
            if (yp < 0 || yp >= HYp || xq < 0 || xq >= HX) continue;
            __align__(16) __half v[8];
            const int col = (((sp >> 3) ^ cv) << 3) | (sp & 7);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = tile[cv * 8 + j][col];
            *reinterpret_cast<uint4 *>(xp + ((long long)n * P + (long long)yp * HX + xq) * C + c) =
                *reinterpret_cast<const uint4 *>(v);
        }
    }
}

// ---------------------------------------------------------------------------
// A unit: image n, group g, pair positions [pu*256, pu*256 + 256); rank r of
// the pair owns [pu*256 + 128*r, +128).  Units are walked cluster-strided.
// Every role reads the tables from the kernel parameters with warp-uniform
// indices; nothing but the bias is copied to shared memory.

template <int ACT>
__device__ __forceinline__ float act_f(float v) {
    return apply_act(v, ACT);
}

template <int ACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    dense_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ PairTables T, const __half *__restrict__ bias,
                      __half *__restrict__ y) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
    const int SA = T.SA, SB = T.SB, KB = T.KB, Np = T.Np, M = T.M;
    const int n_units = T.n_units, a_stride = T.a_stride, a_bytes = T.a_bytes, b_slot = T.b_slot;
    const int BR = T.BR, HX = T.HX, ng = T.n_groups, PU = T.PU;
    const int chunk_rows = T.chunk_rows, n_chunks = T.n_chunks;
    const long long img_rows = (long long)T.HYp * HX;
    // shared-memory layout (identical in both CTAs of the pair)
    uint8_t *sA = smem;
    uint8_t *sB = sA + (size_t)SA * a_stride;
    float *bias_s = reinterpret_cast<float *>(sB + (size_t)SB * b_slot);
    uint64_t *bars = reinterpret_cast<uint64_t *>(bias_s + ((Np + 31) & ~31));   // 128-byte multiple: aligned
    const uint32_t fullA = smem_u32(bars), emptyA = smem_u32(bars + SA);
    const uint32_t fullB = smem_u32(bars + 2 * SA), emptyB = smem_u32(bars + 2 * SA + SB);
    const uint32_t tfull = smem_u32(bars + 2 * SA + 2 * SB);
    const uint32_t tempty = tfull + 16, mdone = tfull + 32;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * SA + 2 * SB + 5);
    int *err = &g_dense_pair_err;

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
            mbar_init(tempty + 8 * b, 16);   // 8 epilogue warps x 2 CTAs
        }
        mbar_init(mdone, 1);
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    for (int m = threadIdx.x; m < ((Np + 31) & ~31); m += kPThreads)
        bias_s[m] = (T.has_bias && m < M) ? __half2float(bias[m]) : 0.f;
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // rank 0's barriers as seen from this CTA
    const uint32_t fullA0 = mapa_shared(fullA, 0), fullB0 = mapa_shared(fullB, 0);
    const uint32_t tempty0 = mapa_shared(tempty, 0);

    if (warp == 0 && lane == 0) {
        // ---------------- input runs (both CTAs; rank 0 expects both halves) ----------------
        int ia = 0;
        bool ok = true;
        for (int u = cid; u < n_units && ok; u += ncl) {
            const int t = u / ng;
            const int pu = t % PU, n = t / PU;
            const int row0 = (int)(n * img_rows) + pu * 256 + 128 * (int)rank;
            for (int kb = 0; kb < KB; ++kb, ++ia) {
                const int s = ia % SA;
                if (ia >= SA && !mbar_wait(emptyA + 8 * s, ((ia / SA) - 1) & 1, err, 1)) {
                    ok = false;
                    break;
                }
                if (rank == 0) mbar_arrive_expect_tx(fullA + 8 * s, 2u * (uint32_t)a_bytes);
                const uint32_t dst = smem_u32(sA + (size_t)s * a_stride);
                for (int ch = 0; ch < n_chunks; ++ch)
                    tma_load_2d_pair(dst + (uint32_t)(ch * chunk_rows * 128), &tmA, fullA0 + 8 * s, kb * 64,
                                     row0 + ch * chunk_rows);
            }
        }
        // rank 0's last barrier phases cover both CTAs' copies in flight
        if (rank == 0) {
            const int first = ia > SA ? ia - SA : 0;
            for (int j = first; j < ia; ++j) mbar_wait(fullA + 8 * (j % SA), (j / SA) & 1, err, 2);
        }
    } else if ((warp == 2 || warp == 3) && lane == 0) {
        // ---------------- weight chunks: two issuing warps, alternate ring entries ----------------
        const int me = warp - 2;
        int ib = 0;
        bool ok = true;
        for (int u = cid; u < n_units && ok; u += ncl) {
            const int g = u % ng;
            const int c0 = T.g_chunk0[g], c1 = c0 + T.g_nchunk[g];
            for (int kb = 0; kb < KB && ok; ++kb) {
                const int rowbase = T.g_brow[g] + kb * T.g_rows_kb[g];
                for (int c = c0; c < c1; ++c, ++ib) {
                    if ((ib & 1) != me) continue;
                    const int s = ib % SB;
                    if (ib >= SB && !mbar_wait(emptyB + 8 * s, ((ib / SB) - 1) & 1, err, 4)) {
                        ok = false;
                        break;
                    }
                    const int half = T.c_half[c];
                    if (rank == 0) mbar_arrive_expect_tx(fullB + 8 * s, 2u * (uint32_t)half * 128);
                    const uint32_t dst = smem_u32(sB + (size_t)s * b_slot);
                    const int row = rowbase + T.c_row0[c] + (int)rank * half;
                    for (int r = 0; r < half; r += BR)
                        tma_load_2d_pair(dst + (uint32_t)r * 128, &tmB, fullB0 + 8 * s, 0, row + r);
                }
            }
        }
        if (rank == 0) {
            const int first = ib > SB ? ib - SB : 0;
            for (int j = first; j < ib; ++j)
                if ((j & 1) == me) mbar_wait(fullB + 8 * (j % SB), (j / SB) & 1, err, 5);
        }
    } else if (warp == 1 && rank == 0) {
        // ---------------- MMA issue (rank 0) ----------------
        // The whole warp walks the loop, so every descriptor it computes is
        // warp-uniform (items are read from the kernel parameters with uniform
        // indices, ring positions advance by counters); one elected lane
        // issues the MMAs and commits.  A single-lane loop cannot keep
        // 64-cycle MMAs back to back.
        const bool issuer = elect_one();
        bool ok = true;
        int local = 0;
        uint32_t sa_slot = 0, sa_phase = 0, sb_slot = 0, sb_phase = 0;
        for (int u = cid; u < n_units && ok; u += ncl, ++local) {
            const int g = u % ng;
            const int c0 = T.g_chunk0[g], c1 = c0 + T.g_nchunk[g];
            const int buf = local & 1, use = local >> 1;
            if (use > 0) ok = __all_sync(0xffffffffu, mbar_wait(tempty + 8 * buf, (use - 1) & 1, err, 7));
            if (!ok) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + (uint32_t)buf * 256;
            for (int kb = 0; kb < KB; ++kb) {
                ok = __all_sync(0xffffffffu, mbar_wait(fullA + 8 * sa_slot, sa_phase, err, 8));
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA) + sa_slot * (uint32_t)a_stride;
                for (int c = c0; c < c1; ++c) {
                    ok = __all_sync(0xffffffffu, mbar_wait(fullB + 8 * sb_slot, sb_phase, err, 9));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t b_addr = smem_u32(sB) + sb_slot * (uint32_t)b_slot;
                    const int i1 = T.c_item0[c] + T.c_nitem[c];
                    for (int it = T.c_item0[c]; it < i1; ++it) {
                        const uint64_t bd = desc_kmajor_sw128(b_addr + (uint32_t)T.item[it].crow * 128);
                        const uint64_t ad = desc_kmajor_sw128(a_addr + (uint32_t)T.item[it].shift * 128);
                        const uint32_t idesc = idesc_f16_f32(256, T.item[it].n);
                        const uint32_t d = dbase + (uint32_t)T.item[it].tcol;
                        const uint32_t acc0 = (kb == 0 && T.item[it].first) ? 0u : 1u;
                        if (issuer) {
                            mma_f16_pair(d, ad, bd, idesc, acc0);
                            mma_f16_pair(d, ad + 2, bd + 2, idesc, 1u);
                            mma_f16_pair(d, ad + 4, bd + 4, idesc, 1u);
                            mma_f16_pair(d, ad + 6, bd + 6, idesc, 1u);
                        }
                        __syncwarp();
                    }
                    if (issuer) mma_commit_pair_mask(emptyB + 8 * sb_slot, 3);
                    __syncwarp();
                    if (++sb_slot == (uint32_t)SB) {
                        sb_slot = 0;
                        sb_phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (issuer) mma_commit_pair_mask(emptyA + 8 * sa_slot, 3);
                __syncwarp();
                if (++sa_slot == (uint32_t)SA) {
                    sa_slot = 0;
                    sa_phase ^= 1u;
                }
            }
            if (!ok) break;
            if (issuer) mma_commit_pair_mask(tfull + 8 * buf, 3);
            __syncwarp();
        }
        if (issuer) mma_commit_pair(mdone);
        __syncwarp();
        mbar_wait(mdone, 0, err, 10);
    } else if (warp >= 4) {
        // ---------------- epilogue (both CTAs) ----------------
        const int lane_base = 32 * (warp & 3);   // the TMEM lane quarter this warp may read
        const int eh = (warp - 4) >> 2;           // which alternate chunks of channels
        const int p = lane_base + lane;
        const int outy = T.outy, outx = T.outx, sy = T.sy, sx = T.sx, nJy = T.nJy, nJx = T.nJx;
        const int pair_x = T.pair_x;
        const bool has_bias = T.has_bias;
        const bool bias_vec = has_bias && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
        const long long plane = (long long)outy * outx;
        int local = 0;
        for (int u = cid; u < n_units; u += ncl, ++local) {
            const int g = u % ng;
            const int t = u / ng;
            const int pu = t % PU, n = t / PU;
            const int buf = local & 1, use = local >> 1;
            if (!mbar_wait(tfull + 8 * buf, use & 1, err, 11)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)buf * 256;
            const int F = pu * 256 + 128 * (int)rank + p;
            const int Jy = F / HX;
            const int Jx = F - Jy * HX;
            const bool pos_ok = Jx < nJx && Jy < nJy;
            const int ph0 = T.g_phase0[g], ph1 = ph0 + T.g_nphase[g];
            __half *yimg = y + (long long)n * M * plane;
            for (int ph = ph0; ph < ph1;) {
                const int ry = T.phase_r[ph][0], rx = T.phase_r[ph][1];
                const int oy = sy * Jy + ry;
                const int ox = sx * Jx + rx;
                const bool valid = pos_ok && oy < outy && ox < outx;
                const bool pair = pair_x && ph + 1 < ph1 && (rx & 1) == 0 && T.phase_r[ph + 1][0] == ry &&
                                  T.phase_r[ph + 1][1] == rx + 1;
                const uint32_t col0 = dbase + (uint32_t)((ph - ph0) * Np);
                __half *base = yimg + (long long)oy * outx + ox;
                // 32 channels per chunk; the two epilogue warps of a lane quarter
                // take alternate chunks
                for (int m0 = 32 * eh; m0 < Np; m0 += 64) {
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
                    __half *dst = base + (long long)m0 * plane;
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
                    if (pair) {
                        // both x phases of a channel are adjacent: one half2 per channel
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < mc0)
                                *reinterpret_cast<__half2 *>(dst + j * plane) =
                                    __floats2half2_rn(act_f<ACT>(__uint_as_float(v0[j]) + bb[j]),
                                                      act_f<ACT>(__uint_as_float(w0[j]) + bb[j]));
                        if (two) {
                            __half *d1 = dst + 16 * plane;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (j < mc1)
                                    *reinterpret_cast<__half2 *>(d1 + j * plane) =
                                        __floats2half2_rn(act_f<ACT>(__uint_as_float(v1[j]) + bb[16 + j]),
                                                          act_f<ACT>(__uint_as_float(w1[j]) + bb[16 + j]));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < mc0) dst[j * plane] = __float2half_rn(act_f<ACT>(__uint_as_float(v0[j]) + bb[j]));
                        if (two) {
                            __half *d1 = dst + 16 * plane;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (j < mc1)
                                    d1[j * plane] = __float2half_rn(act_f<ACT>(__uint_as_float(v1[j]) + bb[16 + j]));
                        }
                    }
                }
                ph += pair ? 2 : 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + 8 * buf);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no MMA, copy or remote arrival of the pair is still in flight
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

size_t pair_smem_bytes(const PairTables &T) {
    return 1024 + (size_t)T.SA * T.a_stride + (size_t)T.SB * T.b_slot + (size_t)((T.Np + 31) & ~31) * 4 +
           (size_t)(2 * T.SA + 2 * T.SB + 5) * 8 + 16;
}

// ---------------------------------------------------------------------------
// host planning

int round_up(int v, int m) { return (v + m - 1) / m * m; }

bool build_pair_tables(const Plan &p, PairTables &T) {
    if (p.dtype != CT_F16 || p.G != 1 || !p.tabled || p.layout != CT_NCHW) return false;
    if (p.C < 1 || p.C % 8 != 0 || p.M < 1 || p.M > 256 || p.N < 1 || p.N > 65535) return false;
    // one or two spatial axes: the leading axis is the trivial one of the plan
    if (p.in[0] != 1 || p.out[0] != 1 || p.s[0] != 1 || p.k[0] != 1) return false;
    if (p.taps[0][0].size() != 1 || p.taps[0][0][0].e != 0) return false;
    for (int a = 1; a < 3; ++a)
        if (p.in[a] < 1 || p.in[a] > (1 << 24) || p.out[a] > (1 << 24)) return false;
    if (p.in[1] * p.in[2] >= (1LL << 31)) return false;
    T.N = (int32_t)p.N;
    T.C = (int32_t)p.C;
    T.M = (int32_t)p.M;
    T.Np = (int32_t)((p.M + 15) / 16 * 16);
    T.KB = (int32_t)ceil_div(p.C, 64);
    T.H = (int32_t)p.in[1];
    T.W = (int32_t)p.in[2];
    T.outy = (int32_t)p.out[1];
    T.outx = (int32_t)p.out[2];
    T.sy = (int32_t)p.s[1];
    T.sx = (int32_t)p.s[2];
    T.pby = (int32_t)p.pb[1];
    T.pbx = (int32_t)p.pb[2];
    T.dy = (int32_t)p.d[1];
    T.dx = (int32_t)p.d[2];
    T.ky = (int32_t)p.k[1];
    T.kx = (int32_t)p.k[2];
    T.nJy = (int32_t)ceil_div(p.out[1], p.s[1]);
    T.nJx = (int32_t)ceil_div(p.out[2], p.s[2]);
    T.has_bias = p.has_bias;
    T.act = p.act;
    T.pair_x = (p.s[2] % 2 == 0) && (p.out[2] % 2 == 0);
    T.dead = has_dead_phases(p);
    // live phases, y-major
    int np = 0;
    for (int ry = 0; ry < p.s[1]; ++ry)
        for (int rx = 0; rx < p.s[2]; ++rx) {
            if (p.taps[1][ry].empty() || p.taps[2][rx].empty()) continue;
            if (np >= kPMaxPhases) return false;
            T.phase_r[np][0] = (int16_t)ry;
            T.phase_r[np][1] = (int16_t)rx;
            ++np;
        }
    if (np == 0) return false;
    T.n_phases = np;
    // groups: whole rows of phases (same ry) merged while within 256 accumulator columns
    const int per = 256 / T.Np;
    int ng = 0;
    for (int ph = 0; ph < np;) {
        int end = ph;
        while (end < np) {
            int row_end = end + 1;
            while (row_end < np && T.phase_r[row_end][0] == T.phase_r[end][0]) ++row_end;
            if (row_end - ph <= per)
                end = row_end;
            else
                break;
        }
        if (end == ph) {
            end = ph + 1;
            while (end < np && end - ph < per && T.phase_r[end][0] == T.phase_r[ph][0]) ++end;
        }
        if (ng >= kPMaxGroups) return false;
        T.g_phase0[ng] = (int16_t)ph;
        T.g_nphase[ng] = (int16_t)(end - ph);
        ++ng;
        ph = end;
    }
    T.n_groups = ng;
    // padded origin and extents from the offsets of every live tap
    int lo[2] = {1 << 20, 1 << 20}, hi[2] = {-(1 << 20), -(1 << 20)};
    for (int ph = 0; ph < np; ++ph)
        for (int a = 0; a < 2; ++a)
            for (const Tap &t : p.taps[1 + a][T.phase_r[ph][a]]) {
                lo[a] = std::min(lo[a], (int)t.e);
                hi[a] = std::max(hi[a], (int)t.e);
            }
    const int span_y = hi[0] - lo[0], span_x = hi[1] - lo[1];
    T.emin_y = lo[0];
    T.emin_x = lo[1];
    const long long HX = (long long)T.nJx + span_x, HYp = (long long)T.nJy + span_y;
    const long long maxshift = span_y * HX + span_x;
    if (maxshift + 128 > kPMaxTileRows) return false;
    T.HX = (int32_t)HX;
    T.HYp = (int32_t)HYp;
    int tile = round_up((int)maxshift + 128, 8);
    T.n_chunks = (tile + 255) / 256;
    T.chunk_rows = round_up((tile + T.n_chunks - 1) / T.n_chunks, 8);
    T.tile_rows = T.chunk_rows * T.n_chunks;
    T.a_bytes = T.tile_rows * 128;
    T.a_stride = round_up(T.a_bytes, 1024);
    const long long plane_pos = (long long)T.nJy * HX;
    T.PU = (int32_t)ceil_div(plane_pos, 256);
    if ((long long)T.N * HYp * HX + T.tile_rows + 256 >= (1LL << 31)) return false;
    const long long units = (long long)T.N * T.PU * ng;
    if (units > (1LL << 30)) return false;
    T.n_units = (int32_t)units;
    // shared memory: three input stages (two when they do not fit) and at
    // least two weight chunks of at most 256 rows per rank.  Measured on the
    // 2-D decoder workload, three 34 KB input stages with three 32 KB chunk
    // slots beat two input stages with 64 KB chunks: the loads, not the
    // MMAs, set the pace there.
    const int fixed = 1024 + ((T.Np + 31) & ~31) * 4 + (2 * 4 + 2 * 12 + 5) * 8 + 16;
    T.SA = (kPSmemBudget - fixed - 3LL * T.a_stride) / 2 >= 128 * 128 ? 3 : 2;
    const long long b_room = (kPSmemBudget - fixed - (long long)T.SA * T.a_stride) / 2;   // bytes of one chunk
    const int ch_max = (int)std::min<long long>(256, b_room / 128 / 8 * 8);                // rows per rank
    if (ch_max < 128) return false;
    // items per group: (phase, tap) pairs grouped by input offset, offsets
    // shared by more phases first, adjacent phases merged into one wide MMA;
    // then consecutive items gathered into chunks of at most ch_max rows per rank
    int ni = 0, nc = 0, rows_total = 0;
    for (int g = 0; g < ng; ++g) {
        struct PairRec { int ph, ey, ex; };
        std::vector<PairRec> pairs;
        for (int ph = T.g_phase0[g]; ph < T.g_phase0[g] + T.g_nphase[g]; ++ph)
            for (const Tap &a : p.taps[1][T.phase_r[ph][0]])
                for (const Tap &b : p.taps[2][T.phase_r[ph][1]]) pairs.push_back({ph, a.e, b.e});
        std::vector<std::array<int, 2>> offs;
        for (auto &q : pairs) offs.push_back({q.ey, q.ex});
        std::sort(offs.begin(), offs.end());
        offs.erase(std::unique(offs.begin(), offs.end()), offs.end());
        auto nph = [&](const std::array<int, 2> &e) {
            int c = 0;
            for (auto &q : pairs) c += (q.ey == e[0] && q.ex == e[1]);
            return c;
        };
        std::stable_sort(offs.begin(), offs.end(),
                         [&](const std::array<int, 2> &a, const std::array<int, 2> &b) { return nph(a) > nph(b); });
        std::vector<char> touched(np, 0);
        T.g_item0[g] = (int16_t)ni;
        int brow = 0;   // weight rows of the group per channel block
        for (auto &e : offs) {
            std::vector<int> phs;
            for (auto &q : pairs)
                if (q.ey == e[0] && q.ex == e[1]) phs.push_back(q.ph);
            std::sort(phs.begin(), phs.end());
            size_t i = 0;
            while (i < phs.size()) {
                size_t j = i + 1;
                while (j < phs.size() && phs[j] == phs[j - 1] + 1 && touched[phs[j]] == touched[phs[i]] &&
                       (int)(j - i + 1) * T.Np <= 256)
                    ++j;
                if (ni >= kPMaxItems) return false;
                PItem &I = T.item[ni];
                I.e[0] = (int16_t)e[0];
                I.e[1] = (int16_t)e[1];
                I.n = (int16_t)((j - i) * T.Np);
                I.shift = (int32_t)((e[0] - lo[0]) * HX + (e[1] - lo[1]));
                I.tcol = (int16_t)((phs[i] - T.g_phase0[g]) * T.Np);
                I.phase0 = (int16_t)phs[i];
                I.first = touched[phs[i]] ? 0 : 1;
                I.crow = 0;
                I.pad = 0;
                brow += I.n;
                for (size_t q = i; q < j; ++q) touched[phs[q]] = 1;
                ++ni;
                i = j;
            }
        }
        T.g_nitem[g] = (int16_t)(ni - T.g_item0[g]);
        T.g_brow[g] = rows_total;
        T.g_rows_kb[g] = brow;
        rows_total += brow * T.KB;
        // chunks
        T.g_chunk0[g] = (int16_t)nc;
        int row0 = 0;
        for (int it = T.g_item0[g]; it < ni;) {
            if (nc >= kPMaxChunks) return false;
            int half = 0, jt = it;
            while (jt < ni && half + T.item[jt].n / 2 <= ch_max) {
                T.item[jt].crow = (int16_t)half;
                half += T.item[jt].n / 2;
                ++jt;
            }
            T.c_item0[nc] = (int16_t)it;
            T.c_nitem[nc] = (int16_t)(jt - it);
            T.c_row0[nc] = row0;
            T.c_half[nc] = half;
            row0 += 2 * half;
            ++nc;
            it = jt;
        }
        T.g_nchunk[g] = (int16_t)(nc - T.g_chunk0[g]);
    }
    T.n_items = ni;
    T.total_rows = rows_total;
    // weight loads: a CTA's half of a chunk is contiguous, loaded in boxes of BR rows
    int br = 256, hmax = 0;
    for (int c = 0; c < nc; ++c) {
        while (T.c_half[c] % br) br /= 2;
        hmax = std::max(hmax, (int)T.c_half[c]);
    }
    if (br < 8) return false;
    T.BR = br;
    T.b_slot = round_up(hmax * 128, 1024);
    // as many weight chunk slots as fit (at least two)
    const long long sb = (kPSmemBudget - fixed - (long long)T.SA * T.a_stride) / T.b_slot;
    if (sb < 2) return false;
    T.SB = (int)std::min<long long>(sb, 12);
    return pair_smem_bytes(T) <= (size_t)kPSmemBudget;
}

// Clusters of two that can be resident at once (one CTA per SM).
template <typename K>
int resident_pairs(K kernel, int smem) {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return 1;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 1024, 1, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sm_count() / 2;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Dynamic shared memory of a launch: at least 120 KB, so that no two CTAs
// share an SM (two pairs waiting on each other's TMEM could never proceed).
size_t pair_launch_smem(const PairTables &T) { return std::max<size_t>(pair_smem_bytes(T), 120 * 1024); }

template <int ACT>
ct_status launch_pair(const PairTables &T, const CUtensorMap &tmA, const CUtensorMap &tmB, const void *bias,
                      void *y, cudaStream_t st) {
    static std::atomic<int> attr_set[64];
    if (!allow_smem(dense_pair_kernel<ACT>, attr_set, kPSmemBudget)) return CT_ERR_DEVICE;
    const size_t smem = pair_launch_smem(T);
    int pairs = resident_pairs(dense_pair_kernel<ACT>, (int)smem);
    if (pairs > T.n_units) pairs = T.n_units;
    dense_pair_kernel<ACT><<<2 * pairs, kPThreads, smem, st>>>(tmA, tmB, T, (const __half *)bias, (__half *)y);
    return launch_status();
}

}  // namespace

bool dense_pair_supports(const Plan &p) {
    PairTables *T = new PairTables();
    const bool ok = build_pair_tables(p, *T);
    delete T;
    return ok;
}

void dense_pair_setup(Plan &p) {
    p.aux.assign((sizeof(PairTables) + 7) / 8, 0);
    PairTables &T = *reinterpret_cast<PairTables *>(p.aux.data());
    build_pair_tables(p, T);
    p.launches = 2 + (T.dead ? 1 : 0);
}

size_t dense_pair_packed_bytes(const Plan &p) { return (size_t)ptables(p).total_rows * 128; }

size_t dense_pair_ws_bytes(const Plan &p) {
    const PairTables &T = ptables(p);
    return (size_t)T.N * T.HYp * T.HX * T.C * 2;
}

ct_status dense_pair_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const PairTables &T = ptables(p);
    const long long total = (long long)T.total_rows * 64;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    pair_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(T, (const __half *)w, (__half *)wp);
    return launch_status();
}

ct_status dense_pair_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y, void *ws,
                         cudaStream_t st) {
    const PairTables &T = ptables(p);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CT_ERR_DEVICE;
    {
        const long long S = (long long)T.H * T.W;
        const long long tiles = ceil_div(S, kPadS);
        if (tiles + 1 > 0x7fffffffLL || ceil_div(T.C, kPadC) > 65535 || S >= (1LL << 31)) return CT_ERR_UNSUPPORTED;
        dim3 grid((unsigned)(tiles + 1), (unsigned)ceil_div(T.C, kPadC), (unsigned)T.N);
        nchw_to_padded_kernel<<<grid, 256, 0, st>>>((const __half *)x, (__half *)ws, T.C, T.H, T.W, T.HYp, T.HX,
                                                    -T.emin_y, -T.emin_x);
        ct_status s1 = launch_status();
        if (s1 != CT_OK) return s1;
    }
    CUtensorMap tmA, tmB;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)T.C, (cuuint64_t)T.N * T.HYp * T.HX};
        const cuuint64_t strides[1] = {(cuuint64_t)T.C * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)T.chunk_rows};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ws, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
    if (T.act == CT_ACT_RELU) return launch_pair<CT_ACT_RELU>(T, tmA, tmB, bias, y, st);
    return launch_pair<CT_ACT_IDENTITY>(T, tmA, tmB, bias, y, st);
}

}  // namespace ct
