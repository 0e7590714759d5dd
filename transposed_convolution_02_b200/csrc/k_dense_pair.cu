// Dense ConvTranspose (group 1, any rank, channels-first or channels-last;
// fp16, or fp32 as 3xTF32) on pairs of SMs: every tcgen05 MMA spans the two
// CTAs of a cluster (cta_group::2, M = 256 positions).  Each SM reads its own
// 128 positions of A and only HALF of every weight tile from its shared
// memory, and keeps the accumulators of its 128 positions in its TMEM,
// double-buffered, so a unit's epilogue runs under the next unit's MMAs.
// Output channels come in tiles of at most 256 (one MMA's N).
//
// Phases as in the halo kernel: output o = s*J + r per axis; tap k of phase r
// reads input i = J + e, e = (r + pad_begin - k*d) / s (ai.onnx.ConvTranspose
// README, implementation notes on the tap-reversed stride-1 form and the
// grouped stride-phase variant).
//
// Input staging: X is re-laid (channels-first) or copied (channels-last)
// into a zero-padded channels-last copy Xp[n][zp][yp][xp][c] with c padded to
// a 16-byte row, zp = iz - emin_z, yp = iy - emin_y, xp = ix - emin_x
// (emin the smallest input offset of any tap per axis), HX = nJx + span_x
// columns, HY = nJy + span_y rows and HZ = nJz + span_z slices per image.
// Output position (Jy, Jx) of slice Jz is numbered F = Jy*HX + Jx, and its
// input under offset (ez, ey, ex) is row F + (ey - emin_y)*HX + (ex - emin_x)
// of padded slice Jz + ez - emin_z.  So a CTA's 128 positions need, per
// slice, ONE contiguous run of 128 + span_y*HX + span_x rows (plain 2-D TMA
// boxes); the span_z + 1 runs sit one after the other in shared memory, both
// CTAs of a pair place them at the same offsets, and every tap of every phase
// is the same rows shifted by a constant (slices count slice_rows rows).
//
// Warps: 0 loads input runs, 1 allocates TMEM (both CTAs) and issues MMAs
// (rank 0), 2-3 load weight chunks, 4-11 drain TMEM (both CTAs; two warps
// per TMEM lane quarter taking alternate (phase, 32-channel) pieces).
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
    int32_t shift;    // shared-memory rows from a position to its input under this offset
    int16_t n;        // MMA N: phases of the run x Np (each CTA holds n/2 weight rows)
    int16_t tcol;     // first accumulator column of the run
    int16_t first;    // first write of these columns (at channel block 0)
    int16_t phase0;   // first phase of the run
    int16_t e[3];     // input offset (z, y, x)
    int16_t crow;     // first row of the item's half inside its chunk's half (either rank)
};

struct PadGeo {
    int C, D, H, W;      // input extents
    int Cd;              // channels of a padded position (C rounded up to a 16-byte row)
    int HZ, HY, HX;      // padded extents
    int oz, oy, ox;      // padded origin: zp = iz + oz, ...
    int halo_blocks;     // blocks x = 0..halo_blocks-1 write the zero halo
};

struct PairTables {
    int32_t N, C, M, Np, KB;
    // f32: fp32 operands as a TF32 high part and its remainder (3xTF32: three
    // MMAs per step), 32 channels per 128-byte row; otherwise fp16, 64 channels
    int32_t f32, cpb, parts;            // parts: 2 (high, low) for f32, else 1
    int32_t nhwc;                       // channels-last X, W ([C, k.., M]) and Y
    // output channels in n_mt tiles of Mt (= Np) channels; every tile has the
    // same groups and items, and its own total_rows of packed weights
    int32_t Mt, n_mt, BL;               // BL: bias entries kept in shared memory
    int32_t Cd;                         // channels of a padded position: C rounded up to a 16-byte row
    int32_t in[3], out[3], s[3], pb[3], d[3], k[3], nJ[3];   // axes z, y, x
    int32_t emin[3], HX, HY, HZ;
    int32_t n_slices, slice_rows, chunk_rows, n_chunks, a_bytes, a_stride;
    int32_t SA, SB, b_slot, BR, BRs;   // weight boxes: BR rows, then BRs rows for a chunk's remainder
    int32_t PU, n_units, n_groups, n_phases, n_items, total_rows;
    int32_t has_bias, dead, pair_x, act;
    int16_t phase_r[kPMaxPhases][3];   // (rz, ry, rx) of every live phase
    int16_t g_phase0[kPMaxGroups], g_nphase[kPMaxGroups], g_item0[kPMaxGroups], g_nitem[kPMaxGroups];
    int32_t g_brow[kPMaxGroups], g_rows_kb[kPMaxGroups];
    int16_t g_chunk0[kPMaxGroups], g_nchunk[kPMaxGroups];
    // a chunk: consecutive items of a group whose weights one barrier covers;
    // inside one channel block its rows are [row0, row0 + parts*half) for
    // rank 0, then the same count for rank 1; with two parts a rank's block
    // holds the high parts (half rows), then the low parts
    int16_t c_item0[kPMaxChunks], c_nitem[kPMaxChunks];
    int32_t c_row0[kPMaxChunks], c_half[kPMaxChunks];
    PItem item[kPMaxItems];
};

__device__ int g_dense_pair_err;

const PairTables &ptables(const Plan &p) { return *reinterpret_cast<const PairTables *>(p.aux.data()); }

// ---------------------------------------------------------------------------
// weight pre-pack: rows of every group, channel block, chunk, rank (and part)
// in the order the kernel loads them; a row holds the 64 (fp16) or 32 (fp32)
// input channels of one output channel m of one phase at one channel block,
// W[kb*cpb + cc][m][kz][ky][kx] at the phase's tap for the item's offset, zero
// outside C and M.  Rows [0, n/2) of an item's N columns feed the pair's
// rank 0, rows [n/2, n) rank 1.  For fp32 a weight w is stored as its TF32
// high part h (low 13 mantissa bits cleared) and the remainder w - h.

__device__ __forceinline__ float tf32_high(float v) { return __uint_as_float(__float_as_uint(v) & 0xffffe000u); }

template <typename E>
__global__ void __launch_bounds__(256) pair_prepack_kernel(const __grid_constant__ PairTables T,
                                                           const E *__restrict__ w, E *__restrict__ wp) {
    const int cpb = T.cpb, parts = T.parts;
    const long long total = (long long)T.n_mt * T.total_rows * cpb;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int cc = (int)(i % cpb);
        const int row_all = (int)(i / cpb);
        const int mt = row_all / T.total_rows;   // output-channel tile
        const int row = row_all - mt * T.total_rows;
        int g = 0;
        while (g + 1 < T.n_groups && row >= T.g_brow[g + 1]) ++g;
        const int rg = row - T.g_brow[g];
        const int kb = rg / T.g_rows_kb[g];
        const int rk = rg % T.g_rows_kb[g];
        int c = T.g_chunk0[g];
        const int c1 = T.g_chunk0[g] + T.g_nchunk[g];
        while (c + 1 < c1 && rk >= T.c_row0[c + 1]) ++c;
        const int half = T.c_half[c];
        const int r2 = rk - T.c_row0[c];
        const int rank = r2 >= parts * half ? 1 : 0;
        const int r3 = r2 - rank * parts * half;
        const int part = r3 >= half ? 1 : 0;   // 1: the remainder (fp32 only)
        const int r4 = r3 - part * half;
        int it = T.c_item0[c];
        const int i1 = T.c_item0[c] + T.c_nitem[c];
        while (it + 1 < i1 && r4 >= T.item[it + 1].crow) ++it;
        const PItem &I = T.item[it];
        const int rr = rank * (I.n / 2) + (r4 - I.crow);
        const int ph = I.phase0 + rr / T.Np;
        const int m = mt * T.Mt + rr % T.Np;   // output channel
        const int ci = kb * cpb + cc;
        float v = 0.f;
        if (ci < T.C && m < T.M) {
            long long kpos = 0;
            bool ok = true;
            for (int a = 0; a < 3; ++a) {
                const int num = T.phase_r[ph][a] + T.pb[a] - I.e[a] * T.s[a];
                const int ka = num / T.d[a];
                ok = ok && num % T.d[a] == 0 && ka >= 0 && ka < T.k[a];
                kpos = kpos * T.k[a] + ka;
            }
            const long long ksz = (long long)T.k[0] * T.k[1] * T.k[2];
            if (ok) v = (float)(T.nhwc ? w[((long long)ci * ksz + kpos) * T.M + m] : w[((long long)ci * T.M + m) * ksz + kpos]);
        }
        if (parts == 2) v = part ? v - tf32_high(v) : tf32_high(v);
        wp[i] = (E)v;
    }
}

// ---------------------------------------------------------------------------
// X[n][c][iz][iy][ix] -> Xp[n][iz + oz][iy + oy][ix + ox][c] (positions
// outside the padded image dropped), plus zeros at every padded position no
// input lands on.  The first halo_blocks blocks along x write the zero halo
// of image blockIdx.z for the 64-channel block blockIdx.y; the others move a
// tile of 64 channels x 128 input positions each (as the plain channels-last
// re-layout, XOR-swizzled exchange).

constexpr int kPadC = 64, kPadS = 128;

// Zero the halo of one image's padded copy, a padded row (zp, yp) at a time:
// rows outside the input are zero for their whole width, the others only in
// the columns left and right of the input.  Warp `wid` of `nw` takes rows
// round-robin; `zero(pos, q)` writes 16-byte chunk q of padded position pos,
// `chunks` of them per position.  One row decode per warp and row, then
// contiguous chunk runs (no per-chunk division beyond the chunk count).
template <typename F>
__device__ __forceinline__ void zero_halo_rows(const PadGeo &g, int wid, int nw, int lane, int chunks, F zero) {
    const int rows = g.HZ * g.HY;
    const int xl = min(max(g.ox, 0), g.HX);              // left halo columns [0, xl)
    const int xr = min(max(g.ox + g.W, xl), g.HX);       // right halo columns [xr, HX)
    for (int row = wid; row < rows; row += nw) {
        const int zp = row / g.HY, yp = row - zp * g.HY;
        const bool full = zp < g.oz || zp >= g.oz + g.D || yp < g.oy || yp >= g.oy + g.H;
        const long long rowpos = (long long)row * g.HX;
        for (int seg = 0; seg < 2; ++seg) {
            const int a = full ? (seg == 0 ? 0 : g.HX) : (seg == 0 ? 0 : xr);
            const int b = full ? (seg == 0 ? g.HX : g.HX) : (seg == 0 ? xl : g.HX);
            const int nq = (b - a) * chunks;
            for (int q = lane; q < nq; q += 32) {
                const int pc = q / chunks;
                zero(rowpos + a + pc, q - pc * chunks);
            }
        }
    }
}

// Blocks that zero the halo: about eight padded rows per warp (64 per block
// of eight warps), so that halo and tile blocks together stay within one
// wave of resident blocks for the workloads' sizes (a second, partial wave
// measured as the re-layout's tail).
inline int halo_blocks_for(const PadGeo &g) {
    const long long rows = (long long)g.HZ * g.HY;
    return (int)std::max<long long>(1, std::min<long long>(256, ceil_div(rows, 64)));
}

// The padded re-layout of image n, one block of 256 threads per task (t is
// the thread's index; `bar` the barrier the tile steps synchronise on, 0 for
// the whole block): halo task h (0 <= h < halo_blocks) zeroes padded rows of
// channel block cb; tile task st moves 64 channels x 128 input positions of
// channel block cb through the 16 KB shared tile: its four 16-byte loads per
// thread, then the 8x8-block transpose in shared memory and the stores.
__device__ __forceinline__ void padded_halo(__half *__restrict__ xp, const PadGeo &g, int n, int cb, int halo, int t) {
    const int Cd = g.Cd;
    const long long P = (long long)g.HZ * g.HY * g.HX;
    const int c0 = cb * kPadC;
    const int c8 = (min(kPadC, Cd - c0)) >> 3;
    __half *img = xp + (long long)n * P * Cd + c0;
    zero_halo_rows(g, halo * 8 + (t >> 5), g.halo_blocks * 8, t & 31, c8,
                   [&](long long pos, int q) {
                       *reinterpret_cast<uint4 *>(img + pos * Cd + q * 8) = make_uint4(0, 0, 0, 0);
                   });
}

__device__ __forceinline__ void padded_tile_load(const __half *__restrict__ x, const PadGeo &g, int n, int cb, int st,
                                                 int t, uint4 (&v)[4]) {
    const int C = g.C;
    const long long S = (long long)g.D * g.H * g.W;
    const int c0 = cb * kPadC;
    const long long s0 = (long long)st * kPadS;
    const bool vec = (S & 7) == 0;
    const int cl = t >> 4, sv = t & 15;
    const long long s = s0 + sv * 8;
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
}

__device__ __forceinline__ void padded_tile_finish(const uint4 (&v)[4], __half *__restrict__ xp, const PadGeo &g,
                                                   int n, int cb, int st, __half *tile, int t, int bar) {
    const int Cd = g.Cd, H = g.H, W = g.W, HY = g.HY, HX = g.HX;
    const long long HW = (long long)H * W;
    const long long S = g.D * HW;
    const long long P2 = (long long)HY * HX;
    const long long P = g.HZ * P2;
    const int c0 = cb * kPadC;
    const long long s0 = (long long)st * kPadS;
    {
        const int cl = t >> 4, sv = t & 15;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int row = cl + 16 * r;
            *reinterpret_cast<uint4 *>(tile + row * kPadS + ((sv ^ (row & 7)) * 8)) = v[r];
        }
    }
    sm100::group_sync(bar);
    // [64 channels][128 positions] -> [128 positions][64 channels], in place
    sm100::transpose_64x128_b16(reinterpret_cast<uint16_t *>(tile), t >> 5, t & 31, bar);
    {
        const int sl = t >> 3, cv = t & 7;
        const int c = c0 + cv * 8;
        // this thread's positions are s0 + sl + 32 r: decode the first, then step
        int iz = (int)(s0 + sl) / (int)HW;                        // S < 2^31
        int iy = ((int)(s0 + sl) - iz * (int)HW) / W;
        int ix = (int)(s0 + sl) - iz * (int)HW - iy * W;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (r > 0) {
                ix += 32;
                while (ix >= W) {
                    ix -= W;
                    if (++iy == H) {
                        iy = 0;
                        ++iz;
                    }
                }
            }
            const int sp = sl + 32 * r;
            const long long s = s0 + sp;
            if (s >= S || c >= Cd) continue;   // channels C..Cd of the row are zeros
            const int zp = iz + g.oz, yp = iy + g.oy, xq = ix + g.ox;
            if (zp < 0 || zp >= g.HZ || yp < 0 || yp >= HY || xq < 0 || xq >= HX) continue;
            *reinterpret_cast<uint4 *>(xp + ((long long)n * P + zp * P2 + (long long)yp * HX + xq) * Cd + c) =
                *reinterpret_cast<const uint4 *>(tile + sp * 64 + ((cv ^ (sp & 7)) * 8));
        }
    }
    sm100::group_sync(bar);   // the tile may be reused by the group's next task
}

__global__ void __launch_bounds__(256) nchw_to_padded_kernel(const __half *__restrict__ x,
                                                             __half *__restrict__ xp, const PadGeo g) {
    __shared__ __align__(128) __half tile[kPadC * kPadS];
    sm100::griddep_launch_dependents();   // the pair kernel may set up while this one runs
    if ((int)blockIdx.x < g.halo_blocks) {
        padded_halo(xp, g, blockIdx.z, blockIdx.y, blockIdx.x, threadIdx.x);
        return;
    }
    uint4 v[4];
    const int st = (int)blockIdx.x - g.halo_blocks;
    padded_tile_load(x, g, blockIdx.z, blockIdx.y, st, threadIdx.x, v);
    padded_tile_finish(v, xp, g, blockIdx.z, blockIdx.y, st, tile, threadIdx.x, 0);
}

// fp32: X -> two padded channels-last planes, the TF32 high parts and the
// remainders (3xTF32 operands); tiles of 32 channels x 128 positions, halo
// blocks as above.  The shared tile has a pitch of 129 words, so the column
// reads of a warp fall in 32 different banks.
constexpr int kPadC32 = 32;

__global__ void __launch_bounds__(256) nchw_to_padded_f32_kernel(const float *__restrict__ x,
                                                                 float *__restrict__ xh, float *__restrict__ xl,
                                                                 const PadGeo g) {
    const int n = blockIdx.z;
    const int C = g.C, Cd = g.Cd, H = g.H, W = g.W, HY = g.HY, HX = g.HX;
    const long long HW = (long long)H * W;
    const long long S = g.D * HW;
    const long long P2 = (long long)HY * HX;
    const long long P = g.HZ * P2;
    const int t = threadIdx.x;
    sm100::griddep_launch_dependents();   // the pair kernel may set up while this one runs
    if ((int)blockIdx.x < g.halo_blocks) {
        const int c0 = blockIdx.y * kPadC32;
        const int c4 = (min(kPadC32, Cd - c0)) >> 2;
        const long long base = (long long)n * P * Cd + c0;
        zero_halo_rows(g, (int)blockIdx.x * 8 + (t >> 5), g.halo_blocks * 8, t & 31, c4,
                       [&](long long pos, int q) {
                           const long long off = base + pos * Cd + q * 4;
                           *reinterpret_cast<float4 *>(xh + off) = make_float4(0.f, 0.f, 0.f, 0.f);
                           *reinterpret_cast<float4 *>(xl + off) = make_float4(0.f, 0.f, 0.f, 0.f);
                       });
        return;
    }
    __shared__ float tile[kPadC32][kPadS + 1];
    const int c0 = blockIdx.y * kPadC32;
    const long long s0 = (long long)(blockIdx.x - g.halo_blocks) * kPadS;
    const bool vec = (S & 3) == 0;
    {
        // 8 threads per channel row, 16 positions each
        const int cl = t >> 3, sv = t & 7;
        const int c = c0 + cl;
        const long long s = s0 + sv * 16;
        const float *src = x + ((long long)n * C + c) * S + s;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 v;
            if (vec && c < C && s + 4 * j + 4 <= S) {
                v = __ldg(reinterpret_cast<const float4 *>(src) + j);
            } else {
                const long long b = s + 4 * j;
                v.x = (c < C && b < S) ? src[4 * j] : 0.f;
                v.y = (c < C && b + 1 < S) ? src[4 * j + 1] : 0.f;
                v.z = (c < C && b + 2 < S) ? src[4 * j + 2] : 0.f;
                v.w = (c < C && b + 3 < S) ? src[4 * j + 3] : 0.f;
            }
            float *d = &tile[cl][sv * 16 + 4 * j];
            d[0] = v.x;
            d[1] = v.y;
            d[2] = v.z;
            d[3] = v.w;
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        // a task: one position and 4 channels
        const int task = t + 256 * r;
        const int q = task & 7, sp = task >> 3;
        const long long s = s0 + sp;
        const int c = c0 + 4 * q;
        if (s >= S || c >= Cd) continue;   // channels C..Cd of the row are zeros
        const int iz = (int)s / (int)HW;   // S < 2^31
        const int rem = (int)s - iz * (int)HW;
        const int iy = rem / W, ix = rem - iy * W;
        const int zp = iz + g.oz, yp = iy + g.oy, xq = ix + g.ox;
        if (zp < 0 || zp >= g.HZ || yp < 0 || yp >= HY || xq < 0 || xq >= HX) continue;
        const float4 v = make_float4(tile[4 * q][sp], tile[4 * q + 1][sp], tile[4 * q + 2][sp], tile[4 * q + 3][sp]);
        const float4 hi = make_float4(tf32_high(v.x), tf32_high(v.y), tf32_high(v.z), tf32_high(v.w));
        const long long off = ((long long)n * P + zp * P2 + (long long)yp * HX + xq) * Cd + c;
        *reinterpret_cast<float4 *>(xh + off) = hi;
        *reinterpret_cast<float4 *>(xl + off) = make_float4(v.x - hi.x, v.y - hi.y, v.z - hi.z, v.w - hi.w);
    }
}

// Channels-last X[n][iz][iy][ix][c] -> the same padded copy(ies): a copy of
// 16-byte channel pieces (fp32: split into high parts and remainders), with
// the zero halo written by the first halo_blocks blocks as above.
template <typename E>
__global__ void __launch_bounds__(256) nhwc_to_padded_kernel(const E *__restrict__ x, E *__restrict__ xh,
                                                             E *__restrict__ xl, const PadGeo g) {
    constexpr int kPer = 16 / sizeof(E);   // elements per 16-byte piece
    const int n = blockIdx.z;
    const int C = g.C, H = g.H, W = g.W, HY = g.HY, HX = g.HX;
    const long long HW = (long long)H * W;
    const long long S = g.D * HW;
    const long long P2 = (long long)HY * HX;
    const long long P = g.HZ * P2;
    const int t = threadIdx.x;
    const int cch = C / kPer;   // pieces per position
    sm100::griddep_launch_dependents();   // the pair kernel may set up while this one runs
    if ((int)blockIdx.x < g.halo_blocks) {
        const long long base = (long long)n * P * C;
        zero_halo_rows(g, (int)blockIdx.x * 8 + (t >> 5), g.halo_blocks * 8, t & 31, cch,
                       [&](long long pos, int q) {
                           const long long off = base + pos * C + (long long)q * kPer;
                           *reinterpret_cast<uint4 *>(xh + off) = make_uint4(0, 0, 0, 0);
                           if (xl) *reinterpret_cast<uint4 *>(xl + off) = make_uint4(0, 0, 0, 0);
                       });
        return;
    }
    const long long work = S * cch;
    const long long stride = (long long)(gridDim.x - g.halo_blocks) * blockDim.x;
    for (long long q = (long long)(blockIdx.x - g.halo_blocks) * blockDim.x + t; q < work; q += stride) {
        const long long sidx = q / cch;
        const int cc = (int)(q - sidx * cch);
        const int iz = (int)sidx / (int)HW;   // S < 2^31
        const int rem = (int)sidx - iz * (int)HW;
        const int iy = rem / W, ix = rem - iy * W;
        const int zp = iz + g.oz, yp = iy + g.oy, xq = ix + g.ox;
        if (zp < 0 || zp >= g.HZ || yp < 0 || yp >= HY || xq < 0 || xq >= HX) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + ((long long)n * S + sidx) * C) + cc);
        const long long off = ((long long)n * P + zp * P2 + (long long)yp * HX + xq) * C + (long long)cc * kPer;
        if (xl) {
            // fp32: the TF32 high parts and the remainders
            const float4 f = *reinterpret_cast<const float4 *>(&v);
            const float4 hi = make_float4(tf32_high(f.x), tf32_high(f.y), tf32_high(f.z), tf32_high(f.w));
            *reinterpret_cast<float4 *>(xh + off) = hi;
            *reinterpret_cast<float4 *>(xl + off) = make_float4(f.x - hi.x, f.y - hi.y, f.z - hi.z, f.w - hi.w);
        } else {
            *reinterpret_cast<uint4 *>(xh + off) = v;
        }
    }
}

// ---------------------------------------------------------------------------
// A unit: image n, output slice jz, group g, pair positions [pu*256, +256) of
// the slice; rank r of the pair owns [pu*256 + 128*r, +128).  Units are
// walked cluster-strided.
// Every role reads the tables from the kernel parameters with warp-uniform
// indices; nothing but the bias is copied to shared memory.

template <int ACT>
__device__ __forceinline__ float act_f(float v) {
    return apply_act(v, ACT);
}

// Output stores of the epilogue for fp16 and fp32 elements.
__device__ __forceinline__ void st_pair(__half *p, float a, float b) {
    *reinterpret_cast<__half2 *>(p) = __floats2half2_rn(a, b);
}
// fp32 outputs are written through to memory: with 3xTF32 the output stream
// is far larger than L2 (the 1-D vocoder workload writes 268 MB), and
// write-through keeps it from evicting the weight chunks that every unit
// re-reads (measured: 665 -> 647 us per call on that workload; fp16 outputs,
// which fit in L2 for the workloads, measured slower with it).
__device__ __forceinline__ void st_pair(float *p, float a, float b) {
    asm volatile("st.global.wt.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void st_one(__half *p, float a) { *p = __float2half_rn(a); }
__device__ __forceinline__ void st_one(float *p, float a) { *p = a; }
// 32 bias values from global memory (16-byte aligned source)
__device__ __forceinline__ void ld_bias32(const __half *b, float (&bb)[32]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 h = __ldg(reinterpret_cast<const uint4 *>(b) + j);
        const __half2 *h2 = reinterpret_cast<const __half2 *>(&h);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(h2[q]);
            bb[8 * j + 2 * q] = f.x;
            bb[8 * j + 2 * q + 1] = f.y;
        }
    }
}
__device__ __forceinline__ void ld_bias32(const float *b, float (&bb)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(b) + j);
        bb[4 * j] = f.x;
        bb[4 * j + 1] = f.y;
        bb[4 * j + 2] = f.z;
        bb[4 * j + 3] = f.w;
    }
}

// 16 consecutive channels of one channels-last position: 16-byte stores when
// the row is whole and aligned, else element by element.
template <int ACT>
__device__ __forceinline__ void store_row16(__half *dst, const uint32_t (&v)[16], const float *b, int mc) {
    if (mc == 16 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
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
            if (j < mc) dst[j] = __float2half_rn(apply_act(__uint_as_float(v[j]) + b[j], ACT));
    }
}
template <int ACT>
__device__ __forceinline__ void store_row16(float *dst, const uint32_t (&v)[16], const float *b, int mc) {
    if (mc == 16 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            reinterpret_cast<float4 *>(dst)[j] = make_float4(apply_act(__uint_as_float(v[4 * j]) + b[4 * j], ACT),
                                                             apply_act(__uint_as_float(v[4 * j + 1]) + b[4 * j + 1], ACT),
                                                             apply_act(__uint_as_float(v[4 * j + 2]) + b[4 * j + 2], ACT),
                                                             apply_act(__uint_as_float(v[4 * j + 3]) + b[4 * j + 3], ACT));
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < mc) dst[j] = apply_act(__uint_as_float(v[j]) + b[j], ACT);
    }
}

// E: the element type, __half (fp16 MMAs) or float (3xTF32: a TF32 high part
// and its remainder for both operands, hi*hi + hi*lo + lo*hi per step).
template <int ACT, typename E>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    dense_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ PairTables T,
                      const E *__restrict__ bias, E *__restrict__ y) {
    using namespace sm100;
    constexpr bool kF32 = sizeof(E) == 4;
    constexpr int kParts = kF32 ? 2 : 1;
    constexpr int kCpb = kF32 ? 32 : 64;   // channels per 128-byte row
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
    const int SA = T.SA, SB = T.SB, KB = T.KB, Np = T.Np, M = T.M;
    const int n_units = T.n_units, a_stride = T.a_stride, a_bytes = T.a_bytes, b_slot = T.b_slot;
    const int BR = T.BR, BRs = T.BRs, HX = T.HX, ng = T.n_groups, PU = T.PU;
    const int chunk_rows = T.chunk_rows, n_chunks = T.n_chunks, n_slices = T.n_slices, slice_rows = T.slice_rows;
    const int nJz = T.nJ[0];
    const long long slice_pos = (long long)T.HY * HX;   // padded positions of one slice
    // shared-memory layout (identical in both CTAs of the pair)
    uint8_t *sA = smem;
    uint8_t *sB = sA + (size_t)SA * a_stride;
    float *bias_s = reinterpret_cast<float *>(sB + (size_t)SB * b_slot);
    uint64_t *bars = reinterpret_cast<uint64_t *>(bias_s + T.BL);   // BL is a multiple of 32: aligned
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
        prefetch_tmap(&tmBs);
    }
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
        // the padded copy is the previous grid's output: wait for it here
        // only, after the set-up and while the weight loads go out
        griddep_wait();
        int ia = 0;
        bool ok = true;
        for (int u = cid; u < n_units && ok; u += ncl) {
            int t = u / ng / T.n_mt;   // the channel tile does not change the input
            const int pu = t % PU;
            t /= PU;
            const int jz = t % nJz, n = t / nJz;
            const long long row0 = ((long long)n * T.HZ + jz) * slice_pos + pu * 256 + 128 * (int)rank;
            for (int kb = 0; kb < KB; ++kb, ++ia) {
                const int s = ia % SA;
                if (ia >= SA && !mbar_wait(emptyA + 8 * s, ((ia / SA) - 1) & 1, err, 1)) {
                    ok = false;
                    break;
                }
                if (rank == 0) mbar_arrive_expect_tx(fullA + 8 * s, 2u * kParts * (uint32_t)a_bytes);
                const uint32_t dst = smem_u32(sA + (size_t)s * a_stride);
                for (int part = 0; part < kParts; ++part)
                    for (int dz = 0; dz < n_slices; ++dz)
                        for (int ch = 0; ch < n_chunks; ++ch)
                            tma_load_3d_pair(dst + (uint32_t)(part * a_bytes + (dz * slice_rows + ch * chunk_rows) * 128),
                                             &tmA, fullA0 + 8 * s, kb * kCpb,
                                             (int)(row0 + dz * slice_pos + ch * chunk_rows), part);
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
                const int rowbase = ((u / ng) % T.n_mt) * T.total_rows + T.g_brow[g] + kb * T.g_rows_kb[g];
                for (int c = c0; c < c1; ++c, ++ib) {
                    if ((ib & 1) != me) continue;
                    const int s = ib % SB;
                    if (ib >= SB && !mbar_wait(emptyB + 8 * s, ((ib / SB) - 1) & 1, err, 4)) {
                        ok = false;
                        break;
                    }
                    const int rows = kParts * T.c_half[c];   // this rank's rows of the chunk
                    if (rank == 0) mbar_arrive_expect_tx(fullB + 8 * s, 2u * (uint32_t)rows * 128);
                    const uint32_t dst = smem_u32(sB + (size_t)s * b_slot);
                    const int row = rowbase + T.c_row0[c] + (int)rank * rows;
                    int r = 0;
                    for (; r + BR <= rows; r += BR) tma_load_2d_pair(dst + (uint32_t)r * 128, &tmB, fullB0 + 8 * s, 0, row + r);
                    for (; r < rows; r += BRs) tma_load_2d_pair(dst + (uint32_t)r * 128, &tmBs, fullB0 + 8 * s, 0, row + r);
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
                    const uint64_t blo = (uint64_t)((uint32_t)T.c_half[c] * 128 >> 4);   // low parts after the high parts
                    const uint64_t alo = (uint64_t)((uint32_t)a_bytes >> 4);
                    for (int it = T.c_item0[c]; it < i1; ++it) {
                        const uint64_t bd = desc_kmajor_sw128(b_addr + (uint32_t)T.item[it].crow * 128);
                        const uint64_t ad = desc_kmajor_sw128(a_addr + (uint32_t)T.item[it].shift * 128);
                        const uint32_t d = dbase + (uint32_t)T.item[it].tcol;
                        const uint32_t acc0 = (kb == 0 && T.item[it].first) ? 0u : 1u;
                        if constexpr (kF32) {
                            const uint32_t idesc = idesc_tf32_f32(256, T.item[it].n);
                            if (issuer) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    mma_tf32_pair(d, ad + 2 * q, bd + 2 * q, idesc, q == 0 ? acc0 : 1u);
                                    mma_tf32_pair(d, ad + 2 * q, bd + blo + 2 * q, idesc, 1u);
                                    mma_tf32_pair(d, ad + alo + 2 * q, bd + 2 * q, idesc, 1u);
                                }
                            }
                        } else {
                            const uint32_t idesc = idesc_f16_f32(256, T.item[it].n);
                            if (issuer) {
                                mma_f16_pair(d, ad, bd, idesc, acc0);
                                mma_f16_pair(d, ad + 2, bd + 2, idesc, 1u);
                                mma_f16_pair(d, ad + 4, bd + 4, idesc, 1u);
                                mma_f16_pair(d, ad + 6, bd + 6, idesc, 1u);
                            }
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
        // the bias, staged by the epilogue warps themselves (its global reads
        // stay off the set-up's path to the first loads)
        for (int m = (int)threadIdx.x - 128; m < T.BL; m += kPThreads - 128)
            bias_s[m] = (T.has_bias && m < M) ? (float)bias[m] : 0.f;
        named_bar_sync(1, kPThreads - 128);
        const int lane_base = 32 * (warp & 3);   // the TMEM lane quarter this warp may read
        const int eh = (warp - 4) >> 2;           // which alternate chunks of channels
        const int p = lane_base + lane;
        const int outz = T.out[0], outy = T.out[1], outx = T.out[2];
        const int sz = T.s[0], sy = T.s[1], sx = T.s[2], nJy = T.nJ[1], nJx = T.nJ[2];
        const int pair_x = T.pair_x, nhwc = T.nhwc;
        const bool has_bias = T.has_bias;
        const bool bias_vec = has_bias && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
        const long long plane = (long long)outz * outy * outx;
        int local = 0;
        for (int u = cid; u < n_units; u += ncl, ++local) {
            const int g = u % ng;
            const int mt = (u / ng) % T.n_mt;
            const int t = u / ng / T.n_mt;
            const int pu = t % PU;
            const int jz = (t / PU) % nJz, n = (t / PU) / nJz;
            const int buf = local & 1, use = local >> 1;
            if (!mbar_wait(tfull + 8 * buf, use & 1, err, 11)) break;
            tc_fence_after();
            const uint32_t dbase = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)buf * 256;
            const int F = pu * 256 + 128 * (int)rank + p;
            const int Jy = F / HX;
            const int Jx = F - Jy * HX;
            const bool pos_ok = Jx < nJx && Jy < nJy;
            const int ph0 = T.g_phase0[g], ph1 = ph0 + T.g_nphase[g];
            E *yimg = y + (long long)n * M * plane;
            const int cb = mt * T.Mt;                 // first output channel of this tile
            const int Mrem = min(T.Mt, M - cb);       // its channels that exist
            int piece = 0;   // (phase, 32-channel chunk) pieces, dealt alternately to the two warps of a quarter
            for (int ph = ph0; ph < ph1;) {
                const int rz = T.phase_r[ph][0], ry = T.phase_r[ph][1], rx = T.phase_r[ph][2];
                const int oz = sz * jz + rz;
                const int oy = sy * Jy + ry;
                const int ox = sx * Jx + rx;
                const bool valid = pos_ok && oz < outz && oy < outy && ox < outx;
                const bool pair = pair_x && ph + 1 < ph1 && (rx & 1) == 0 && T.phase_r[ph + 1][0] == rz &&
                                  T.phase_r[ph + 1][1] == ry && T.phase_r[ph + 1][2] == rx + 1;
                const uint32_t col0 = dbase + (uint32_t)((ph - ph0) * Np);
                const long long opos = ((long long)oz * outy + oy) * outx + ox;
                E *base = yimg + opos;                  // channels-first: channel stride plane
                E *rowl = yimg + opos * M;              // channels-last: the position's channel row
                for (int m0 = 0; m0 < Np; m0 += 32, ++piece) {
                    if ((piece & 1) != eh) continue;
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
                    const int mc0 = min(16, Mrem - m0), mc1 = min(16, Mrem - m0 - 16);
                    E *dst = base + (long long)(cb + m0) * plane;
                    float bb[32];
                    if (bias_vec && m0 + 32 <= Mrem) {
                        ld_bias32(bias + cb + m0, bb);
                    } else if (!has_bias) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) bb[j] = 0.f;
                    } else {   // the last, partial chunk of channels, or an unaligned bias
#pragma unroll
                        for (int j = 0; j < 32; ++j) bb[j] = bias_s[cb + m0 + j];
                    }
                    if (nhwc) {
                        // channels-last: 16 channels of a position as 16-byte pieces;
                        // the second x phase is the next position
                        E *dr = rowl + cb + m0;
                        store_row16<ACT>(dr, v0, bb, mc0);
                        if (two) store_row16<ACT>(dr + 16, v1, bb + 16, mc1);
                        if (pair) {
                            store_row16<ACT>(dr + M, w0, bb, mc0);
                            if (two) store_row16<ACT>(dr + M + 16, w1, bb + 16, mc1);
                        }
                    } else if (pair) {
                        // both x phases of a channel are adjacent: one half2 per channel
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < mc0)
                                st_pair(dst + j * plane, act_f<ACT>(__uint_as_float(v0[j]) + bb[j]),
                                        act_f<ACT>(__uint_as_float(w0[j]) + bb[j]));
                        if (two) {
                            E *d1 = dst + 16 * plane;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (j < mc1)
                                    st_pair(d1 + j * plane, act_f<ACT>(__uint_as_float(v1[j]) + bb[16 + j]),
                                            act_f<ACT>(__uint_as_float(w1[j]) + bb[16 + j]));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j < mc0) st_one(dst + j * plane, act_f<ACT>(__uint_as_float(v0[j]) + bb[j]));
                        if (two) {
                            E *d1 = dst + 16 * plane;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (j < mc1) st_one(d1 + j * plane, act_f<ACT>(__uint_as_float(v1[j]) + bb[16 + j]));
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
    return 1024 + (size_t)T.SA * T.a_stride + (size_t)T.SB * T.b_slot + (size_t)T.BL * 4 +
           (size_t)(2 * T.SA + 2 * T.SB + 5) * 8 + 16;
}

// ---------------------------------------------------------------------------
// host planning

int round_up(int v, int m) { return (v + m - 1) / m * m; }

bool build_pair_tables(const Plan &p, PairTables &T) {
    if ((p.dtype != CT_F16 && p.dtype != CT_F32) || p.G != 1 || !p.tabled) return false;
    // rows of the channels-last copy must be 16-byte multiples for TMA: a
    // channels-last X must already have them; the channels-first re-layout
    // pads with zeros
    const int row_elems = p.dtype == CT_F16 ? 8 : 4;
    if (p.C < 1 || (p.layout == CT_NHWC && p.C % row_elems != 0) || p.M < 1 || p.M > 16384 || p.N < 1 ||
        p.N > 65535)
        return false;
    for (int a = 0; a < 3; ++a)
        if (p.in[a] < 1 || p.in[a] > (1 << 24) || p.out[a] > (1 << 24)) return false;
    if (p.in[0] * p.in[1] * p.in[2] >= (1LL << 31)) return false;
    T.N = (int32_t)p.N;
    T.C = (int32_t)p.C;
    T.M = (int32_t)p.M;
    // output channels in tiles of at most 256 (one MMA's N), as even as 16 allows
    T.n_mt = (int32_t)ceil_div(p.M, 256);
    T.Mt = (int32_t)((ceil_div(p.M, T.n_mt) + 15) / 16 * 16);
    T.Np = T.Mt;
    T.BL = (T.n_mt * T.Mt + 31) / 32 * 32;
    T.f32 = p.dtype == CT_F32;
    T.nhwc = p.layout == CT_NHWC;
    T.Cd = (int32_t)ceil_div(p.C, row_elems) * row_elems;
    T.parts = T.f32 ? 2 : 1;
    T.cpb = T.f32 ? 32 : 64;
    T.KB = (int32_t)ceil_div(p.C, T.cpb);
    for (int a = 0; a < 3; ++a) {
        T.in[a] = (int32_t)p.in[a];
        T.out[a] = (int32_t)p.out[a];
        T.s[a] = (int32_t)p.s[a];
        T.pb[a] = (int32_t)p.pb[a];
        T.d[a] = (int32_t)p.d[a];
        T.k[a] = (int32_t)p.k[a];
        T.nJ[a] = (int32_t)ceil_div(p.out[a], p.s[a]);
    }
    T.has_bias = p.has_bias;
    T.act = p.act;
    T.pair_x = (p.s[2] % 2 == 0) && (p.out[2] % 2 == 0);
    T.dead = has_dead_phases(p);
    // live phases, z-major then y
    int np = 0;
    for (int rz = 0; rz < p.s[0]; ++rz)
        for (int ry = 0; ry < p.s[1]; ++ry)
            for (int rx = 0; rx < p.s[2]; ++rx) {
                if (p.taps[0][rz].empty() || p.taps[1][ry].empty() || p.taps[2][rx].empty()) continue;
                if (np >= kPMaxPhases) return false;
                T.phase_r[np][0] = (int16_t)rz;
                T.phase_r[np][1] = (int16_t)ry;
                T.phase_r[np][2] = (int16_t)rx;
                ++np;
            }
    if (np == 0) return false;
    T.n_phases = np;
    // groups: whole rows of phases (same rz, ry) merged while within 256 accumulator columns
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
            if (row_end - ph <= per)
                end = row_end;
            else
                break;
        }
        if (end == ph) {
            end = ph + 1;
            while (end < np && end - ph < per && same_row(end, ph)) ++end;
        }
        if (ng >= kPMaxGroups) return false;
        T.g_phase0[ng] = (int16_t)ph;
        T.g_nphase[ng] = (int16_t)(end - ph);
        ++ng;
        ph = end;
    }
    T.n_groups = ng;
    // padded origin and extents from the offsets of every live tap
    int lo[3], hi[3];
    for (int a = 0; a < 3; ++a) {
        lo[a] = 1 << 20;
        hi[a] = -(1 << 20);
    }
    for (int ph = 0; ph < np; ++ph)
        for (int a = 0; a < 3; ++a)
            for (const Tap &t : p.taps[a][T.phase_r[ph][a]]) {
                lo[a] = std::min(lo[a], (int)t.e);
                hi[a] = std::max(hi[a], (int)t.e);
            }
    for (int a = 0; a < 3; ++a) T.emin[a] = lo[a];
    const int span_z = hi[0] - lo[0], span_y = hi[1] - lo[1], span_x = hi[2] - lo[2];
    const long long HX = (long long)T.nJ[2] + span_x, HY = (long long)T.nJ[1] + span_y;
    const long long HZ = (long long)T.nJ[0] + span_z;
    // per slice: one run of 128 positions plus the y/x reach of the taps
    const long long run = span_y * HX + span_x + 128;
    if (run * (span_z + 1) > kPMaxTileRows) return false;
    T.HX = (int32_t)HX;
    T.HY = (int32_t)HY;
    T.HZ = (int32_t)HZ;
    T.n_slices = span_z + 1;
    const int slice = round_up((int)run, 8);
    T.n_chunks = (slice + 255) / 256;
    T.chunk_rows = round_up((slice + T.n_chunks - 1) / T.n_chunks, 8);
    T.slice_rows = T.chunk_rows * T.n_chunks;
    T.a_bytes = T.n_slices * T.slice_rows * 128;
    T.a_stride = round_up(T.parts * T.a_bytes, 1024);   // all parts of one stage
    const long long plane_pos = (long long)T.nJ[1] * HX;
    T.PU = (int32_t)ceil_div(plane_pos, 256);
    if ((long long)T.N * HZ * HY * HX + T.slice_rows + 256 >= (1LL << 31)) return false;
    if ((long long)T.N * HZ * HY * HX * T.Cd >= (1LL << 40)) return false;
    const long long units = (long long)T.N * T.nJ[0] * T.PU * ng * T.n_mt;
    if (units > (1LL << 30)) return false;
    T.n_units = (int32_t)units;
    // shared memory: three input stages (two when they do not fit) and at
    // least two weight chunks of at most 256 rows per rank.  Measured on the
    // 2-D decoder workload, three 34 KB input stages with three 32 KB chunk
    // slots beat two input stages with 64 KB chunks: the loads, not the
    // MMAs, set the pace there.
    const int fixed = 1024 + T.BL * 4 + (2 * 4 + 2 * 12 + 5) * 8 + 16;
    T.SA = (kPSmemBudget - fixed - 3LL * T.a_stride) / 2 >= 128 * 128 ? 3 : 2;
    const long long b_room = (kPSmemBudget - fixed - (long long)T.SA * T.a_stride) / 2;   // bytes of one chunk
    const int ch_max = (int)std::min<long long>(256 / T.parts, b_room / 128 / T.parts / 8 * 8);   // rows per rank and part
    if (ch_max < 128 / T.parts) return false;
    // items per group: (phase, tap) pairs grouped by input offset, offsets
    // shared by more phases first, adjacent phases merged into one wide MMA;
    // then consecutive items gathered into chunks of at most ch_max rows per rank
    int ni = 0, nc = 0, rows_total = 0;
    for (int g = 0; g < ng; ++g) {
        struct PairRec { int ph, ez, ey, ex; };
        std::vector<PairRec> pairs;
        for (int ph = T.g_phase0[g]; ph < T.g_phase0[g] + T.g_nphase[g]; ++ph)
            for (const Tap &a : p.taps[0][T.phase_r[ph][0]])
                for (const Tap &b : p.taps[1][T.phase_r[ph][1]])
                    for (const Tap &c : p.taps[2][T.phase_r[ph][2]]) pairs.push_back({ph, a.e, b.e, c.e});
        std::vector<std::array<int, 3>> offs;
        for (auto &q : pairs) offs.push_back({q.ez, q.ey, q.ex});
        std::sort(offs.begin(), offs.end());
        offs.erase(std::unique(offs.begin(), offs.end()), offs.end());
        auto nph = [&](const std::array<int, 3> &e) {
            int c = 0;
            for (auto &q : pairs) c += (q.ez == e[0] && q.ey == e[1] && q.ex == e[2]);
            return c;
        };
        std::stable_sort(offs.begin(), offs.end(),
                         [&](const std::array<int, 3> &a, const std::array<int, 3> &b) { return nph(a) > nph(b); });
        std::vector<char> touched(np, 0);
        T.g_item0[g] = (int16_t)ni;
        int brow = 0;   // weight rows of the group per channel block
        for (auto &e : offs) {
            std::vector<int> phs;
            for (auto &q : pairs)
                if (q.ez == e[0] && q.ey == e[1] && q.ex == e[2]) phs.push_back(q.ph);
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
                I.e[2] = (int16_t)e[2];
                I.n = (int16_t)((j - i) * T.Np);
                I.shift = (int32_t)((e[0] - lo[0]) * T.slice_rows + (e[1] - lo[1]) * HX + (e[2] - lo[2]));
                I.tcol = (int16_t)((phs[i] - T.g_phase0[g]) * T.Np);
                I.phase0 = (int16_t)phs[i];
                I.first = touched[phs[i]] ? 0 : 1;
                I.crow = 0;
                brow += I.n;
                for (size_t q = i; q < j; ++q) touched[phs[q]] = 1;
                ++ni;
                i = j;
            }
        }
        T.g_nitem[g] = (int16_t)(ni - T.g_item0[g]);
        T.g_brow[g] = rows_total;
        T.g_rows_kb[g] = brow * T.parts;
        rows_total += brow * T.parts * T.KB;
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
            row0 += 2 * T.parts * half;
            ++nc;
            it = jt;
        }
        T.g_nchunk[g] = (int16_t)(nc - T.g_chunk0[g]);
    }
    T.n_items = ni;
    T.total_rows = rows_total;
    if ((long long)T.n_mt * rows_total >= (1LL << 30)) return false;
    // weight loads: a CTA's half of a chunk is contiguous, loaded in boxes of
    // BR rows and the remainder in boxes of BRs rows
    int hmax = 0;   // rows per rank of the largest chunk (all parts)
    for (int c = 0; c < nc; ++c) hmax = std::max(hmax, T.parts * (int)T.c_half[c]);
    int br = 256;
    while (br > hmax) br /= 2;
    int brs = br;
    for (int c = 0; c < nc; ++c)
        while (((T.parts * T.c_half[c]) % br) % brs) brs /= 2;
    if (br < 8 || brs < 8) return false;
    T.BR = br;
    T.BRs = brs;
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

template <int ACT, typename E>
ct_status launch_pair(const PairTables &T, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmBs,
                      const void *bias, void *y, bool pdl, cudaStream_t st) {
    static std::atomic<int> attr_set[64];
    if (!allow_smem(dense_pair_kernel<ACT, E>, attr_set, kPSmemBudget)) return CT_ERR_DEVICE;
    const size_t smem = pair_launch_smem(T);
    int pairs = resident_pairs(dense_pair_kernel<ACT, E>, (int)smem);
    if (pairs > T.n_units) pairs = T.n_units;
    // programmatic dependent launch: the kernel's set-up overlaps the tail of
    // the re-layout (or the bias fill) before it; the input producer waits
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // programmatic launch only right after this call's own re-layout: the
    // weight loads start before the wait for that grid (it does not write
    // them; the grids before it completed, as it was launched normally)
    cfg.numAttrs = pdl ? 1 : 0;
    const E *b = (const E *)bias;
    E *yy = (E *)y;
    if (cudaLaunchKernelEx(&cfg, dense_pair_kernel<ACT, E>, tmA, tmB, tmBs, T, b, yy) != cudaSuccess) {
        cudaGetLastError();
        return CT_ERR_DEVICE;
    }
    return launch_status();
}

}  // namespace

// Automatic selection: for fp32 always (3xTF32 on the tensor cores measured
// 5x (channels-first) and 8x (channels-last) faster than the FFMA kernel on
// the 1-D fp32 vocoder workload); for fp16 channels-first with one or two
// spatial axes.  On the 3-D fp16 upsample workload (32 output channels) the
// halo kernel was measured faster: there the epilogue's stores, not the
// MMAs, set the pace, and the padded copy of a volume costs more than the
// plain re-layout.  For fp16 channels-last the two measured the same on the
// 2-D decoder workload, and the halo kernel needs no workspace.
// 1x1 stride-1 fp16 shapes (a plain GEMM per image, no halo) go to the halo
// kernel when its row mode applies (out_x a multiple of 8): its units are
// whole rows and its output tiles leave by TMA tensor stores, measured
// 30.9 against 33.1 us per call on X[8,512,64,64] x W[512,256,1,1].
bool dense_pair_preferred(const Plan &p) {
    if (p.dtype == CT_F32) return true;
    bool one_by_one = true;
    for (int a = 0; a < 3; ++a) one_by_one = one_by_one && p.k[a] == 1 && p.s[a] == 1;
    if (one_by_one && p.layout == CT_NCHW && p.out[2] % 8 == 0) return false;
    return p.layout == CT_NCHW && p.in[0] == 1 && p.out[0] == 1 && p.k[0] == 1 && p.s[0] == 1;
}

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

size_t dense_pair_packed_bytes(const Plan &p) { return (size_t)ptables(p).n_mt * ptables(p).total_rows * 128; }

size_t dense_pair_ws_bytes(const Plan &p) {
    const PairTables &T = ptables(p);
    return (size_t)T.parts * T.N * T.HZ * T.HY * T.HX * T.Cd * (T.f32 ? 4 : 2);
}

ct_status dense_pair_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const PairTables &T = ptables(p);
    const long long total = (long long)T.n_mt * T.total_rows * T.cpb;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (T.f32)
        pair_prepack_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(T, (const float *)w, (float *)wp);
    else
        pair_prepack_kernel<__half><<<(unsigned)blocks, 256, 0, st>>>(T, (const __half *)w, (__half *)wp);
    return launch_status();
}

ct_status dense_pair_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y, void *ws,
                         cudaStream_t st, int parts) {
    const PairTables &T = ptables(p);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CT_ERR_DEVICE;
    if (parts & CT_PART_PREPARE) {
        const long long S = (long long)T.in[0] * T.in[1] * T.in[2];
        const long long tiles = ceil_div(S, kPadS);
        PadGeo g;
        g.C = T.C;
        g.Cd = T.Cd;
        g.D = T.in[0];
        g.H = T.in[1];
        g.W = T.in[2];
        g.HZ = T.HZ;
        g.HY = T.HY;
        g.HX = T.HX;
        g.oz = -T.emin[0];
        g.oy = -T.emin[1];
        g.ox = -T.emin[2];
        g.halo_blocks = halo_blocks_for(g);
        if (tiles + g.halo_blocks > 0x7fffffffLL || ceil_div(T.Cd, T.cpb) > 65535 || S >= (1LL << 31))
            return CT_ERR_UNSUPPORTED;
        dim3 grid((unsigned)(tiles + g.halo_blocks), (unsigned)ceil_div(T.Cd, T.cpb), (unsigned)T.N);
        const size_t plane_elems = (size_t)T.N * T.HZ * T.HY * T.HX * T.Cd;
        if (T.nhwc) {
            // channels-last X: a padding copy of 16-byte pieces, about 8 per thread
            const long long pieces = (long long)T.C / (T.f32 ? 4 : 8);
            g.halo_blocks = halo_blocks_for(g);
            const long long copy_blocks = std::max<long long>(1, std::min<long long>(8192, ceil_div(S * pieces, 2048)));
            dim3 gridc((unsigned)(g.halo_blocks + copy_blocks), 1, (unsigned)T.N);
            if (T.f32)
                nhwc_to_padded_kernel<float><<<gridc, 256, 0, st>>>((const float *)x, (float *)ws,
                                                                    (float *)ws + plane_elems, g);
            else
                nhwc_to_padded_kernel<__half><<<gridc, 256, 0, st>>>((const __half *)x, (__half *)ws, nullptr, g);
        } else if (T.f32) {
            float *xh = (float *)ws;
            float *xl = xh + plane_elems;
            nchw_to_padded_f32_kernel<<<grid, 256, 0, st>>>((const float *)x, xh, xl, g);
        } else {
            nchw_to_padded_kernel<<<grid, 256, 0, st>>>((const __half *)x, (__half *)ws, g);
        }
        ct_status s1 = launch_status();
        if (s1 != CT_OK) return s1;
    }
    CUtensorMap tmA, tmB, tmBs;
    {
        // (channel, padded position, part): fp32 keeps the high parts and the
        // remainders as two planes of the workspace
        const size_t eb = T.f32 ? 4 : 2;
        const cuuint64_t rows = (cuuint64_t)T.N * T.HZ * T.HY * T.HX;
        const cuuint64_t dims[3] = {(cuuint64_t)T.Cd, rows, (cuuint64_t)T.parts};
        const cuuint64_t strides[2] = {(cuuint64_t)T.Cd * eb, (cuuint64_t)(rows * T.Cd * eb)};
        const cuuint32_t box[3] = {(cuuint32_t)T.cpb, (cuuint32_t)T.chunk_rows, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmA, T.f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, ws, dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    {
        const CUtensorMapDataType dt = T.f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        const cuuint64_t dims[2] = {(cuuint64_t)T.cpb, (cuuint64_t)T.n_mt * T.total_rows};
        const cuuint64_t strides[1] = {128};
        const cuuint32_t es[2] = {1, 1};
        const cuuint32_t box[2] = {(cuuint32_t)T.cpb, (cuuint32_t)T.BR};
        const cuuint32_t box_s[2] = {(cuuint32_t)T.cpb, (cuuint32_t)T.BRs};
        if (enc(&tmB, dt, 2, const_cast<void *>(wp), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            enc(&tmBs, dt, 2, const_cast<void *>(wp), dims, strides, box_s, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    if (T.dead && (parts & CT_PART_PREPARE)) {
        ct_status s2 = launch_dead_fill(p, bias, y, st);
        if (s2 != CT_OK) return s2;
    }
    if (!(parts & CT_PART_MAIN)) return CT_OK;
    const bool pdl = (parts & CT_PART_PREPARE) != 0;   // the re-layout runs just before
    if (T.f32) {
        if (T.act == CT_ACT_RELU) return launch_pair<CT_ACT_RELU, float>(T, tmA, tmB, tmBs, bias, y, pdl, st);
        return launch_pair<CT_ACT_IDENTITY, float>(T, tmA, tmB, tmBs, bias, y, pdl, st);
    }
    if (T.act == CT_ACT_RELU) return launch_pair<CT_ACT_RELU, __half>(T, tmA, tmB, tmBs, bias, y, pdl, st);
    return launch_pair<CT_ACT_IDENTITY, __half>(T, tmA, tmB, tmBs, bias, y, pdl, st);
}

int dense_pair_take_error(cudaStream_t st) { return take_error_word(g_dense_pair_err, st); }

}  // namespace ct
