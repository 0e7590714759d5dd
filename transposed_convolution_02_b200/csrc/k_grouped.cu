// Grouped fp16 ConvTranspose (small per-group channel counts), rank 1-2,
// channels-first: the grouped stride-phase kernel.
//
// ai.onnx.ConvTranspose README, implementation notes: the grouped
// stride-phase variant has one invocation own output pixels and a block of
// the group's output channels, every gathered input sample feeding the whole
// block, and the group's weight slab staged once per workgroup.  Here a CTA
// owns (image n, group g, a block of JB phase rows J_y, all columns, all
// M/group output channels):
//   1. the group's input rows (plus the halo the taps need) arrive in shared
//      memory channel-major by one TMA tile load (or by plain loads when the
//      rows are not 16-byte aligned) and are re-laid channel-contiguous:
//      pixel p holds its Cg channels in 2*Cg bytes followed by 16 bytes of
//      padding, an odd number of 16-byte units, so any 8 consecutive pixels
//      fall in distinct bank groups and a tap's ldmatrix rows are a plain
//      byte offset from the segment's;
//   2. output rows whose vertical stride phase receives no tap are pure bias
//      and are written straight from registers with 16-byte stores while the
//      input tile is in flight;
//   3. every other output row is cut into segments of 16 phase columns J_x
//      (16*s_x outputs).  A warp computes one segment: for each horizontal
//      phase with taps, a GEMM (group output channels) x (16 pixels) with the
//      reduction over (tap, input channel) on mma.sync m16n8k16 -- the packed
//      weights are the A operand, the re-laid input the B operand, so each
//      thread's accumulator holds two consecutive pixels of one channel.  The
//      results (plus bias) land in a per-warp staging tile whose columns of
//      tap-less phases hold the bias from the start; the finished tile goes
//      out as contiguous 16-byte row pieces.
// Output o = s*J + r (r the phase) receives the taps k with
// (r + pad_begin - k*d) divisible by s, reading input J + (r + pad_begin - k*d)/s,
// so the zero-inserted input never exists.
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "ct_cuda_util.h"
#include "ct_divmagic.h"
#include "ct_internal.h"
#include "sm100.cuh"

namespace ct {

__device__ int g_grouped_err;

namespace {

using namespace sm100;

constexpr int kGThreads = 256;
constexpr int kGWarps = kGThreads / 32;
constexpr int kGMaxS = 8;
constexpr int kGMaxPairs = 64;
constexpr int kGMaxSteps = 320;   // (tap pair, k-step) entries, each phase padded to a multiple of 4
constexpr int kGSmem = 200 * 1024;

struct GroupedArgs {
    int32_t N, C, M, G, Cg, Mg, KS, MT;     // KS = Cg/16 k-steps, MT = ceil(Mg/16) m-tiles
    int32_t in_y, in_x, out_y, out_x, s_y, s_x, k_y, k_x;
    int32_t nJy, nJx, JB, SR, SW, npix, emin_y, emin_x;
    int32_t n_rb, n_seg, n_pairs, has_bias, vec8, act;
    int32_t n_live_ry, n_dead_ry, n_live_rx;
    int32_t pst;                              // bytes per re-laid pixel (2*Cg + 16)
    int32_t segp;                             // staging row pitch (halves)
    int32_t one_phase;                        // steps of the one-phase path, 0 when it does not apply
    int32_t use_tma, x0, dx, BW;              // input tile: columns x0 + [0, BW); slab column c is tile column c + dx
    // shared-memory layout (byte offsets): input tile / staging union at 0, slab,
    // A fragments, step offsets, bias, barrier
    int32_t off_slab, off_w, off_steps, off_bias, off_bar, smem_total, raw_bytes, stage_bytes;
    // streaming form of the one-phase path (grouped_stream_kernel): persistent
    // CTAs, the input tile SRt x BW (channel stride an odd number of 16-byte
    // units), bias tiles for the tap-less rows at off_btile (two of
    // btile_bytes), the group's bias at off_sb (two of 64 halves)
    int32_t stream, SRt, grid, off_btile, btile_bytes, off_sb, off_wst, n_seg32;
    DivMagic d_qn, d_hn, d_seg32;
    DivMagic d_npix, d_sw, d_seg, d_lry, d_drow, d_segw, d_rb, d_g, d_cols, d_cprs, d_cprc;
    int8_t live_ry[kGMaxS], dead_ry[kGMaxS], live_rx[kGMaxS];
    uint8_t ph_q0[kGMaxS][kGMaxS], ph_nq[kGMaxS][kGMaxS];   // tap pairs of phase (ry, rx)
    int16_t ph_sp[kGMaxS][kGMaxS];            // first step-table entry of phase (ry, rx)
    int32_t n_steps;                          // step-table entries
    int32_t steps[kGMaxSteps];                // slab byte offset of each (tap pair, k-step)
    int16_t q_ky[kGMaxPairs], q_kx[kGMaxPairs];
};

const GroupedArgs &gargs(const Plan &p) { return *reinterpret_cast<const GroupedArgs *>(p.aux.data()); }

__device__ __forceinline__ void sts_b16(uint32_t a, __half v) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(a), "h"(__half_as_ushort(v)) : "memory");
}
__device__ __forceinline__ void sts_v4(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t bias_word(__half b) {
    const __half2 b2 = __halves2half2(b, b);
    return *reinterpret_cast<const uint32_t *>(&b2);
}

// Segments of the one-phase path: outputs o = 2*J + rx of row oy, channel m,
// get bias (other column phase) and value in one 32-bit word per J, packed by
// one f32x2 -> f16x2 conversion.  The weight fragments (A operand) stay in
// registers for the whole CTA; B fragments are loaded two steps ahead of the
// MMAs that use them.  Each lane stores its two J of channels gid and gid + 8
// as two 8-byte pieces: the four lanes of a channel row write 32 contiguous
// bytes, a whole sector.
template <int NSTEP, int ACT>
__device__ __forceinline__ void one_phase_rows(const GroupedArgs &A, const uint4 *__restrict__ wp, uint32_t s_w,
                                               const __half *sb, uint32_t s_slab, __half *yg,
                                               long long plane, int g, int jy0, int jbv, int warp,
                                               int lane, int nwarps) {
    const int gid = lane >> 2, tig = lane & 3;
    uint4 af[NSTEP];
    uint32_t offs[NSTEP];
#pragma unroll
    for (int j = 0; j < NSTEP; ++j) {
        // the group's fragments: staged in shared memory (s_w), else from global
        af[j] = s_w ? lds_v4(s_w + 16 * (j * 32 + lane)) : __ldg(wp + ((size_t)g * NSTEP + j) * 32 + lane);
        offs[j] = (uint32_t)A.steps[j];
    }
    const int ry = A.live_ry[0], rx = A.live_rx[0];
    const __half b0h = sb[gid], b1h = sb[gid + 8];
    const float bf0 = __half2float(b0h), bf1 = __half2float(b1h);
    // the other column phase's outputs: activated bias (exact in fp16)
    const float bo0 = __half2float(__float2half_rn(apply_act(bf0, ACT)));
    const float bo1 = __half2float(__float2half_rn(apply_act(bf1, ACT)));
    // 8-byte pieces: channels gid and gid + 8, J = 2*tig + [0, 2)
    const bool ok0 = gid < A.Mg, ok1 = gid + 8 < A.Mg;
    __half *y0 = yg + (long long)gid * plane + 4 * tig;
    __half *y1 = y0 + 8 * plane;
    const int lpix = 8 * (lane >> 4) + (lane & 7);
    const uint32_t lrow = s_slab + 16 * ((lane >> 3) & 1);
    const int items = jbv * A.n_seg;
    for (int it = warp; it < items; it += nwarps) {
        const int jyl = divq(it, A.d_seg);
        const int jx0 = (it - jyl * A.n_seg) * 16;
        const int oy = A.s_y * (jy0 + jyl) + ry;
        if (oy >= A.out_y) continue;
        const uint32_t lb = lrow + (uint32_t)(jyl * A.SW + min(jx0 + lpix, A.nJx - 1)) * A.pst;
        float acc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            acc[nt][0] = acc[nt][1] = bf0;
            acc[nt][2] = acc[nt][3] = bf1;
        }
        uint32_t bq[3][4];
        auto load_b = [&](int j, uint32_t(&b)[4]) {
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                         : "r"(lb + offs[j]));
        };
        load_b(0, bq[0]);
        if (NSTEP > 1) load_b(1, bq[1]);
#pragma unroll
        for (int j = 0; j < NSTEP; ++j) {
            if (j + 2 < NSTEP) load_b(j + 2, bq[(j + 2) % 3]);
            const uint32_t(&b)[4] = bq[j % 3];
            asm volatile(
                "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[0][0]), "+f"(acc[0][1]), "+f"(acc[0][2]), "+f"(acc[0][3])
                : "r"(af[j].x), "r"(af[j].y), "r"(af[j].z), "r"(af[j].w), "r"(b[0]), "r"(b[1]));
            asm volatile(
                "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[1][0]), "+f"(acc[1][1]), "+f"(acc[1][2]), "+f"(acc[1][3])
                : "r"(af[j].x), "r"(af[j].y), "r"(af[j].z), "r"(af[j].w), "r"(b[2]), "r"(b[3]));
        }
        // words: channel gid at J = jx0 + 8*nt + 2*tig + {0,1} (acc[nt][0..1]),
        // channel gid + 8 (acc[nt][2..3]); (bias, value) order inside a word:
        // value high when rx == 1.  nJx is even (out_x % 4 == 0), so each J
        // pair lies inside the row or wholly past it.
        const long long rowoff = (long long)oy * A.out_x + 2 * jx0;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            if (jx0 + 8 * nt + 2 * tig >= A.nJx) continue;
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v = apply_act(acc[nt][i], ACT), o = i < 2 ? bo0 : bo1;
                const __half2 h2 = rx ? __floats2half2_rn(o, v) : __floats2half2_rn(v, o);
                w[i] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            if (ok0) *reinterpret_cast<uint2 *>(y0 + rowoff + 16 * nt) = make_uint2(w[0], w[1]);
            if (ok1) *reinterpret_cast<uint2 *>(y1 + rowoff + 16 * nt) = make_uint2(w[2], w[3]);
        }
    }
}

// one_phase_rows for the persistent kernel: items of 32 J (four n-tiles of
// 8) whose MMAs share each step's weight fragment, read from shared memory
// (s_w) once per step, so the per-item work (position decode, accumulator
// set-up, loop) is spread over twice the outputs and the four accumulator
// chains hide each other's MMA latency.  B fragments are loaded one step
// ahead.  Stores as one_phase_rows does.
template <int NSTEP, int ACT>
__device__ __forceinline__ void one_phase_rows32(const GroupedArgs &A, uint32_t s_w, const __half *sb,
                                                 uint32_t s_slab, __half *yg, long long plane, int jy0, int jbv,
                                                 int warp, int lane, int nwarps) {
    const int gid = lane >> 2, tig = lane & 3;
    const int ry = A.live_ry[0], rx = A.live_rx[0];
    const float bf0 = __half2float(sb[gid]), bf1 = __half2float(sb[gid + 8]);
    // the other column phase's outputs: activated bias (exact in fp16)
    const float bo0 = __half2float(__float2half_rn(apply_act(bf0, ACT)));
    const float bo1 = __half2float(__float2half_rn(apply_act(bf1, ACT)));
    const bool ok0 = gid < A.Mg, ok1 = gid + 8 < A.Mg;
    __half *y0 = yg + (long long)gid * plane + 4 * tig;
    __half *y1 = y0 + 8 * plane;
    const int lpix = 8 * (lane >> 4) + (lane & 7);
    const uint32_t lrow = s_slab + 16 * ((lane >> 3) & 1);
    const uint32_t aw = s_w + 16 * lane;   // this lane's A fragment of step j at aw + 512 * j
    const int items = jbv * A.n_seg32;
    for (int it = warp; it < items; it += nwarps) {
        const int jyl = divq(it, A.d_seg32);
        const int jx0 = (it - jyl * A.n_seg32) * 32;
        const int oy = A.s_y * (jy0 + jyl) + ry;
        if (oy >= A.out_y) continue;
        const uint32_t rowb = lrow + (uint32_t)(jyl * A.SW) * A.pst;
        const uint32_t lb0 = rowb + (uint32_t)min(jx0 + lpix, A.nJx - 1) * A.pst;
        const uint32_t lb1 = rowb + (uint32_t)min(jx0 + 16 + lpix, A.nJx - 1) * A.pst;
        float acc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            acc[nt][0] = acc[nt][1] = bf0;
            acc[nt][2] = acc[nt][3] = bf1;
        }
        uint32_t bq[2][8];
        auto load_b = [&](int j, uint32_t(&b)[8]) {
            const uint32_t o = (uint32_t)A.steps[j];
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                         : "r"(lb0 + o));
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7])
                         : "r"(lb1 + o));
        };
        load_b(0, bq[0]);
#pragma unroll
        for (int j = 0; j < NSTEP; ++j) {
            if (j + 1 < NSTEP) load_b(j + 1, bq[(j + 1) & 1]);
            const uint32_t(&b)[8] = bq[j & 1];
            const uint4 a = lds_v4(aw + 512 * j);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
                asm volatile(
                    "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                    "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                    : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
                    : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b[2 * nt]), "r"(b[2 * nt + 1]));
        }
        const long long rowoff = (long long)oy * A.out_x + 2 * jx0;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            if (jx0 + 8 * nt + 2 * tig >= A.nJx) continue;
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v = apply_act(acc[nt][i], ACT), o = i < 2 ? bo0 : bo1;
                const __half2 h2 = rx ? __floats2half2_rn(o, v) : __floats2half2_rn(v, o);
                w[i] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            if (ok0) *reinterpret_cast<uint2 *>(y0 + rowoff + 16 * nt) = make_uint2(w[0], w[1]);
            if (ok1) *reinterpret_cast<uint2 *>(y1 + rowoff + 16 * nt) = make_uint2(w[2], w[3]);
        }
    }
}

// Resident CTAs per SM the one-phase path is compiled for: the register cap
// its launch bounds give the compiler.
constexpr int kGOnePhaseMinBlocks = 3;

// NSTEP > 0: the one-phase path -- one output channel tile (MT == 1), a
// single stride phase with taps, s_x == 2, NSTEP (tap pair, k-step) steps
// whose weight fragments and slab offsets stay in registers, and outputs
// stored straight from the accumulators as (bias, value) pairs.
// ACT: the output activation (ct_activation), fixed at compile time.
template <int MT, int NSTEP, int ACT>
__global__ void __launch_bounds__(kGThreads, NSTEP > 0 ? kGOnePhaseMinBlocks : (MT <= 2 ? 4 : 2))
    grouped_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ GroupedArgs A,
                   const __half *__restrict__ x, const uint4 *__restrict__ wp,
                   const __half *__restrict__ bias, __half *__restrict__ y) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t s0 = smem_u32(sm);          // input tile, later the per-warp staging tiles
    const uint32_t s_slab = s0 + A.off_slab;   // re-laid input [npix][pst]
    const uint32_t s_w = s0 + A.off_w;         // A fragments [pair][ks][mt][lane][16 B]
    const uint32_t s_steps = s0 + A.off_steps; // slab byte offset of each (pair, k-step)
    __half *sb = reinterpret_cast<__half *>(sm + A.off_bias);   // bias of the group, 64 halves
    const uint32_t bar = s0 + A.off_bar;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bq = divq(blockIdx.x, A.d_rb);
    const int rb = blockIdx.x - bq * A.n_rb;
    const int n = divq(bq, A.d_g);
    const int g = bq - n * A.G;
    const int jy0 = rb * A.JB;
    const int jbv = min(A.JB, A.nJy - jy0);
    const long long plane = (long long)A.out_y * A.out_x;
    __half *yg = y + ((long long)n * A.M + (long long)g * A.Mg) * plane;

    // 1a. the input tile, first of all: rows jy0 + emin_y + [0, SR), columns
    //     x0 + [0, BW), the group's Cg channels; zero outside the input.  The
    //     other threads wait on the barrier only after a __syncthreads.
    if (tid == 0 && A.use_tma) {
        mbar_init(bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(bar, (uint32_t)A.raw_bytes);
        tma_load_3d(s0, &tmx, bar, A.x0, jy0 + A.emin_y, n * A.C + g * A.Cg);
    }
    if (tid < 64) sb[tid] = (A.has_bias && tid < A.Mg) ? bias[g * A.Mg + tid] : __float2half(0.f);
    // weights of the group (A-operand fragments) and the per-step tap offsets
    if (NSTEP == 0) {
        const int words = A.n_pairs * A.KS * MT * 32;
        const uint4 *src = wp + (size_t)g * words;
        for (int i = tid; i < words; i += kGThreads) sts_v4(s_w + 16 * i, __ldg(src + i));
        for (int i = tid; i < A.n_steps; i += kGThreads)
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(s_steps + 4 * i), "r"(A.steps[i]) : "memory");
    }

    // 2. rows of tap-less vertical phases: bias only, while the tile is in flight
    {
        const int cols = A.vec8 ? A.out_x >> 3 : A.out_x;  // pieces per channel row
        const int width = A.vec8 ? 8 : 1;                 // halves per piece
        const bool narrow = cols <= 32;
        const int lm = narrow ? divq(lane, A.d_cols) : 0;  // this lane's first channel and piece
        const int lc = narrow ? lane - lm * cols : lane;
        const int mstep = narrow ? divq(32, A.d_cols) : 1;
        const int rows = jbv * A.n_dead_ry;
        for (int r = warp; r < rows; r += kGWarps) {
            const int jyl = divq(r, A.d_drow);
            const int oy = A.s_y * (jy0 + jyl) + A.dead_ry[r - jyl * A.n_dead_ry];
            if (oy >= A.out_y) continue;
            __half *yr = yg + (long long)oy * A.out_x;
            if (lm >= mstep) continue;
            __half *p = yr + (long long)lm * plane;
            for (int m = lm; m < A.Mg; m += mstep, p += mstep * plane) {
                const __half b = __float2half_rn(apply_act(A.has_bias ? __half2float(__ldg(bias + g * A.Mg + m)) : 0.f, ACT));
                for (int c = lc; c < cols; c += 32) {
                    if (A.vec8) {
                        const uint32_t w = bias_word(b);
                        *reinterpret_cast<uint4 *>(p + c * width) = make_uint4(w, w, w, w);
                    } else {
                        p[c] = b;
                    }
                    if (narrow) break;
                }
            }
        }
    }

    // 1b. re-lay the input channel-contiguous: slab pixel (row, col) <- tile
    //     (row, col + dx); a task is one pixel and 8 channels
    __syncthreads();   // barrier initialised, bias and tables staged
    if (A.use_tma) {
        mbar_wait(bar, 0, &g_grouped_err, 1);
        const uint32_t cs = (uint32_t)A.SR * A.BW * 2;   // channel stride of the tile
        for (int pix = tid; pix < A.npix; pix += kGThreads) {
            const int r = divq(pix, A.d_sw);
            uint32_t src = s0 + (uint32_t)(r * A.BW + (pix - r * A.SW) + A.dx) * 2;
            const uint32_t dst = s_slab + (uint32_t)pix * A.pst;
            for (int hc = 0; hc < 2 * A.KS; hc += 2) {   // 2*KS is even
                uint32_t h[16];
#pragma unroll
                for (int i = 0; i < 16; ++i, src += cs) h[i] = lds_u16(src);
                sts_v4(dst + 16 * hc, make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                                 h[6] | (h[7] << 16)));
                sts_v4(dst + 16 * hc + 16, make_uint4(h[8] | (h[9] << 16), h[10] | (h[11] << 16),
                                                      h[12] | (h[13] << 16), h[14] | (h[15] << 16)));
            }
        }
    } else {
        // rows not 16-byte aligned: gather from global, 8 channel loads per task,
        // coalesced across the warp (consecutive pixels)
        const int tasks = A.KS * 2 * A.npix;
        const long long cstride = (long long)A.in_y * A.in_x;
        const unsigned short *xg = reinterpret_cast<const unsigned short *>(x) +
                                   ((long long)n * A.C + (long long)g * A.Cg) * cstride;
        for (int t = tid; t < tasks; t += kGThreads) {
            const int hc = divq(t, A.d_npix);
            const int pix = t - hc * A.npix;
            const int row = divq(pix, A.d_sw);
            const int iy = jy0 + A.emin_y + row, ix = A.emin_x + (pix - row * A.SW);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if ((unsigned)iy < (unsigned)A.in_y && (unsigned)ix < (unsigned)A.in_x) {
                const unsigned short *src = xg + (long long)(hc * 8) * cstride + (long long)iy * A.in_x + ix;
                uint32_t h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) h[i] = __ldg(src + (long long)i * cstride);
                v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
            }
            sts_v4(s_slab + (uint32_t)pix * A.pst + 16 * hc, v);
        }
    }
    __syncthreads();

    if constexpr (NSTEP > 0) {
        one_phase_rows<NSTEP, ACT>(A, wp, 0u, sb, s_slab, yg, plane, g, jy0, jbv, warp, lane, kGWarps);
        return;
    }
    // staging tile (over the consumed input tile): every column starts as the
    // bias of its channel (the final value of the tap-less horizontal phases;
    // the others are overwritten)
    const uint32_t stg_base = s0 + (uint32_t)(warp * (MT * 16) * A.segp) * 2;
    {
        const int cpr = A.segp >> 3;
        for (int e = lane; e < MT * 16 * cpr; e += 32) {
            const int m = divq(e, A.d_cprs);
            const uint32_t w = bias_word(__float2half_rn(apply_act(__half2float(sb[m]), ACT)));
            sts_v4(stg_base + (uint32_t)(m * A.segp + 8 * (e - m * cpr)) * 2, make_uint4(w, w, w, w));
        }
    }
    __syncwarp();

    // 3. segments of rows with taps
    const int gid = lane >> 2, tig = lane & 3;
    float bv[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) bv[mt][hh] = __half2float(sb[mt * 16 + gid + 8 * hh]);
    // this lane's ldmatrix row: pixel lpix of the segment, channels 8*((lane >> 3) & 1) + [0, 8)
    const int lpix = 8 * (lane >> 4) + (lane & 7);
    const uint32_t lrow = s_slab + 16 * ((lane >> 3) & 1);
    // this lane's staging element: channel gid, pixel 2*tig (bytes)
    const uint32_t stg_lane = stg_base + (uint32_t)(gid * A.segp + 2 * tig * A.s_x) * 2;
    const uint32_t row8 = 16 * A.segp;          // 8 staging rows, bytes
    const uint32_t colJ = 2 * A.s_x;            // one phase column J, bytes
    const int seg_out = 16 * A.s_x;             // outputs of a segment row
    const int cpr = 2 * A.s_x;                  // 16-byte pieces of a segment row
    const int rpp = divq(32, A.d_cprc);         // channel rows per pass of the warp
    const int my_m = divq(lane, A.d_cprc), my_c = lane - my_m * cpr;
    const uint32_t stg_copy = stg_base + (uint32_t)(my_m * A.segp + 8 * my_c) * 2;
    const uint32_t stg_copy_step = (uint32_t)(rpp * A.segp) * 2;
    __half *ylane = yg + (long long)my_m * plane + 8 * my_c;   // this lane's first row piece
    const long long ystep = (long long)rpp * plane;
    constexpr uint32_t ablk = MT * 512;         // A fragments of one (pair, k-step)
    const int KS = A.KS;
    const int items = jbv * A.n_live_ry * A.n_seg;
    for (int it = warp; it < items; it += kGWarps) {
        const int t1 = divq(it, A.d_seg);
        const int sg = it - t1 * A.n_seg;
        const int jyl = divq(t1, A.d_lry);
        const int ry = A.live_ry[t1 - jyl * A.n_live_ry];
        const int oy = A.s_y * (jy0 + jyl) + ry;
        if (oy >= A.out_y) continue;
        const int jx0 = sg * 16;
        const uint32_t lb = lrow + (uint32_t)(jyl * A.SW + min(jx0 + lpix, A.nJx - 1)) * A.pst;
        for (int lx = 0; lx < A.n_live_rx; ++lx) {
            const int rx = A.live_rx[lx];
            // accumulators start at the bias of their channel
            float acc[MT][2][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[mt][nt][j] = bv[mt][j >> 1];
            // the phase's (tap pair, k-step) steps: A fragments from entry
            // q0*KS on, slab offsets from its padded step-table entry on
            const int ns = A.ph_nq[ry][rx] * KS;
            uint32_t aa = s_w + (uint32_t)(A.ph_q0[ry][rx] * KS) * ablk + 16 * lane;
            uint32_t ta = s_steps + 4 * A.ph_sp[ry][rx];
            auto step = [&](uint32_t off, uint32_t a_addr) {
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(lb + off));
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint4 a = lds_v4(a_addr + 512 * mt);
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                        : "+f"(acc[mt][0][0]), "+f"(acc[mt][0][1]), "+f"(acc[mt][0][2]), "+f"(acc[mt][0][3])
                        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                        : "+f"(acc[mt][1][0]), "+f"(acc[mt][1][1]), "+f"(acc[mt][1][2]), "+f"(acc[mt][1][3])
                        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b2), "r"(b3));
                }
            };
            int i = 0;
            for (; i + 4 <= ns; i += 4, ta += 16, aa += 4 * ablk) {
                const uint4 o = lds_v4(ta);
                step(o.x, aa);
                step(o.y, aa + ablk);
                step(o.z, aa + 2 * ablk);
                step(o.w, aa + 3 * ablk);
            }
            if (i < ns) {   // 1-3 steps left; the table is padded to whole groups of 4
                const uint4 o = lds_v4(ta);
                step(o.x, aa);
                if (i + 1 < ns) step(o.y, aa + ablk);
                if (i + 2 < ns) step(o.z, aa + 2 * ablk);
            }
            // accumulator (channel gid / gid+8, pixels 2*tig, 2*tig+1) + bias -> staging
            const uint32_t sl = stg_lane + 2 * rx;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t o = sl + (2 * mt + hh) * row8 + 8 * nt * colJ;
                        sts_b16(o, __float2half_rn(apply_act(acc[mt][nt][2 * hh], ACT)));
                        sts_b16(o + colJ, __float2half_rn(apply_act(acc[mt][nt][2 * hh + 1], ACT)));
                    }
        }
        __syncwarp();
        // the segment rows of every channel: outputs s_x*jx0 + [0, 16 s_x), cut at out_x
        const int off = oy * A.out_x + A.s_x * jx0;
        const int lim = A.out_x - A.s_x * jx0;
        if (A.vec8) {
            if (my_m < rpp && 8 * my_c < lim) {
                __half *p = ylane + off;
                uint32_t sa = stg_copy;
                for (int m = my_m; m < A.Mg; m += rpp, p += ystep, sa += stg_copy_step)
                    *reinterpret_cast<uint4 *>(p) = lds_v4(sa);
            }
        } else {
            const __half *st = reinterpret_cast<const __half *>(sm + (stg_base - s0));
            __half *yr = yg + off;
            for (int e = lane; e < A.Mg * seg_out; e += 32) {
                const int m = divq(e, A.d_segw);
                const int c = e - m * seg_out;
                if (c < lim) yr[(long long)m * plane + c] = st[(size_t)m * A.segp + c];
            }
        }
        __syncwarp();
    }
}

// weight pre-pack into mma.sync A fragments (rows = output channels of the
// group, columns = 16 input channels of one k-step):
// [g][pair][ks][mt][lane][8 halves]; lane half e = 2*reg + b holds
//   row gid + 8*(reg & 1), column 2*tig + b + 8*(reg >> 1)
__global__ void __launch_bounds__(256) grouped_prepack_kernel(const __grid_constant__ GroupedArgs A,
                                                              const __half *__restrict__ w,
                                                              __half *__restrict__ wp) {
    const long long per_g = (long long)A.n_pairs * A.KS * A.MT * 256;   // halves
    const long long total = per_g * A.G;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        long long r = i;
        const int e = (int)(r & 7);
        r >>= 3;
        const int lane = (int)(r & 31);
        r >>= 5;
        const int mt = (int)(r % A.MT);
        r /= A.MT;
        const int ks = (int)(r % A.KS);
        r /= A.KS;
        const int q = (int)(r % A.n_pairs);
        const int g = (int)(r / A.n_pairs);
        const int reg = e >> 1, b = e & 1;
        const int m = mt * 16 + (lane >> 2) + 8 * (reg & 1);
        const int k = ks * 16 + 2 * (lane & 3) + b + 8 * (reg >> 1);
        __half v = __float2half(0.f);
        if (m < A.Mg) {
            const long long c = (long long)g * A.Cg + k;
            const long long kpos = (long long)A.q_ky[q] * A.k_x + A.q_kx[q];
            v = w[(c * A.Mg + m) * ((long long)A.k_y * A.k_x) + kpos];
        }
        wp[i] = v;
    }
}


// The one-phase path as a persistent kernel.  CTA c walks blocks c, c +
// gridDim.x, ... (neighbouring CTAs take neighbouring row blocks, so the
// halo rows they share are read from DRAM once).  Warp 7 is the producer:
//   * it loads each block's input tile and the group's weight fragments with
//     TMA while the previous block is computed (one barrier for both; the
//     fragments in two alternating buffers);
//   * it stages the block's bias and a [Mg][out_x] tile of its activated
//     value, and writes the block's tap-less output rows from that tile with
//     TMA tensor stores (two tiles and bias buffers alternate; a tile is
//     refilled only once the stores of two blocks back have read it).  It
//     issues no global stores of its own, so its proxy fence before the bulk
//     stores does not wait for the compute warps' outputs, and it prepares
//     the next block's rows while the compute warps work on this one.
// Per block, all warps re-lay the input tile channel-contiguous: each 8
// channels x 8 pixels piece is read transposed with ldmatrix.trans and
// written with stmatrix as 8 pixel rows of the slab (the tile's channel
// stride is an odd number of 16-byte units, so the 8 rows of a piece fall in
// distinct banks).  The tile is then free: the producer starts the next
// load, and warps 0-6 compute the rows with taps as one_phase_rows does.
template <int NSTEP, int ACT>
__global__ void __launch_bounds__(kGThreads, kGOnePhaseMinBlocks)
    grouped_stream_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmy,
                          const __grid_constant__ GroupedArgs A, const uint4 *__restrict__ wp,
                          const __half *__restrict__ bias, __half *__restrict__ y) {
    extern __shared__ __align__(1024) uint8_t sm[];
    constexpr int kProducer = kGWarps - 1;
    constexpr uint32_t kWBytes = NSTEP * 512;   // one group's A fragments
    const uint32_t s0 = smem_u32(sm);
    const uint32_t s_tile = s0;
    const uint32_t s_slab = s0 + A.off_slab;
    const uint32_t s_btile = s0 + A.off_btile;
    const uint32_t s_wst = s0 + A.off_wst;
    const uint32_t bar = s0 + A.off_bar;
    const uint32_t s_sink = bar + 16;   // 16 bytes that absorb the pixels outside the slab
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_blocks = A.N * A.G * A.n_rb;
    const long long plane = (long long)A.out_y * A.out_x;
    const uint32_t cs = (uint32_t)A.SRt * A.BW * 2;   // channel stride of the tile, bytes
    const int qn = A.BW >> 3, hn = A.Cg >> 3;
    const int pieces = A.SR * qn * hn;                 // 8 x 8 pieces of the slab's rows
    const bool loader = warp == kProducer && lane == 0;

    auto coords = [&](int b, int &n, int &g, int &jy0) {
        const int bq = divq(b, A.d_rb);
        n = divq(bq, A.d_g);
        g = bq - n * A.G;
        jy0 = (b - bq * A.n_rb) * A.JB;
    };
    // the tile and the fragments of block b (its k-th) on the barrier
    auto load_block = [&](int b, int k) {
        int n, g, jy0;
        coords(b, n, g, jy0);
        mbar_arrive_expect_tx(bar, (uint32_t)A.raw_bytes + kWBytes);
        tma_load_3d(s_tile, &tmx, bar, A.x0, jy0 + A.emin_y, n * A.C + g * A.Cg);
        bulk_load(s_wst + (uint32_t)(k & 1) * kWBytes, wp + (size_t)g * NSTEP * 32, kWBytes, bar);
    };
    if (loader) {
        mbar_init(bar, 1);
        fence_barrier_init();
        prefetch_tmap(&tmx);
        prefetch_tmap(&tmy);
        if ((int)blockIdx.x < n_blocks) load_block(blockIdx.x, 0);
    }
    __syncthreads();

    int k = 0;
    bool ok = true;
    for (int b = blockIdx.x; b < n_blocks; b += gridDim.x, ++k) {
        int n, g, jy0;
        coords(b, n, g, jy0);
        const int jbv = min(A.JB, A.nJy - jy0);
        __half *sb = reinterpret_cast<__half *>(sm + A.off_sb) + 64 * (k & 1);
        if (warp == kProducer) {
            sb[lane] = (A.has_bias && lane < A.Mg) ? bias[g * A.Mg + lane] : __float2half(0.f);
            sb[lane + 32] = (A.has_bias && lane + 32 < A.Mg) ? bias[g * A.Mg + lane + 32] : __float2half(0.f);
            if (A.n_dead_ry > 0) {
                const uint32_t bt = s_btile + (uint32_t)(k & 1) * A.btile_bytes;
                if (lane == 0) bulk_wait_group_read<1>();   // the stores of block k - 2 have read this tile
                __syncwarp();
                const int cpr = A.out_x >> 3;   // 16-byte pieces per channel row
                for (int e = lane; e < A.Mg * cpr; e += 32) {
                    const int m = divq(e, A.d_cols);
                    const uint32_t w = bias_word(__float2half_rn(apply_act(__half2float(sb[m]), ACT)));
                    sts_v4(bt + 16 * e, make_uint4(w, w, w, w));
                }
                fence_proxy_async();   // the tile, written here, before the bulk stores read it
                __syncwarp();
                if (lane == 0) {
                    for (int jyl = 0; jyl < jbv; ++jyl)
                        for (int d = 0; d < A.n_dead_ry; ++d) {
                            const int oy = A.s_y * (jy0 + jyl) + A.dead_ry[d];
                            if (oy < A.out_y) tma_store_3d(&tmy, bt, 0, oy, n * A.M + g * A.Mg);
                        }
                    bulk_commit_group();
                }
            }
        }
        // the block's input tile and fragments; every compute warp has finished the previous block
        ok = mbar_wait(bar, k & 1, &g_grouped_err, 2);
        if (!__syncthreads_and(ok)) break;
        {
            const int i = lane & 7, sub = lane >> 3;
            for (int o = 4 * warp; o < pieces; o += 4 * kGWarps) {
                const int pc = min(o + sub, pieces - 1);
                const int t = divq(pc, A.d_qn);   // piece = (r * hn + h) * qn + q
                const int q = pc - t * qn;
                const int r = divq(t, A.d_hn);
                const int h = t - r * hn;
                uint32_t v[4];
                ldmatrix_x4_trans(s_tile + (uint32_t)(8 * h + i) * cs + (uint32_t)(r * A.BW + 8 * q) * 2, v);
                const int c = 8 * q + i - A.dx;   // slab column of this lane's pixel row
                const uint32_t dst = (c >= 0 && c < A.SW) ? s_slab + (uint32_t)(r * A.SW + c) * A.pst + 16 * h : s_sink;
                stmatrix_x4(dst, v);
            }
        }
        __syncthreads();   // slab complete, tile consumed
        if (warp == kProducer) {
            if (lane == 0 && b + (int)gridDim.x < n_blocks) {
                fence_proxy_async();
                load_block(b + (int)gridDim.x, k + 1);
            }
        } else {
            __half *yg = y + ((long long)n * A.M + (long long)g * A.Mg) * plane;
            one_phase_rows32<NSTEP, ACT>(A, s_wst + (uint32_t)(k & 1) * kWBytes, sb, s_slab, yg, plane, jy0, jbv,
                                         warp, lane, kProducer);
        }
    }
    if (!ok && loader) mbar_wait(bar, k & 1, &g_grouped_err, 3);   // the load that timed out, drained
    if (loader) bulk_wait_group_all();
}
}  // namespace

bool grouped_setup(const Plan &p, GroupedArgs &A, int jb);

// Steps of the one-phase path (0: the generic path serves the plan).
int one_phase_steps(const GroupedArgs &A) {
    if (A.MT != 1 || A.n_live_ry != 1 || A.n_live_rx != 1 || A.s_x != 2 || A.out_x % 4 != 0) return 0;
    const int ns = A.n_pairs * A.KS;
    switch (ns) {
        case 1: case 2: case 3: case 4: case 6: case 8: case 9: case 12: return ns;
    }
    return 0;
}

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool grouped_supports(const Plan &p) {
    if (p.dtype != CT_F16 || p.layout != CT_NCHW || !p.tabled) return false;
    if (p.rank > 2 || p.G < 2) return false;
    if (p.Cg % 16 != 0 || p.Cg > 64 || p.Mg % 8 != 0 || p.Mg > 64) return false;
    if (p.N < 1 || p.in[1] < 1 || p.in[2] < 1) return false;
    if (p.s[1] > kGMaxS || p.s[2] > kGMaxS) return false;
    int np = 0, nq = 0;
    for (int ry = 0; ry < p.s[1]; ++ry)
        for (int rx = 0; rx < p.s[2]; ++rx) {
            const size_t t = p.taps[1][ry].size() * p.taps[2][rx].size();
            if (t) {
                ++np;
                nq += (int)t;
            }
        }
    if (np == 0 || nq > kGMaxPairs) return false;
    GroupedArgs *A = new GroupedArgs();
    const bool ok = grouped_setup(p, *A, 1) && A->smem_total <= kGSmem;
    delete A;
    return ok;
}

// Fill the arguments for J-row blocks of `jb` rows; false when an index
// would leave the ranges the kernel's 32-bit arithmetic covers.
bool grouped_setup(const Plan &p, GroupedArgs &A, int jb) {
    A = GroupedArgs();
    A.N = (int32_t)p.N;
    A.C = (int32_t)p.C;
    A.M = (int32_t)p.M;
    A.G = (int32_t)p.G;
    A.Cg = (int32_t)p.Cg;
    A.Mg = (int32_t)p.Mg;
    A.KS = A.Cg / 16;
    A.MT = (A.Mg + 15) / 16;
    A.in_y = (int32_t)p.in[1];
    A.in_x = (int32_t)p.in[2];
    A.out_y = (int32_t)p.out[1];
    A.out_x = (int32_t)p.out[2];
    A.s_y = (int32_t)p.s[1];
    A.s_x = (int32_t)p.s[2];
    A.k_y = (int32_t)p.k[1];
    A.k_x = (int32_t)p.k[2];
    A.has_bias = p.has_bias;
    A.act = p.act;
    if ((long long)A.out_y * A.out_x >= (1LL << 30) || (long long)A.in_y * A.in_x >= (1LL << 30)) return false;
    int nq = 0;
    int emin_y = 1 << 20, emax_y = -(1 << 20), emin_x = 1 << 20, emax_x = -(1 << 20);
    for (int ry = 0; ry < A.s_y; ++ry) {
        if (p.taps[1][ry].empty())
            A.dead_ry[A.n_dead_ry++] = (int8_t)ry;
        else
            A.live_ry[A.n_live_ry++] = (int8_t)ry;
    }
    for (int rx = 0; rx < A.s_x; ++rx)
        if (!p.taps[2][rx].empty()) A.live_rx[A.n_live_rx++] = (int8_t)rx;
    for (int ry = 0; ry < A.s_y; ++ry)
        for (int rx = 0; rx < A.s_x; ++rx) {
            if (p.taps[1][ry].empty() || p.taps[2][rx].empty()) continue;
            A.ph_q0[ry][rx] = (uint8_t)nq;
            for (const Tap &ty : p.taps[1][ry])
                for (const Tap &tx : p.taps[2][rx]) {
                    if (nq >= kGMaxPairs) return false;
                    A.q_ky[nq] = (int16_t)ty.k;
                    A.q_kx[nq] = (int16_t)tx.k;
                    emin_y = std::min(emin_y, (int)ty.e);
                    emax_y = std::max(emax_y, (int)ty.e);
                    emin_x = std::min(emin_x, (int)tx.e);
                    emax_x = std::max(emax_x, (int)tx.e);
                    ++nq;
                }
            A.ph_nq[ry][rx] = (uint8_t)(nq - A.ph_q0[ry][rx]);
        }
    if (nq == 0 || A.n_live_ry == 0 || A.n_live_rx == 0) return false;
    A.n_pairs = nq;
    A.emin_y = emin_y;
    A.emin_x = emin_x;
    A.nJy = (int32_t)ceil_div(p.out[1], p.s[1]);
    A.nJx = (int32_t)ceil_div(p.out[2], p.s[2]);
    A.SW = A.nJx + (emax_x - emin_x);
    A.JB = std::max(1, std::min(jb, A.nJy));
    A.SR = A.JB + (emax_y - emin_y);
    A.npix = A.SR * A.SW;
    A.pst = 2 * A.Cg + 16;
    // step table: per phase, the slab byte offset of each (tap pair, k-step)
    // in the order the pairs were listed, padded to a multiple of 4 entries
    {
        int t = 0;
        for (int ry = 0; ry < A.s_y; ++ry)
            for (int rx = 0; rx < A.s_x; ++rx) {
                if (p.taps[1][ry].empty() || p.taps[2][rx].empty()) continue;
                A.ph_sp[ry][rx] = (int16_t)t;
                for (const Tap &ty : p.taps[1][ry])
                    for (const Tap &tx : p.taps[2][rx])
                        for (int ks = 0; ks < A.KS; ++ks) {
                            if (t >= kGMaxSteps) return false;
                            A.steps[t++] = ((ty.e - emin_y) * A.SW + (tx.e - emin_x)) * A.pst + 32 * ks;
                        }
                while (t % 4) {
                    if (t >= kGMaxSteps) return false;
                    A.steps[t++] = 0;
                }
            }
        A.n_steps = t;
    }
    A.n_rb = (int32_t)ceil_div(A.nJy, A.JB);
    A.n_seg = (int32_t)ceil_div(A.nJx, 16);
    A.vec8 = (A.out_x % 8) == 0;
    A.segp = 16 * A.s_x + 16;
    // input tile by TMA: the row pitch must be a multiple of 16 bytes and the
    // tile's first column 16-byte aligned, so it starts at emin_x rounded down
    // to a multiple of 8 and is dx columns wider
    A.x0 = emin_x >= 0 ? emin_x / 8 * 8 : -((-emin_x + 7) / 8 * 8);
    A.dx = emin_x - A.x0;
    A.BW = (int32_t)round_up((size_t)(A.SW + A.dx), 8);
    A.use_tma = (A.in_x % 8 == 0) && A.BW <= 256 && A.SR <= 256;
    A.raw_bytes = A.use_tma ? A.Cg * A.SR * A.BW * 2 : 0;
    A.one_phase = one_phase_steps(A);
    A.stage_bytes = A.one_phase ? 0 : kGWarps * A.MT * 16 * A.segp * 2;
    const size_t region0 = round_up((size_t)std::max(A.raw_bytes, A.stage_bytes), 128);
    const size_t slab = round_up((size_t)A.npix * A.pst, 128);
    const size_t wbytes = (size_t)A.n_pairs * A.KS * A.MT * 512;
    const size_t steps = round_up((size_t)A.n_steps * 4, 16);
    A.off_slab = (int32_t)region0;
    A.off_w = (int32_t)(region0 + slab);
    A.off_steps = (int32_t)(A.off_w + wbytes);
    A.off_bias = (int32_t)(A.off_steps + steps);
    A.off_bar = A.off_bias + 128;
    const size_t total = (size_t)A.off_bar + 16;
    if (total > (size_t)(1 << 30)) return false;
    A.smem_total = (int32_t)total;
    // the kernel's 32-bit index ranges: slab tasks, staging, items
    const long long tasks = (long long)A.KS * 2 * A.npix;
    const long long seg_elems = (long long)A.Mg * 16 * A.s_x;
    if (tasks >= (1LL << 24) || seg_elems >= (1LL << 24)) return false;
    const long long items = (long long)A.JB * A.n_live_ry * A.n_seg;
    if (items >= (1LL << 24) || (long long)A.JB * A.n_dead_ry >= (1LL << 24)) return false;
    A.d_npix = make_magic((uint32_t)A.npix);
    A.d_sw = make_magic((uint32_t)A.SW);
    A.d_seg = make_magic((uint32_t)A.n_seg);
    A.d_lry = make_magic((uint32_t)A.n_live_ry);
    A.d_drow = make_magic((uint32_t)std::max(1, A.n_dead_ry));
    A.d_segw = make_magic((uint32_t)(16 * A.s_x));
    A.d_rb = make_magic((uint32_t)A.n_rb);
    A.d_g = make_magic((uint32_t)A.G);
    A.d_cols = make_magic((uint32_t)(A.vec8 ? A.out_x / 8 : A.out_x));
    A.d_cprs = make_magic((uint32_t)(A.segp / 8));
    A.d_cprc = make_magic((uint32_t)(2 * A.s_x));
    return true;
}

size_t grouped_packed_bytes(const Plan &p) {
    GroupedArgs A;
    grouped_setup(p, A, 1);
    return (size_t)A.G * A.n_pairs * A.KS * A.MT * 32 * 16;
}

// CTAs of grouped_stream_kernel<NSTEP> resident per SM with `smem` bytes of
// shared memory (the occupancy calculator when a device answers, else the
// launch bound and the shared-memory capacity).
template <int NSTEP>
int stream_blocks_per_sm_n(int smem) {
    static std::atomic<int> attr_set[64];
    int n = 0;
    if (allow_smem(grouped_stream_kernel<NSTEP, CT_ACT_IDENTITY>, attr_set, kGSmem) &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, grouped_stream_kernel<NSTEP, CT_ACT_IDENTITY>, kGThreads,
                                                      (size_t)smem) == cudaSuccess &&
        n > 0)
        return n;
    cudaGetLastError();
    return std::min(kGOnePhaseMinBlocks, (228 * 1024) / (smem + 1024));
}

int stream_blocks_per_sm(int nstep, int smem) {
    switch (nstep) {
        case 1: return stream_blocks_per_sm_n<1>(smem);
        case 2: return stream_blocks_per_sm_n<2>(smem);
        case 3: return stream_blocks_per_sm_n<3>(smem);
        case 4: return stream_blocks_per_sm_n<4>(smem);
        case 6: return stream_blocks_per_sm_n<6>(smem);
        case 8: return stream_blocks_per_sm_n<8>(smem);
        case 9: return stream_blocks_per_sm_n<9>(smem);
        case 12: return stream_blocks_per_sm_n<12>(smem);
    }
    return 0;
}

// The streaming form of the one-phase path for J-row blocks of `jb` rows:
// the input tile widened so that its channel stride is an odd number of
// 16-byte units (SRt rows, BW columns, both giving an odd count), the bias
// tiles and the shared-memory layout.  False when the shape or the block
// does not suit it.
bool stream_setup(const Plan &p, GroupedArgs &A, int jb) {
    if (!grouped_setup(p, A, jb)) return false;
    if (!A.one_phase || !A.use_tma || !A.vec8 || A.out_x > 256 || A.Mg > 64) return false;
    if ((long long)A.N * A.M >= (1LL << 31) || (long long)A.N * A.C >= (1LL << 31)) return false;
    if ((A.BW / 8) % 2 == 0) A.BW += 8;
    A.SRt = A.SR | 1;
    if (A.BW > 256 || A.SRt > 256) return false;
    A.raw_bytes = A.Cg * A.SRt * A.BW * 2;
    A.btile_bytes = A.n_dead_ry > 0 ? (int32_t)round_up((size_t)A.Mg * A.out_x * 2, 128) : 0;
    const size_t tile = round_up((size_t)A.raw_bytes, 128);
    const size_t slab = round_up((size_t)A.npix * A.pst, 128);
    A.off_slab = (int32_t)tile;
    A.off_btile = (int32_t)(tile + slab);
    A.off_wst = A.off_btile + 2 * A.btile_bytes;
    A.off_sb = A.off_wst + 2 * A.one_phase * 512;
    A.off_bar = A.off_sb + 2 * 64 * 2;
    A.smem_total = A.off_bar + 32;   // barrier, then a 16-byte sink for pixels outside the slab
    if (A.smem_total > kGSmem) return false;
    A.d_qn = make_magic((uint32_t)(A.BW / 8));
    A.d_hn = make_magic((uint32_t)(A.Cg / 8));
    A.n_seg32 = (A.nJx + 31) / 32;
    A.d_seg32 = make_magic((uint32_t)A.n_seg32);
    A.stream = 1;
    return true;
}

// Pick the streaming form's J-row block: among blocks whose shared memory
// leaves kGOnePhaseMinBlocks CTAs per SM, the fewest rounds of the grid
// times the 32-J items each compute warp takes per block plus one (the
// re-layout and per-block set-up in item units).
bool stream_plan(const Plan &p, GroupedArgs &A) {
    const long long sms = sm_count();
    long long best_cost = -1;
    int best_jb = 0, best_per_sm = 0;
    for (int jb = 2; jb <= 32; ++jb) {
        GroupedArgs T;
        if (!stream_setup(p, T, jb)) continue;
        const int per_sm = stream_blocks_per_sm(T.one_phase, T.smem_total);
        if (per_sm < kGOnePhaseMinBlocks) continue;
        const long long slots = (long long)per_sm * sms;
        const long long blocks = (long long)T.N * T.G * T.n_rb;
        const long long cost = ceil_div(blocks, slots) * (ceil_div((long long)T.JB * T.n_seg32, kGWarps - 1) + 1);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_jb = jb;
            best_per_sm = per_sm;
        }
        if (T.JB >= T.nJy) break;
    }
    if (best_cost < 0 || !stream_setup(p, A, best_jb)) return false;
    const long long blocks = (long long)A.N * A.G * A.n_rb;
    if (blocks > 0x7fffffffLL) return false;
    A.grid = (int32_t)std::min<long long>(blocks, (long long)best_per_sm * sms);
    return true;
}

void grouped_plan(Plan &p) {
    p.aux.assign((sizeof(GroupedArgs) + 7) / 8, 0);
    GroupedArgs &A = *reinterpret_cast<GroupedArgs *>(p.aux.data());
    if (stream_plan(p, A)) {
        p.launches = 1;
        return;
    }
    // J rows per CTA: the largest power of two whose shared memory stays
    // within 56 KB (four CTAs per SM) while the grid still gives every SM
    // a dozen CTAs; one row at least.
    const long long sms = sm_count();
    int best = 1;
    for (int jb = 1; jb <= 64; jb *= 2) {
        GroupedArgs T;
        if (!grouped_setup(p, T, jb)) break;
        if (jb > 1 && (T.smem_total > 56 * 1024 || (long long)T.N * T.G * T.n_rb < 12 * sms)) break;
        best = jb;
        if (T.JB >= T.nJy) break;
    }
    grouped_setup(p, A, best);
    p.launches = 1;
}


ct_status grouped_prepack(const Plan &p, const void *w, void *wp, cudaStream_t st) {
    const GroupedArgs &A = gargs(p);
    const long long total = (long long)A.G * A.n_pairs * A.KS * A.MT * 256;
    long long blocks = ceil_div(total, 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    grouped_prepack_kernel<<<(unsigned)blocks, 256, 0, st>>>(A, (const __half *)w, (__half *)wp);
    return launch_status();
}

template <int MT, int NSTEP, int ACT>
ct_status launch_grouped_act(const CUtensorMap &tm, const GroupedArgs &A, const void *x, const void *wp,
                             const void *bias, void *y, unsigned grid, cudaStream_t st) {
    static std::atomic<int> attr_set[64];
    if (!allow_smem(grouped_kernel<MT, NSTEP, ACT>, attr_set, kGSmem)) return CT_ERR_DEVICE;
    grouped_kernel<MT, NSTEP, ACT><<<grid, kGThreads, (size_t)A.smem_total, st>>>(
        tm, A, (const __half *)x, (const uint4 *)wp, (const __half *)bias, (__half *)y);
    return launch_status();
}

template <int MT, int NSTEP>
ct_status launch_grouped(const CUtensorMap &tm, const GroupedArgs &A, const void *x, const void *wp,
                         const void *bias, void *y, unsigned grid, cudaStream_t st) {
    if (A.act == CT_ACT_RELU) return launch_grouped_act<MT, NSTEP, CT_ACT_RELU>(tm, A, x, wp, bias, y, grid, st);
    return launch_grouped_act<MT, NSTEP, CT_ACT_IDENTITY>(tm, A, x, wp, bias, y, grid, st);
}

template <int NSTEP, int ACT>
ct_status launch_stream_act(const CUtensorMap &tmx, const CUtensorMap &tmy, const GroupedArgs &A, const void *wp,
                            const void *bias, void *y, cudaStream_t st) {
    static std::atomic<int> attr_set[64];
    if (!allow_smem(grouped_stream_kernel<NSTEP, ACT>, attr_set, kGSmem)) return CT_ERR_DEVICE;
    grouped_stream_kernel<NSTEP, ACT><<<(unsigned)A.grid, kGThreads, (size_t)A.smem_total, st>>>(
        tmx, tmy, A, (const uint4 *)wp, (const __half *)bias, (__half *)y);
    return launch_status();
}

template <int NSTEP>
ct_status launch_stream(const CUtensorMap &tmx, const CUtensorMap &tmy, const GroupedArgs &A, const void *wp,
                        const void *bias, void *y, cudaStream_t st) {
    if (A.act == CT_ACT_RELU) return launch_stream_act<NSTEP, CT_ACT_RELU>(tmx, tmy, A, wp, bias, y, st);
    return launch_stream_act<NSTEP, CT_ACT_IDENTITY>(tmx, tmy, A, wp, bias, y, st);
}

ct_status grouped_stream_run(const GroupedArgs &A, const void *x, const void *wp, const void *bias, void *y,
                             cudaStream_t st) {
    if (A.grid <= 0) return CT_OK;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CT_ERR_DEVICE;
    CUtensorMap tmx, tmy;
    memset(&tmx, 0, sizeof(tmx));
    memset(&tmy, 0, sizeof(tmy));
    {
        // X as (x, y, image * channel); the box is one block's input tile
        const cuuint64_t dims[3] = {(cuuint64_t)A.in_x, (cuuint64_t)A.in_y, (cuuint64_t)A.N * A.C};
        const cuuint64_t strides[2] = {(cuuint64_t)A.in_x * 2, (cuuint64_t)A.in_x * A.in_y * 2};
        const cuuint32_t box[3] = {(cuuint32_t)A.BW, (cuuint32_t)A.SRt, (cuuint32_t)A.Cg};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    {
        // Y as (x, y, image * channel); the box is one output row of a group's channels
        const cuuint64_t dims[3] = {(cuuint64_t)A.out_x, (cuuint64_t)A.out_y, (cuuint64_t)A.N * A.M};
        const cuuint64_t strides[2] = {(cuuint64_t)A.out_x * 2, (cuuint64_t)A.out_x * A.out_y * 2};
        const cuuint32_t box[3] = {(cuuint32_t)A.out_x, 1, (cuuint32_t)A.Mg};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmy, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    switch (A.one_phase) {
        case 1: return launch_stream<1>(tmx, tmy, A, wp, bias, y, st);
        case 2: return launch_stream<2>(tmx, tmy, A, wp, bias, y, st);
        case 3: return launch_stream<3>(tmx, tmy, A, wp, bias, y, st);
        case 4: return launch_stream<4>(tmx, tmy, A, wp, bias, y, st);
        case 6: return launch_stream<6>(tmx, tmy, A, wp, bias, y, st);
        case 8: return launch_stream<8>(tmx, tmy, A, wp, bias, y, st);
        case 9: return launch_stream<9>(tmx, tmy, A, wp, bias, y, st);
        case 12: return launch_stream<12>(tmx, tmy, A, wp, bias, y, st);
    }
    return CT_ERR_UNSUPPORTED;
}

ct_status grouped_run(const Plan &p, const void *x, const void *wp, const void *bias, void *y,
                      cudaStream_t st) {
    const GroupedArgs &A = gargs(p);
    if (A.stream) return grouped_stream_run(A, x, wp, bias, y, st);
    if (A.smem_total > kGSmem) return CT_ERR_UNSUPPORTED;
    const long long grid = (long long)A.N * A.G * A.n_rb;
    if (grid > 0x7fffffffLL) return CT_ERR_UNSUPPORTED;
    CUtensorMap tm;
    memset(&tm, 0, sizeof(tm));
    if (A.use_tma) {
        EncodeTiledFn enc = encode_fn();
        if (!enc) return CT_ERR_DEVICE;
        const cuuint64_t dims[3] = {(cuuint64_t)A.in_x, (cuuint64_t)A.in_y, (cuuint64_t)A.N * A.C};
        const cuuint64_t strides[2] = {(cuuint64_t)A.in_x * 2, (cuuint64_t)A.in_x * A.in_y * 2};
        const cuuint32_t box[3] = {(cuuint32_t)A.BW, (cuuint32_t)A.SR, (cuuint32_t)A.Cg};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CT_ERR_DEVICE;
    }
    switch (A.one_phase) {
        case 1: return launch_grouped<1, 1>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 2: return launch_grouped<1, 2>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 3: return launch_grouped<1, 3>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 4: return launch_grouped<1, 4>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 6: return launch_grouped<1, 6>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 8: return launch_grouped<1, 8>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 9: return launch_grouped<1, 9>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 12: return launch_grouped<1, 12>(tm, A, x, wp, bias, y, (unsigned)grid, st);
    }
    switch (A.MT) {
        case 1: return launch_grouped<1, 0>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 2: return launch_grouped<2, 0>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 3: return launch_grouped<3, 0>(tm, A, x, wp, bias, y, (unsigned)grid, st);
        case 4: return launch_grouped<4, 0>(tm, A, x, wp, bias, y, (unsigned)grid, st);
    }
    return CT_ERR_UNSUPPORTED;
}

int grouped_take_error(cudaStream_t st) { return take_error_word(g_grouped_err, st); }

}  // namespace ct
