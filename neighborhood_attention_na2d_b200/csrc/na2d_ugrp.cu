// na2d_ugrp.cu -- NA2D forward on the 5th-generation tensor cores (tcgen05)
// for maps whose dilation groups are between k and 16 pixels on each side,
// with k >= 9 (f16 / bf16, D = 32): for instance the segmentation-scale
// k = 13, d = 8 layer on a 128 x 128 map, whose groups are 16 x 16.
//
// What it computes is the same as the other forward kernels ("Dilated
// Neighborhood Attention Transformer", gitcode DiNAT article, section
// "DiNAT 的核心思想": natten2dqkrpb -> softmax -> natten2dav, fused, NATTEN
// clamp rule).  In a group at most 16 long the windows of 8 consecutive query
// rows together cover at most k + 1 key rows when k >= 13, and at most 12
// and 13 rows for k = 9 and 11 (the clamp keeps the window starts of
// neighbouring rows together), so 8 x 16 queries against a key tile of NKR
// group rows (NKR <= 14) form a dense contraction whose scores are mostly
// used (169 of 224 at k = 13): it is one M = 128 tcgen05 tile.
//
// Work unit: one dilation group.  Its Q, K and V arrive by TMA as a 16 x 16
// box of pixels (columns past the group's width zero-filled, rows past its
// height whatever finite values follow), 64 bytes per pixel, 64-byte
// swizzled: slot 16 * row + col is tile row 16 * row + col.  Strip e (group
// rows 8e .. 8e + 7) is the M = 128 tile of Q rows 128e .. 128e + 127; its
// keys are the group rows kr0[e] .. kr0[e] + NKR - 1 (tile rows from
// 16 kr0[e]), split into a lower and an upper half of key rows.
//   1. S = Q K^T per half: two tcgen05.mma (K = 16 each, both operands
//      K-major in shared memory), N = 16 rows of the half, fp32 in tensor
//      memory (TMEM).
//   2. softmax: one thread per query (its TMEM lane), packed fp32x2
//      arithmetic.  Scores are scaled and biased from a shared-memory table
//      that holds, per query column and relative key row, the 16 bias values
//      of a key row in log2 units with the window mask folded in (-1e30
//      outside the window; a key row outside the query's window reads an
//      all-masked row, so every row is processed without branches).  Pass 1
//      writes the biased scores back and takes their maximum; pass 2
//      exponentiates (a quarter of the columns on the FMA pipe) and writes P
//      as 16-bit pairs over the upper half's scores.
//   3. O = P V: NKR tcgen05.mma (K = 16 keys = one key row each, A = P in
//      TMEM, B = V MN-major in shared memory).
//   4. epilogue: the same thread loads its O row, divides by its row sum and
//      stores 64 bytes; it runs after the next unit's softmax.
// Warpgroup e (warps 4e .. 4e + 3) runs strip e of every unit, with two TMEM
// score regions of 16 ceil(NKR / 2) columns and an O buffer of 32 columns.
// Warp 8, lane 0 issues the TMA copies into a ring of NSTG stages; warps 9
// and 10, lane 0, issue the MMAs of strip 0 and strip 1 (the next unit's
// upper-half Q K^T, this unit's P.V, the next unit's lower-half Q K^T) and
// signal completion with tcgen05.commit on mbarriers; warp 9 owns the TMEM
// allocation.  Every wait is bounded: one that runs out counts the event,
// raises the block's abort flag, and the block winds down (its MMAs and
// copies in flight are waited for before TMEM and shared memory are
// released).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <set>
#include <type_traits>

#include "na2d_device.cuh"
#include "na2d_launch.h"
#include "na2d_tcgen05.cuh"

namespace na2d {
namespace {

constexpr int NSTG = 3;                    // shared-memory stages (units in flight)
constexpr uint32_t kGroupBytes = 16384;    // one tensor of a unit: 16 x 16 pixels of 64 bytes
constexpr uint32_t kStage = 3 * kGroupBytes;
constexpr int kMaxNKR = 14;                // two S buffers of 16 NKR columns and two O buffers fit in TMEM
constexpr int kThreads = 352;              // 8 softmax warps, producer warp, two MMA warps
constexpr int kWarpTma = 8, kWarpMma = 9;  // MMA warps 9 (strip 0) and 10 (strip 1)
constexpr float kMasked = -1.0e30f;        // bias outside the window: exp2 gives 0

__device__ unsigned int g_ugrp_timeouts;

struct UgrpParams {
    CUtensorMap tq, tk, tv;   // 5-D group views, 32 x 1 x 16 x 1 x 16 boxes
    unsigned char *out;
    const void *rpb;
    int H, W, heads, d, k;
    int Lgy, Lgx;             // group height and width
    int GU;                   // units (groups): B * heads * d * d
    int NKR;                  // key rows of a strip's tile
    int kr0[2];               // first group row of strip 0 / 1's key tile
    float c_log2;             // log2(e) / sqrt(D)
    long long wait_limit;     // SM clocks a data wait may take
    uint32_t qstride;         // bytes per query column of a bias table
    uint32_t tab_bytes;       // bytes per bias table (16 query columns)
    uint32_t off_tab, off_bar, off_rpb;   // byte offsets from the 1024-aligned base
};

// Stores 8 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st8(uint32_t ta, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(ta), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// 2^x for x <= 0 on the FMA and integer pipes, for a share of the
// exponentials that the MUFU pipe (4 results per clock and sub-partition)
// would otherwise serialise: x = r + f with r = round(x) and |f| <= 1/2; 2^f
// from a cubic fitted to it on [-1/2, 1/2] (least squares on the relative
// error, with p(0) = 1; largest relative error 1.0e-4, below the 16-bit
// rounding of P), then r added to the exponent field.  Arguments below -125
// (masked keys) give 2^-125, which rounds to zero in f16 and contributes
// nothing measurable in bf16.
// Two at a time with packed fp32x2 arithmetic.
__device__ __forceinline__ void ex2_fma2(float &y0, float &y1, float x0, float x1) {
    x0 = fmaxf(x0, -125.f);
    x1 = fmaxf(x1, -125.f);
    float xr0, xr1, r0, r1, f0, f1, p0, p1;
    add2(xr0, xr1, x0, x1, 12582912.f, 12582912.f);   // 1.5 * 2^23: round(x) in the low mantissa bits
    add2(r0, r1, xr0, xr1, -12582912.f, -12582912.f);
    fma2(f0, f1, r0, r1, -1.f, x0, x1);                 // f = x - round(x)
    fma2(p0, p1, f0, f1, 0.05500755f, 0.24220777f, 0.24220777f);
    fma2v(p0, p1, p0, p1, f0, f1, 0.69328272f, 0.69328272f);
    fma2v(p0, p1, p0, p1, f0, f1, 1.f, 1.f);
    y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(xr0) << 23));
    y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(xr1) << 23));
}

// ---------------------------------------------------------------------------
// Kernel.
// ---------------------------------------------------------------------------
template <typename T, int NKR>
__global__ void __launch_bounds__(kThreads, 1) fwd_ugrp_kernel(const __grid_constant__ UgrpParams p) {
    static_assert(NKR >= 2 && NKR <= kMaxNKR, "key tile of 2 .. 14 group rows");
    // The key tile's rows in two halves: lower rows 0 .. NL - 1 and upper rows
    // NL .. NKR - 1, whose scores are computed by separate MMAs into two
    // TMEM regions of HS columns each.  For unit j with h = j & 1 the upper
    // scores go to region h and the lower ones to region 1 - h; P is written
    // into region h (over the upper scores: order index o = upper rows first,
    // then lower rows, at column 8o).  Unit j + 1's upper scores then go to
    // region 1 - h, free once unit j's softmax has read its lower scores, and
    // can be computed before unit j's P.V; its lower scores follow the P.V.
    constexpr int NL = NKR / 2, NH = NKR - NL;
    constexpr int HS = 16 * NH;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;   // swizzled tiles need 1024-byte alignment
    unsigned char *smem = smem_raw + (sbase - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u_begin = (int)((int64_t)p.GU * blockIdx.x / gridDim.x);
    const int u_end = (int)((int64_t)p.GU * (blockIdx.x + 1) / gridDim.x);
    grid_dep_launch();
    if (u_begin >= u_end) return;
    const int nst = u_end - u_begin;
    const int dd = p.d * p.d;
    // the block's units lie in at most two (batch, head) planes (the launch
    // sizes the ranges so), each with its own bias table
    const int bh_first = u_begin / dd;
    if ((u_end - 1) / dd - bh_first > 1) {   // never, by the launch; counted rather than overrun the tables
        if (threadIdx.x == 0) atomicAdd(&g_ugrp_timeouts, 1u);
        return;
    }

    const uint32_t bar_full = sbase + p.off_bar;        // [NSTG] stage landed (TMA bytes)
    const uint32_t bar_empty = bar_full + 8 * NSTG;     // [NSTG] stage consumed (two commits)
    const uint32_t bar_sh = bar_empty + 8 * NSTG;       // [2] upper scores of strip e ready (commit)
    const uint32_t bar_sl = bar_sh + 16;                // [2] lower scores ready (commit)
    const uint32_t bar_p = bar_sl + 16;                 // [2] P_e written (4 warps)
    const uint32_t bar_o = bar_p + 16;                  // [2] O_e ready (commit)
    const uint32_t bar_drain = bar_o + 16;              // [2] all MMAs of an MMA warp done (commit)
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_bar + 16 * NSTG + 80);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_bar + 16 * NSTG + 84);

    auto issue_unit = [&](int j) {
        const uint32_t fb = bar_full + 8 * (j % NSTG);
        const uint32_t st = sbase + (uint32_t)(j % NSTG) * kStage;
        mb_expect_tx(fb, kStage);
        const int g = u_begin + j;
        const int bh = g / dd, rem = g - bh * dd, gy = rem / p.d, gx = rem - gy * p.d;
        const int row = bh * p.Lgy;   // merged (plane, group row) coordinate of group row 0
        tma_load_5d(st, &p.tq, fb, gx, 0, gy, row);
        tma_load_5d(st + kGroupBytes, &p.tk, fb, gx, 0, gy, row);
        tma_load_5d(st + 2 * kGroupBytes, &p.tv, fb, gx, 0, gy, row);
    };
    const int n_first = min(2, nst);

    // ---- prologue.  The producer thread initialises the barriers and starts
    // the first units' copies; meanwhile the other threads build the bias
    // tables and allocate TMEM.
    {
        if (warp == kWarpTma && lane == 0) {
            for (int i = 0; i < NSTG; ++i) {
                mb_init(bar_full + 8 * i, 1);
                mb_init(bar_empty + 8 * i, 2);
            }
            for (int i = 0; i < 2; ++i) {
                mb_init(bar_sh + 8 * i, 1);
                mb_init(bar_sl + 8 * i, 1);
                mb_init(bar_p + 8 * i, 4);
                mb_init(bar_o + 8 * i, 1);
                mb_init(bar_drain + 8 * i, 1);
            }
            *abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
            grid_dep_wait();   // before the first copy
            for (int j = 0; j < n_first; ++j) issue_unit(j);
        }
        grid_dep_wait();   // before the bias tables' reads
        // table t (plane bh_first + t), query column qc, row a, key column j:
        // a < 2k - 1 is the relative key row a - (k - 1); a = 2k - 1 is an
        // all-masked row.  Entry: rpb[h, a, j - qc + k - 1] * log2(e) when key
        // column j is in the window of query column qc, else kMasked.  Query
        // columns past the group's width take the last column's window and
        // bias (their outputs are not stored).
        const int k = p.k, nrel = 2 * k - 1, nr2 = nrel * nrel;
        const int nplanes = (u_end - 1) / dd - bh_first + 1;
        // the planes' bias rows first, in log2 units (all loads in flight at once)
        float *rpbs = reinterpret_cast<float *>(smem + p.off_rpb);
        const T *rpb = reinterpret_cast<const T *>(p.rpb);
        for (int i = threadIdx.x; i < nplanes * nr2; i += kThreads) {
            const int t = i / nr2, r = i - t * nr2;
            const int h = (int)((bh_first + t) % p.heads);
            rpbs[i] = rpb ? Elem<T>::to_f(rpb[(int64_t)h * nr2 + r]) * kLog2e : 0.f;
        }
        __syncthreads();
        // one 16-entry table row (plane t, query column qc, row a) per step
        const int rows_per_tab = 16 * 2 * k;
        for (int ri = threadIdx.x; ri < nplanes * rows_per_tab; ri += kThreads) {
            const int t = ri / rows_per_tab, rr = ri - t * rows_per_tab;
            const int qc = rr / (2 * k), a = rr - qc * (2 * k);
            const int qcc = min(qc, p.Lgx - 1);
            const int wx = window_start(qcc, p.Lgx, k);
            // key column j of query column qcc is bias column j - qcc + k - 1
            const float *src = rpbs + t * nr2 + a * nrel + (k - 1 - qcc);
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = (a < nrel && (unsigned)(j - wx) < (unsigned)k) ? src[j] : kMasked;
            float4 *dst = reinterpret_cast<float4 *>(smem + p.off_tab + (uint32_t)t * p.tab_bytes +
                                                     (uint32_t)qc * p.qstride + (uint32_t)a * 64u);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        }
        if (warp == kWarpMma) tmem_alloc(smem_u32(tmem_slot));
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma) {
        // =================== TMA producer ===================
        if (lane == 0) {
            int issued = n_first;
            for (int j = n_first; j < nst; ++j) {
                const int s = j % NSTG;
                if (j >= NSTG && !mb_wait(bar_empty + 8 * s, (uint32_t)(((j / NSTG) - 1) & 1), p.wait_limit)) {
                    atomicAdd(&g_ugrp_timeouts, 1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                issue_unit(j);
                ++issued;
            }
            // copies still in flight land before shared memory is released
            for (int j = max(0, issued - NSTG); j < issued; ++j)
                mb_wait(bar_full + 8 * (j % NSTG), (uint32_t)((j / NSTG) & 1));
        }
    } else if (warp == kWarpMma || warp == kWarpMma + 1) {
        // =================== MMA issuers ===================
        // Warp kWarpMma + e issues strip e of every unit: unit 0's upper and
        // lower Q K^T, then per unit j: unit j + 1's upper Q K^T (into the
        // region unit j's softmax has finished reading), O_j = P_j V_j, unit
        // j + 1's lower Q K^T (into the region of P_j, after the P.V that
        // reads it: tcgen05.mma of one thread execute in issue order).  O_j
        // is free again once the warpgroup's epilogue of unit j - 1, which
        // precedes its P_j, has read it.
        const int e = warp - kWarpMma;
        if (lane == 0) {
            constexpr uint32_t idesc_hi = idesc_f16<T>(16 * NH, 0);
            constexpr uint32_t idesc_lo = idesc_f16<T>(16 * NL, 0);
            constexpr uint32_t idesc_pv = idesc_f16<T>(32, 1);
            const uint32_t koff = (uint32_t)p.kr0[e] * 1024u;   // 16 pixels of 64 bytes per group row
            const uint32_t dR = tmem + (uint32_t)(e * 2 * HS), dO = tmem + (uint32_t)(4 * HS + 32 * e);
            // one half of unit j's Q K^T; the upper half first waits for the unit's copies
            auto issue_qk = [&](int j, bool upper) -> bool {
                const int s = j % NSTG;
                if (upper) {
                    if (!mb_wait(bar_full + 8 * s, (uint32_t)((j / NSTG) & 1), p.wait_limit) || *abort_flag)
                        return false;
                    tc_fence_after();
                }
                const uint32_t st = sbase + (uint32_t)s * kStage;
                const int h = j & 1;
                // K-major, 64-byte rows: 8-row groups 512 bytes apart; the
                // second K = 16 step starts 32 bytes into the rows
                const uint64_t da = sw64_desc(st + (uint32_t)e * 8192u, 16, 512);
                const uint64_t db = sw64_desc(st + kGroupBytes + koff + (upper ? (uint32_t)NL * 1024u : 0u), 16, 512);
                const uint32_t dS = dR + (uint32_t)((upper ? h : 1 - h) * HS);
                umma_ss(dS, da, db, upper ? idesc_hi : idesc_lo, 0);
                umma_ss(dS, da + 2, db + 2, upper ? idesc_hi : idesc_lo, 1);
                umma_commit((upper ? bar_sh : bar_sl) + 8 * e);
                return true;
            };
            bool ok = issue_qk(0, true) && issue_qk(0, false);
            for (int j = 0; ok && j < nst; ++j) {
                const int s = j % NSTG;
                if (!mb_wait(bar_p + 8 * e, (uint32_t)(j & 1), p.wait_limit) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (j + 1 < nst && !issue_qk(j + 1, true)) {
                    ok = false;
                    break;
                }
                const uint32_t vt = sbase + (uint32_t)s * kStage + 2 * kGroupBytes + koff;
                const uint32_t aP = dR + (uint32_t)((j & 1) * HS);
                // V MN-major: 64-byte rows of 32 channels, 8-key groups 512
                // bytes apart; k-step o takes P columns 8o .. 8o + 7, i.e. key
                // row NL + o for o < NH and o - NH after
#pragma unroll
                for (int o = 0; o < NKR; ++o) {
                    const int t = o < NH ? NL + o : o - NH;
                    umma_ts(dO, aP + 8u * (uint32_t)o, sw64_desc(vt + 1024u * (uint32_t)t, 16, 512), idesc_pv,
                            o > 0 ? 1u : 0u);
                }
                umma_commit(bar_o + 8 * e);
                umma_commit(bar_empty + 8 * s);
                if (j + 1 < nst) issue_qk(j + 1, false);
            }
            if (!ok) {
                atomicAdd(&g_ugrp_timeouts, 1u);
                *abort_flag = 1;
            }
            // every MMA this thread issued has completed before TMEM is released
            umma_commit(bar_drain + 8 * e);
            mb_wait(bar_drain + 8 * e, 0);
        }
    } else {
        // =================== softmax warpgroups ===================
        const int e = warp >> 2;                      // strip of this warpgroup
        const int q4 = warp & 3;                      // lane quarter of this warp
        const int m = q4 * 32 + lane;                 // tile row = TMEM lane
        const int qr = m >> 4, qc = m & 15;           // query slot within the strip
        const int row = 8 * e + qr;                   // group row
        const bool qok = row < p.Lgy && qc < p.Lgx;
        const int rowc = min(row, p.Lgy - 1);
        const int k = p.k;
        // key-tile rows wy .. wy + k - 1 are this query's window rows
        const int wy = window_start(rowc, p.Lgy, k) - p.kr0[e];
        // table row of key-tile row i: a0 + i (relative row + k - 1) when valid
        const int a0 = p.kr0[e] - rowc + k - 1;
        const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
        const uint32_t tR = tl + (uint32_t)(e * 2 * HS), tO = tl + (uint32_t)(4 * HS + 32 * e);
        const float c = p.c_log2;
        const bool st32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
        const unsigned char *tab_q = smem + p.off_tab + (uint32_t)qc * p.qstride;
        const int nrel = 2 * k - 1;

        float l_prev = 1.f;   // row sum of the unit whose output is pending
        // Position of unit j's group (plane bh, group row gy and column gx),
        // advanced by one group per unit by carries instead of divisions.
        struct GPos {
            int bh, gy, gx;
        };
        GPos pos;
        pos.bh = u_begin / dd;
        pos.gy = (u_begin - pos.bh * dd) / p.d;
        pos.gx = u_begin - pos.bh * dd - pos.gy * p.d;
        GPos prev = pos;
        auto advance = [&](GPos &x) {
            if (++x.gx == p.d) {
                x.gx = 0;
                if (++x.gy == p.d) {
                    x.gy = 0;
                    ++x.bh;
                }
            }
        };
        // O of unit jj (ready once its P.V completed) / row sum -> 64 bytes;
        // at is unit jj's position
        auto epilogue = [&](int jj, const GPos &at) -> bool {
            const bool oko = mb_wait(bar_o + 8 * e, (uint32_t)(jj & 1), p.wait_limit);
            if (!__all_sync(0xffffffffu, oko)) {
                if (lane == 0) {
                    atomicAdd(&g_ugrp_timeouts, 1u);
                    *abort_flag = 1;
                }
                return false;
            }
            tc_fence_after();
            float o[32];
            tmem_ld32(tO, o);
            tmem_ld_wait();
            if (qok) {
                float inv;
                asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(inv) : "f"(l_prev));
                store_pixel64<T>(
                    p.out + ((((size_t)at.bh * p.H + at.gy + (size_t)p.d * row) * p.W) + at.gx + (size_t)p.d * qc) * 64,
                    o, inv, st32);
            }
            return true;
        };
        constexpr int kB = 2;   // key rows per wait for the TMEM loads
        // batches unrolled two deep (one deep at NKR = 11 and 12, where two spill registers)
        constexpr int kU = (NKR == 11 || NKR == 12) ? 1 : 2;
        const float4 *tq = nullptr;
        float mxr[kB], lr[kB][2];
        // pass 1 over CNT key rows from i_first, scores at TMEM column col0 +
        // 16o: biased scores (log2 units) written back, running maxima.  No
        // branches: a row outside this query's window reads the table's
        // all-masked row.
        auto pass1 = [&](uint32_t col0, int i_first, auto CNT) {
            constexpr int cnt = decltype(CNT)::value;
#pragma unroll kU
            for (int o0 = 0; o0 < cnt; o0 += kB) {
                float x[kB][16];
#pragma unroll
                for (int r = 0; r < kB; ++r)
                    if (o0 + r < cnt) tmem_ld16(col0 + 16u * (uint32_t)(o0 + r), x[r]);
                tmem_ld_wait();
#pragma unroll
                for (int r = 0; r < kB; ++r) {
                    if (o0 + r >= cnt) continue;
                    const int i = i_first + o0 + r;
                    float *y = x[r];
                    const float4 *br = tq + ((unsigned)(i - wy) < (unsigned)k ? (a0 + i) : nrel) * 4;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float4 bb = br[t];
                        fma2(y[4 * t + 0], y[4 * t + 1], y[4 * t + 0], y[4 * t + 1], c, bb.x, bb.y);
                        fma2(y[4 * t + 2], y[4 * t + 3], y[4 * t + 2], y[4 * t + 3], c, bb.z, bb.w);
                    }
                    const float m0 = max3(max3(y[0], y[1], y[2]), max3(y[3], y[4], y[5]), max3(y[6], y[7], y[8]));
                    const float m1 = max3(max3(y[9], y[10], y[11]), max3(y[12], y[13], y[14]), y[15]);
                    mxr[r] = max3(mxr[r], m0, m1);
                    uint32_t sb[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) sb[t] = __float_as_uint(y[t]);
                    tmem_st16(col0 + 16u * (uint32_t)(o0 + r), sb);
                }
            }
        };
        // pass 2 over CNT key rows, scores at scol0 + 16o, P (16-bit pairs)
        // to pcol0 + 8o: exp2(score - max), columns 6, 7, 14 and 15 of a row
        // on the FMA pipe, the rest on MUFU; row sums in two fp32 lanes per
        // row slot
        auto pass2 = [&](uint32_t scol0, uint32_t pcol0, float mx, auto CNT) {
            constexpr int cnt = decltype(CNT)::value;
#pragma unroll kU
            for (int o0 = 0; o0 < cnt; o0 += kB) {
                float x[kB][16];
#pragma unroll
                for (int r = 0; r < kB; ++r)
                    if (o0 + r < cnt) tmem_ld16(scol0 + 16u * (uint32_t)(o0 + r), x[r]);
                tmem_ld_wait();
#pragma unroll
                for (int r = 0; r < kB; ++r) {
                    if (o0 + r >= cnt) continue;
                    uint32_t pk[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        float x0, x1, p0, p1;
                        fma2(x0, x1, x[r][2 * t], x[r][2 * t + 1], 1.f, -mx, -mx);
                        if ((t & 3) == 3) {
                            ex2_fma2(p0, p1, x0, x1);
                        } else {
                            p0 = ex2(x0);
                            p1 = ex2(x1);
                        }
                        add2(lr[r][0], lr[r][1], lr[r][0], lr[r][1], p0, p1);
                        pk[t] = Pack2<T>::run(p0, p1);
                    }
                    tmem_st8(pcol0 + 8u * (uint32_t)(o0 + r), pk);
                }
            }
        };
        // a bounded wait for one of this strip's score commits; false ends the warpgroup
        auto wait_scores = [&](uint32_t bar, int j) -> bool {
            const bool ok = mb_wait(bar + 8 * e, (uint32_t)(j & 1), p.wait_limit);
            if (!__all_sync(0xffffffffu, ok) || __any_sync(0xffffffffu, *abort_flag != 0)) {
                if (lane == 0) {
                    atomicAdd(&g_ugrp_timeouts, 1u);
                    *abort_flag = 1;
                }
                return false;
            }
            tc_fence_after();
            return true;
        };
        for (int j = 0; j < nst; ++j, prev = pos, advance(pos)) {
            tq = reinterpret_cast<const float4 *>(tab_q + (uint32_t)(pos.bh - bh_first) * p.tab_bytes);
            // region of the upper scores (and of P), region of the lower scores
            const uint32_t up = tR + (uint32_t)((j & 1) * HS), lo = tR + (uint32_t)((1 - (j & 1)) * HS);
            // ---- pass 1: the upper rows as soon as their scores land (the
            // previous unit's P.V may still run), then the lower rows
            mxr[0] = mxr[1] = -3.0e38f;
            if (!wait_scores(bar_sh, j)) break;
            pass1(up, NL, std::integral_constant<int, NH>{});
            if (!wait_scores(bar_sl, j)) break;
            pass1(lo, 0, std::integral_constant<int, NL>{});
            const float mx = fmaxf(mxr[0], mxr[1]);
            tmem_st_wait();
            // ---- pass 2: P of the upper rows over their own scores (P row o
            // at 8o overwrites scores of row o / 2 <= o, already read), then
            // P of the lower rows after them (over upper scores, all read)
            lr[0][0] = lr[0][1] = lr[1][0] = lr[1][1] = 0.f;
            pass2(up, up, mx, std::integral_constant<int, NH>{});
            pass2(lo, up + 8u * NH, mx, std::integral_constant<int, NL>{});
            // ---- the previous unit's epilogue (its P.V completed while this
            // unit's scores were computed), before P_j is handed over: P.V_j
            // overwrites O_e only after the arrive below
            if (j > 0 && !epilogue(j - 1, prev)) break;
            l_prev = (lr[0][0] + lr[0][1]) + (lr[1][0] + lr[1][1]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mb_arrive(bar_p + 8 * e);
            if (j == nst - 1) epilogue(j, pos);
        }
    }
    // ---- teardown: TMEM released by the warp that took it, after every
    // thread is done with it
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem);
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct UgrpCache {
    std::mutex mu;
    std::map<int, std::pair<int, int>> dev;   // device -> (SMs, opt-in smem per block)
    std::set<std::pair<int, const void *>> attr;
};
UgrpCache &gcache() {
    static UgrpCache c;
    return c;
}

cudaError_t ugrp_device(int *sms, int *smem_cap, const void *kern) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    UgrpCache &c = gcache();
    std::lock_guard<std::mutex> lock(c.mu);
    auto it = c.dev.find(dev);
    if (it == c.dev.end()) {
        int n = 0, m = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&m, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
        it = c.dev.emplace(dev, std::make_pair(n, m)).first;
    }
    *sms = it->second.first;
    *smem_cap = it->second.second;
    if (!c.attr.count({dev, kern})) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, *smem_cap);
        if (e != cudaSuccess) return e;
        c.attr.insert({dev, kern});
    }
    return cudaSuccess;
}

std::atomic<long long> &ugrp_limit_store() {
    static std::atomic<long long> v{0};
    return v;
}

// Key tile of each strip: NKR group rows covering the windows of the strip's
// query rows (8e .. min(8e + 7, Lg - 1)), starting at kr0[e] and inside the
// group.
int strip_key_rows(int Lg, int k, int kr0[2]) {
    int nkr = 0;
    int first[2];
    for (int e = 0; e < 2; ++e) {
        const int r0 = 8 * e, r1 = std::min(8 * e + 7, Lg - 1);
        first[e] = window_start(r0, Lg, k);
        nkr = std::max(nkr, window_start(r1, Lg, k) - first[e] + k);
    }
    for (int e = 0; e < 2; ++e) kr0[e] = std::min(first[e], Lg - nkr);
    return nkr;
}

template <typename T> void (*ugrp_kernel(int nkr))(UgrpParams) {
    switch (nkr) {
    case 9: return fwd_ugrp_kernel<T, 9>;
    case 10: return fwd_ugrp_kernel<T, 10>;
    case 11: return fwd_ugrp_kernel<T, 11>;
    case 12: return fwd_ugrp_kernel<T, 12>;
    case 13: return fwd_ugrp_kernel<T, 13>;
    case 14: return fwd_ugrp_kernel<T, 14>;
    default: return nullptr;
    }
}

template <typename T>
cudaError_t launch_ugrp_t(const Problem &pr, const void *q, const void *k, const void *v, const void *rpb, void *out,
                          cudaStream_t st, bool *launched) {
    UgrpParams up{};
    const int64_t bh = pr.bh();
    const int dd = pr.d * pr.d;
    const int64_t gu = bh * dd;
    up.Lgy = pr.H / pr.d;
    up.Lgx = pr.W / pr.d;
    if (gu <= 0 || gu >= INT32_MAX || bh * up.Lgy >= INT32_MAX) return cudaSuccess;
    up.NKR = strip_key_rows(up.Lgy, pr.k, up.kr0);
    void (*kfn)(UgrpParams) = ugrp_kernel<T>(up.NKR);   // NKR is 9 .. 14 for k = 9 .. 13 and groups <= 16
    if (!kfn) return cudaSuccess;
    const void *kern = reinterpret_cast<const void *>(kfn);
    int sms = 0, cap = 0;
    cudaError_t e = ugrp_device(&sms, &cap, kern);
    if (e != cudaSuccess) return e;
    if (!encode_group_map(&up.tq, q, pr.dtype, bh, pr.H, pr.W, pr.d, 16, 16, 1) ||
        !encode_group_map(&up.tk, k, pr.dtype, bh, pr.H, pr.W, pr.d, 16, 16, 1) ||
        !encode_group_map(&up.tv, v, pr.dtype, bh, pr.H, pr.W, pr.d, 16, 16, 1))
        return cudaSuccess;
    up.out = static_cast<unsigned char *>(out);
    up.rpb = rpb;
    up.H = pr.H; up.W = pr.W; up.heads = pr.heads; up.d = pr.d; up.k = pr.k;
    up.GU = (int)gu;
    up.c_log2 = kLog2e / std::sqrt((float)pr.D);
    const long long lim = ugrp_limit_store().load();
    up.wait_limit = lim > 0 ? lim : (1LL << 31);
    // bias table: per query column 2k rows of 16 floats, plus 16 bytes so
    // that the 8 query columns a quarter-warp reads lie in different banks
    up.qstride = (uint32_t)(2 * pr.k * 64 + 16);
    up.tab_bytes = 16 * up.qstride;
    up.off_tab = NSTG * kStage;
    up.off_bar = up.off_tab + 2 * up.tab_bytes;
    up.off_rpb = up.off_bar + 16 * NSTG + 96;   // after the barriers, abort flag and TMEM slot: two planes' (2k - 1)^2 bias values
    const int nrel = 2 * pr.k - 1;
    const uint32_t smem = up.off_rpb + 2u * nrel * nrel * 4u + 1024;   // + 1024 bytes for aligning the base
    if ((int)smem > cap) return cudaSuccess;
    // units per block at most d^2 + 1, so that a block's units lie in at
    // most two (batch, head) planes
    const int64_t grid = std::max<int64_t>(std::min<int64_t>(gu, sms), (gu + dd) / (dd + 1));
    if (grid >= INT32_MAX) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t el = cudaLaunchKernelEx(&cfg, kfn, up);
    *launched = true;
    note_kernel("fwd_ugrp_kernel");
    return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace

bool ugrp_supported(const Problem &p) {
    if (p.dtype != DType::F16 && p.dtype != DType::BF16) return false;
    if (p.D != 32 || p.k < 9 || p.k > 13 || !(p.k & 1) || p.d < 1) return false;
    if (p.H % p.d || p.W % p.d) return false;
    const int Lgy = p.H / p.d, Lgx = p.W / p.d;
    return Lgy >= p.k && Lgy <= 16 && Lgx >= p.k && Lgx <= 16;
}

cudaError_t launch_forward_ugrp(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                void *out, cudaStream_t st, bool *launched) {
    *launched = false;
    if (!ugrp_supported(p)) return cudaSuccess;
    if (p.dtype == DType::F16) return launch_ugrp_t<__half>(p, q, k, v, rpb, out, st, launched);
    return launch_ugrp_t<__nv_bfloat16>(p, q, k, v, rpb, out, st, launched);
}

void set_ugrp_wait_limit(long long clocks) { ugrp_limit_store().store(clocks); }

cudaError_t read_ugrp_faults(unsigned int *count, cudaStream_t st) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_ugrp_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_ugrp_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace na2d
