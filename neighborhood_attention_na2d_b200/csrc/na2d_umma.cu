// na2d_umma.cu -- NA2D forward on the 5th-generation tensor cores (tcgen05)
// for maps whose dilation groups are all exactly 7 x 7: H = W = 7d, k = 7,
// D = 32, f16 / bf16.
//
// What it computes is the same as na2d_tc.cu ("Dilated Neighborhood Attention
// Transformer", gitcode DiNAT article, section "DiNAT 的核心思想":
// natten2dqkrpb -> softmax -> natten2dav, fused, NATTEN clamp rule).  When a
// dilation group is exactly k = 7 long on both axes, every query of the group
// has the whole group as its window (clamped start 0), so a group is a dense
// 49 x 49 attention with a relative-position bias.
//
// Work unit: two groups, A and B, as one M = 128 tile.  Each group's Q, K
// and V arrive by TMA as a 7 x 8 box of pixels (the group's 7 x 7 and a
// zero-filled column), 64 bytes per pixel, 64-byte swizzled: slot
// s = 8 * row + col is tile row s (A) or 64 + s (B); slot row 7 is a spare
// that holds zeros.
//   1. S = Q K^T: two tcgen05.mma (K = 16 each, A and B K-major in shared
//      memory), S = [128 x 128] fp32 in tensor memory (TMEM).  Only the
//      diagonal 64 x 64 blocks (a query and a key of the same group) are used.
//   2. softmax: one thread per tile row (its TMEM lane) loads its 56 scores,
//      adds the bias (pre-multiplied by sqrt(D), kept in registers per head),
//      exponentiates in fp32 and writes P as 16-bit pairs into its
//      warpgroup's P columns: 32 columns for its group's 64 keys; the other
//      group's 32 columns hold zeros, written once before the first unit.
//   3. O = P V: eight tcgen05.mma with A = P in TMEM and B = V (MN-major in
//      shared memory), O = [128 x 32] fp32 in TMEM.
//   4. epilogue: the same thread loads its O row, divides by its row sum and
//      stores 64 bytes.
// Warps 0-3 and 4-7 are two softmax warpgroups taking alternate units, each
// with its own S columns (TMEM columns 0-127 / 128-255) and P columns
// (256-319 / 320-383); O rotates over four 32-column buffers (384-511).  A
// warpgroup runs the softmax of its unit j and then the epilogue of its unit
// j - 2, so it never waits for a P.V that was just issued, and one
// warpgroup's softmax overlaps the other's MMAs and epilogue.  Warp 8, lane 0
// issues the TMA copies into a ring of NSTG stages; warps 9 and 10, lane 0,
// issue the MMAs of the even and the odd units and signal completion with
// tcgen05.commit on mbarriers: once unit j's P is handed over, the Q K^T two
// units ahead goes first (its S columns are free, so the warpgroup's next
// scores are not queued behind this P.V), then unit j's P.V.  Before a
// warpgroup rewrites P it waits for the P.V two units back, which read it.
// Warp 9 owns the TMEM allocation.  Every wait is bounded: one that runs out counts the event,
// raises the block's abort flag, and the block winds down (its MMAs and
// copies in flight are waited for before TMEM and shared memory are
// released).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
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

constexpr int KW = 7;
constexpr int NSTG = 6;                  // shared-memory stages (units in flight)
constexpr uint32_t kBlk = 4096;          // one group's 8 x 8 block of one tensor
constexpr uint32_t kRowsBytes = 56 * 64; // the 7 x 8 slots a copy writes (slot row 7 is spare)
constexpr uint32_t kTile = 2 * kBlk;     // one tensor of a unit (128 rows of 64 bytes)
constexpr uint32_t kStage = 3 * kTile;   // Q, K, V tiles of a unit
constexpr int kTabPitch = 16;            // floats per bias-table row (13 used)
constexpr int kTabHead = 13 * kTabPitch;
constexpr int kThreads = 352;            // 8 softmax warps, producer warp, two MMA warps
constexpr int kWarpTma = 8, kWarpMma = 9;   // MMA warps 9 (even units) and 10 (odd units)

__device__ unsigned int g_umma_timeouts;

struct UmmaParams {
    CUtensorMap tq, tk, tv;   // 5-D group views, 32 x 1 x 8 x 1 x 8 boxes
    unsigned char *out;
    const void *rpb;
    int H, W, heads, d;
    int GU;                   // groups: B * heads * d * d
    int NU;                   // units: ceil(GU / 2)
    float c_log2;             // log2(e) / sqrt(D)
    float sqrt_d;
    uint32_t off_tab, off_bar;   // byte offsets from the 1024-aligned base
};

// ---------------------------------------------------------------------------
// Kernel.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) fwd_umma_kernel(const __grid_constant__ UmmaParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;   // swizzled tiles need 1024-byte alignment
    unsigned char *smem = smem_raw + (sbase - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u_begin = (int)((int64_t)p.NU * blockIdx.x / gridDim.x);
    const int u_end = (int)((int64_t)p.NU * (blockIdx.x + 1) / gridDim.x);
    grid_dep_launch();
    if (u_begin >= u_end) return;
    const int nst = u_end - u_begin;
    const int dd = p.d * p.d;

    float *tab = reinterpret_cast<float *>(smem + p.off_tab);
    const uint32_t bar_full = sbase + p.off_bar;        // [NSTG] stage landed (TMA bytes)
    const uint32_t bar_empty = bar_full + 8 * NSTG;     // [NSTG] stage consumed (commit)
    const uint32_t bar_s = bar_empty + 8 * NSTG;        // [2] S ready (commit)
    const uint32_t bar_p = bar_s + 16;                  // [2] P written (4 warps)
    const uint32_t bar_o = bar_p + 16;                  // [4] O ready (commit)
    const uint32_t bar_drain = bar_o + 32;              // [2] all MMAs of an MMA warp done (commit)
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_bar + 16 * NSTG + 80);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_bar + 16 * NSTG + 84);

    // One unit's copies into stage j % NSTG: Q, K, V of groups 2u and 2u + 1;
    // a unit without a second group loads the first one twice (finite
    // values; its outputs are not stored).
    auto issue_unit = [&](int j) {
        const uint32_t fb = bar_full + 8 * (j % NSTG);
        const uint32_t st = sbase + (uint32_t)(j % NSTG) * kStage;
        mb_expect_tx(fb, 6u * kRowsBytes);
        const int g0 = 2 * (u_begin + j);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int g = min(g0 + e, p.GU - 1);
            const int bh = g / dd, rem = g - bh * dd, gy = rem / p.d, gx = rem - gy * p.d;
            const int row = bh * KW;   // merged (plane, group row) coordinate of group row 0
            tma_load_5d(st + (uint32_t)e * kBlk, &p.tq, fb, gx, 0, gy, row);
            tma_load_5d(st + kTile + (uint32_t)e * kBlk, &p.tk, fb, gx, 0, gy, row);
            tma_load_5d(st + 2 * kTile + (uint32_t)e * kBlk, &p.tv, fb, gx, 0, gy, row);
        }
    };
    // Units whose copies start in the prologue: two.  With every stage
    // requested at once by every block, the first unit's bytes and the bias
    // table's reads queue behind all of them (measured: 18.5 us per launch at
    // B = 32, DiNAT stage 1, against 16.7 us with two and 17.3 us with none).
    const int n_first = min(2, nst);

    // ---- prologue.  The producer thread initialises the barriers and starts
    // the first units' copies; meanwhile the other threads zero
    // the spare slot row 7 of every block, which the 7-row copies never write
    // (V's must be finite: P is 0 there, and 0 * NaN would not be), build the
    // bias table and allocate TMEM.
    {
        if (warp == kWarpTma && lane == 0) {
            for (int i = 0; i < NSTG; ++i) {
                mb_init(bar_full + 8 * i, 1);
                mb_init(bar_empty + 8 * i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mb_init(bar_s + 8 * i, 1);
                mb_init(bar_p + 8 * i, 4);
            }
            for (int i = 0; i < 4; ++i) mb_init(bar_o + 8 * i, 1);
            mb_init(bar_drain, 1);
            mb_init(bar_drain + 8, 1);
            *abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
            grid_dep_wait();   // before the first copy
            for (int j = 0; j < n_first; ++j) issue_unit(j);
        }
        // 6 * NSTG blocks x 512 bytes (slots 56 .. 63)
        for (int i = threadIdx.x; i < 6 * NSTG * 32; i += kThreads) {
            uint4 *z = reinterpret_cast<uint4 *>(smem + (i >> 5) * kBlk + kRowsBytes) + (i & 31);
            *z = make_uint4(0, 0, 0, 0);
        }
        grid_dep_wait();   // before the bias table's reads
        const T *rpb = reinterpret_cast<const T *>(p.rpb);
        for (int i = threadIdx.x; i < p.heads * kTabHead; i += kThreads) {
            const int h = i / kTabHead, a = (i / kTabPitch) % 13, b = i % kTabPitch;
            float v = 0.f;
            if (rpb && b < 13) v = Elem<T>::to_f(rpb[(h * 13 + a) * 13 + b]) * p.sqrt_d;
            tab[i] = v;
        }
        // the zeros (generic proxy) are ordered before the MMA reads (async
        // proxy) of the same bytes
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
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
                if (!mb_wait(bar_empty + 8 * s, (uint32_t)(((j / NSTG) - 1) & 1))) {
                    atomicAdd(&g_umma_timeouts, 1u);
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
        // Warp kWarpMma + e issues the MMAs of the units j with j % 2 = e,
        // whose S / P buffer is e and whose softmax is warpgroup e's: all
        // ordering a unit needs stays within one issuing thread, and the two
        // threads' MMAs overlap (one thread's issue, not the tensor core,
        // bounds these small products).  Order per thread: S_e, then per
        // unit j: O_j = P_j V_j, S_{j+2} = Q K^T; S_{j+2} reuses buffer e
        // after the P.V that reads P_j (tcgen05.mma of one thread execute in
        // issue order).
        const int e = warp - kWarpMma;
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16<T>(128, 0);
            constexpr uint32_t idesc_pv = idesc_f16<T>(32, 1);
            auto issue_qk = [&](int j) -> bool {
                const int s = j % NSTG;
                if (!mb_wait(bar_full + 8 * s, (uint32_t)((j / NSTG) & 1)) || *abort_flag) return false;
                tc_fence_after();
                const uint32_t st = sbase + (uint32_t)s * kStage;
                // K-major, 64-byte rows: 8-row groups 512 bytes apart; the
                // second K = 16 step starts 32 bytes into the rows
                const uint64_t da = sw64_desc(st, 16, 512), db = sw64_desc(st + kTile, 16, 512);
                const uint32_t dS = tmem + (uint32_t)(j & 1) * 128;
                umma_ss(dS, da, db, idesc_qk, 0);
                umma_ss(dS, da + 2, db + 2, idesc_qk, 1);
                umma_commit(bar_s + 8 * (j & 1));
                return true;
            };
            bool ok = e >= nst || issue_qk(e);
            for (int j = e; ok && j < nst; j += 2) {
                const int b = j & 1, s = j % NSTG;
                if (!mb_wait(bar_p + 8 * b, (uint32_t)((j >> 1) & 1)) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the next unit's scores first (its S buffer was read before
                // P_j was handed over), then P_j V_j
                if (j + 2 < nst && !issue_qk(j + 2)) {
                    ok = false;
                    break;
                }
                const uint32_t vt = sbase + (uint32_t)s * kStage + 2 * kTile;
                const uint32_t dO = tmem + 384u + (uint32_t)(j & 3) * 32;
                const uint32_t aP = tmem + 256u + (uint32_t)b * 64;
                // V MN-major: 64-byte rows of 32 channels, 8-key groups 512
                // bytes apart; k-step t takes keys 16t .. 16t + 15
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    umma_ts(dO, aP + 8u * t, sw64_desc(vt + 1024u * t, 16, 512), idesc_pv, t > 0 ? 1u : 0u);
                umma_commit(bar_o + 8 * (j & 3));
                umma_commit(bar_empty + 8 * s);
            }
            if (!ok) {
                atomicAdd(&g_umma_timeouts, 1u);
                *abort_flag = 1;
            }
            // every MMA this thread issued has completed before TMEM is released
            umma_commit(bar_drain + 8 * e);
            mb_wait(bar_drain + 8 * e, 0);
        }
    } else {
        // =================== softmax warpgroups ===================
        // Warpgroup w takes units j = w, w + 2, ...: softmax of unit j, then
        // the epilogue of its previous unit j - 2 (whose P.V has had the
        // softmax's time to complete); O buffers rotate over 4 (j & 3).
        const int w = warp >> 2;                      // warpgroup = S / P buffer
        const int q4 = warp & 3;                      // lane quarter of this warp
        const int m = q4 * 32 + lane;                 // tile row = TMEM lane
        const int e = m >> 6;                         // group A (0) or B (1); uniform per warp
        const int slot = m & 63, qy = slot >> 3, qx = slot & 7;
        const bool qok = qy < KW && qx < KW;
        const int qyc = min(qy, KW - 1), qxc = min(qx, KW - 1);
        const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
        const uint32_t tS = tl + (uint32_t)w * 128 + (uint32_t)e * 64;
        const uint32_t tP = tl + 256u + (uint32_t)w * 64;   // P of this warpgroup's units
        const float c = p.c_log2;
        const bool st32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
        float bias[KW * KW];
        int cur_h = -1;
        float l_prev = 1.f;
        // O of unit jj (ready once its P.V completed) / row sum -> 64 bytes
        // Position of this thread's group in unit j (g = 2 (u_begin + j) + e):
        // plane bh, head h, group row gy and column gx.  A warpgroup's units are
        // two apart, four groups, so the position advances by carries instead
        // of divisions (prev: the position two units back, whose output is
        // written after this unit's softmax).
        struct GPos {
            int g, bh, h, gy, gx;
        };
        GPos pos;
        pos.g = 2 * (u_begin + w) + e;
        pos.bh = pos.g / dd;
        pos.h = pos.bh % p.heads;
        pos.gy = (pos.g - pos.bh * dd) / p.d;
        pos.gx = pos.g - pos.bh * dd - pos.gy * p.d;
        GPos prev = pos;
        auto advance = [&](GPos &x) {
            x.g += 4;
            x.gx += 4;
            while (x.gx >= p.d) {
                x.gx -= p.d;
                if (++x.gy == p.d) {
                    x.gy = 0;
                    ++x.bh;
                    if (++x.h == p.heads) x.h = 0;
                }
            }
        };
        auto epilogue_store = [&](int jj) -> bool {
            const bool ok = mb_wait(bar_o + 8 * (jj & 3), (uint32_t)((jj >> 2) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    atomicAdd(&g_umma_timeouts, 1u);
                    *abort_flag = 1;
                }
                return false;
            }
            tc_fence_after();
            float o[32];
            tmem_ld32(tl + 384u + (uint32_t)(jj & 3) * 32, o);
            tmem_ld_wait();
            if (prev.g < p.GU && qok) {   // prev: unit jj's position
                float inv;
                asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(inv) : "f"(l_prev));
                store_pixel64<T>(
                    p.out + ((((size_t)prev.bh * p.H + prev.gy + (size_t)p.d * qy) * p.W) + prev.gx + (size_t)p.d * qx) * 64,
                    o, inv, st32);
            }
            return true;
        };
        {   // the other group's P columns of this thread's lane: zeros, once
            uint32_t zero[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) zero[i] = 0u;
            tmem_st16(tP + (uint32_t)(e ^ 1) * 32, zero);
            tmem_st16(tP + (uint32_t)(e ^ 1) * 32 + 16, zero);
            tmem_st_wait();
        }
        for (int j = w;; j += 2, prev = pos, advance(pos)) {
            if (j < nst) {
                // (a group past the last one, of an odd count, takes the head
                // that follows; its outputs are not stored)
                const int h = pos.h;
                if (h != cur_h) {
                    cur_h = h;
                    // bias of key (ky, kx): table row ky - qy + 6, column kx - qx + 6
                    const float *tb = tab + h * kTabHead + (6 - qyc) * kTabPitch + (6 - qxc);
#pragma unroll
                    for (int ky = 0; ky < KW; ++ky)
#pragma unroll
                        for (int kx = 0; kx < KW; ++kx) bias[ky * KW + kx] = tb[ky * kTabPitch + kx];
                }
                const bool ok = mb_wait(bar_s + 8 * w, (uint32_t)((j >> 1) & 1));
                if (!__all_sync(0xffffffffu, ok) || __any_sync(0xffffffffu, *abort_flag != 0)) {
                    if (lane == 0) {
                        atomicAdd(&g_umma_timeouts, 1u);
                        *abort_flag = 1;
                    }
                    break;
                }
                tc_fence_after();
                // scores of keys 8 * ky + kx, ky, kx < 8 (kx = 7 and ky = 7 are pads)
                float s[56];
                tmem_ld32(tS, s);
                tmem_ld16(tS + 32, s + 32);
                tmem_ld8(tS + 48, s + 48);
                tmem_ld_wait();
                float mx = -3.0e38f;
#pragma unroll
                for (int ky = 0; ky < KW; ++ky) {
                    // bias of columns 0-5 as three packed adds, column 6 alone
                    float *r = s + ky * 8;
                    const float *b = bias + ky * KW;
                    add2(r[0], r[1], r[0], r[1], b[0], b[1]);
                    add2(r[2], r[3], r[2], r[3], b[2], b[3]);
                    add2(r[4], r[5], r[4], r[5], b[4], b[5]);
                    r[6] += b[6];
                    mx = max3(mx, max3(r[0], r[1], r[2]), max3(r[3], r[4], fmaxf(r[5], r[6])));
                }
                const float nm = -mx * c;
                float l0 = 0.f, l1 = 0.f;   // two lanes of the row sum
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 28; ++i) {
                    float p0, p1;
                    if (((2 * i + 1) & 7) < KW) {
                        float x0, x1;
                        fma2(x0, x1, s[2 * i], s[2 * i + 1], c, nm, nm);
                        p0 = ex2(x0);
                        p1 = ex2(x1);
                    } else {   // column 7 is a pad
                        p0 = ex2(fmaf(s[2 * i], c, nm));
                        p1 = 0.f;
                    }
                    add2(l0, l1, l0, l1, p0, p1);
                    pk[i] = Pack2<T>::run(p0, p1);
                }
#pragma unroll
                for (int i = 28; i < 32; ++i) pk[i] = 0u;
                // P of unit j - 2 has been read by its P.V before it is
                // overwritten (that P.V completed long ago; bounded wait)
                if (j >= 2) {
                    const bool okp = mb_wait(bar_o + 8 * ((j - 2) & 3), (uint32_t)(((j - 2) >> 2) & 1));
                    if (!__all_sync(0xffffffffu, okp)) {
                        if (lane == 0) {
                            atomicAdd(&g_umma_timeouts, 1u);
                            *abort_flag = 1;
                        }
                        break;
                    }
                    tc_fence_after();
                }
                // own group's keys: P columns 32e .. 32e + 31 (the other
                // group's columns hold the zeros written before the loop)
                tmem_st16(tP + (uint32_t)e * 32, pk);
                tmem_st16(tP + (uint32_t)e * 32 + 16, pk + 16);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mb_arrive(bar_p + 8 * w);
                if (j < 2) {
                    l_prev = l0 + l1;
                    continue;
                }
                // ---- epilogue of unit j - 2 below, then keep this unit's sum
                const float l_this = l0 + l1;
                if (!epilogue_store(j - 2)) break;
                l_prev = l_this;
            } else {
                if (j >= 2 && j - 2 < nst) epilogue_store(j - 2);
                break;
            }
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
struct UmmaCache {
    std::mutex mu;
    std::map<int, std::pair<int, int>> dev;   // device -> (SMs, opt-in smem per block)
    std::set<std::pair<int, const void *>> attr;
};
UmmaCache &ucache() {
    static UmmaCache c;
    return c;
}

cudaError_t umma_device(int *sms, int *smem_cap, const void *kern) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    UmmaCache &c = ucache();
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

uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <typename T>
cudaError_t launch_umma_t(const Problem &pr, const void *q, const void *k, const void *v, const void *rpb, void *out,
                          cudaStream_t st, bool *launched) {
    const void *kern = reinterpret_cast<const void *>(&fwd_umma_kernel<T>);
    int sms = 0, cap = 0;
    cudaError_t e = umma_device(&sms, &cap, kern);
    if (e != cudaSuccess) return e;
    UmmaParams up{};
    const int64_t bh = pr.bh();
    const int64_t gu = bh * pr.d * pr.d;
    if (gu <= 0 || gu >= INT32_MAX || bh * KW >= INT32_MAX) return cudaSuccess;
    if (!encode_group_map(&up.tq, q, pr.dtype, bh, pr.H, pr.W, pr.d, 8, 7, 1) ||
        !encode_group_map(&up.tk, k, pr.dtype, bh, pr.H, pr.W, pr.d, 8, 7, 1) ||
        !encode_group_map(&up.tv, v, pr.dtype, bh, pr.H, pr.W, pr.d, 8, 7, 1))
        return cudaSuccess;
    up.out = static_cast<unsigned char *>(out);
    up.rpb = rpb;
    up.H = pr.H; up.W = pr.W; up.heads = pr.heads; up.d = pr.d;
    up.GU = (int)gu;
    up.NU = (int)((gu + 1) / 2);
    up.c_log2 = kLog2e / std::sqrt((float)pr.D);
    up.sqrt_d = std::sqrt((float)pr.D);
    up.off_tab = NSTG * kStage;
    up.off_bar = align_up(up.off_tab + (uint32_t)(pr.heads * kTabHead * 4), 16);
    // + 1024 bytes for aligning the base; at least 116 KB so that two blocks
    // never share an SM (each takes all 512 TMEM columns)
    const uint32_t smem = std::max<uint32_t>(up.off_bar + 16 * NSTG + 88 + 1024, 116u * 1024u);
    if ((int)smem > cap) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min(up.NU, sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t el = cudaLaunchKernelEx(&cfg, fwd_umma_kernel<T>, up);
    *launched = true;
    note_kernel("fwd_umma_kernel");
    return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace

bool umma_supported(const Problem &p) {
    if (p.dtype != DType::F16 && p.dtype != DType::BF16) return false;
    return p.k == KW && p.D == 32 && p.heads <= 64 && p.H == KW * p.d && p.W == KW * p.d;
}

cudaError_t launch_forward_umma(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                void *out, cudaStream_t st, bool *launched) {
    *launched = false;
    if (!umma_supported(p)) return cudaSuccess;
    if (p.dtype == DType::F16) return launch_umma_t<__half>(p, q, k, v, rpb, out, st, launched);
    return launch_umma_t<__nv_bfloat16>(p, q, k, v, rpb, out, st, launched);
}

cudaError_t read_umma_faults(unsigned int *count, cudaStream_t st) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_umma_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_umma_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace na2d
