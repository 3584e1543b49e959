// na2d_stream.cu -- streaming fused NA2D forward for k = 7 on the tensor cores
// (f16 / bf16, D = 32).
//
// What it computes is the same as na2d_tc.cu ("Dilated Neighborhood Attention
// Transformer", gitcode DiNAT article, section "DiNAT 的核心思想":
// natten2dqkrpb -> softmax -> natten2dav, fused, NATTEN clamp rule); this file
// only changes how the work is scheduled and staged.
//
// Two schedules:
//  * SLIDE (d = 1, 14 <= W <= 64, H >= 8): the map is walked in "steps" of up
//    to SP query-row pairs of one image.  A query-row pair needs 8 consecutive
//    key rows (the union of its two clamped windows), and consecutive pairs
//    share 6 of them, so every K / V row is brought into a shared-memory ring
//    once per CTA and reused by up to four pairs.  A CTA owns a contiguous
//    range of pairs in (batch*head, pair) order: c CTAs per image when the
//    images fit on the SMs (no range then crosses an image), else an even
//    split over one CTA per SM.
//  * DENSE (H = W = 7d, every dilation group exactly 7 x 7): a group is a
//    dense 49 x 49 attention.  A step is NWC / 4 consecutive groups, staged
//    whole.  These maps normally run on the tcgen05 kernel (na2d_umma.cu);
//    this schedule is its fallback.
//
// Loading, by a producer warp NS - 1 steps ahead through full / empty
// mbarriers: SLIDE issues one bulk copy (cp.async.bulk) per new image row of
// K, V and Q from one thread, with the byte count on the stage's full
// barrier; DENSE issues 16-byte cp.async with fixed per-lane offsets, each
// lane arriving once its copies have landed.  In the ramp-up each of the
// first NS steps is requested once the previous step's rows have landed, so
// that the first step's rows do not queue behind the next ones.  All waits
// are bounded.  The kernel is launched with programmatic stream
// serialisation and reads no global memory before the previous kernel on
// the stream has completed.
//
// Per warp, one 16-query tile per step: 2 query rows x 8 query columns.  Its
// keys form n-tiles of 4 key rows x 2 key columns (14 n-tiles = 8 x 14 keys for
// SLIDE, 8 n-tiles = 8 x 8 padded keys for DENSE), so the C-fragment pair a
// thread holds is two horizontally adjacent keys.  The relative-position bias
// (pre-multiplied by sqrt(D), masked keys at -1e30) is the C input of the first
// QK^T MMA, so adding it costs no instruction.  Each lane's bias values are
// kept in tensor memory (TMEM, one lane quarter and 64 columns per warp),
// rewritten only when the head or the tile's window geometry changes and read
// back with tcgen05.ld per chunk of key columns; keeping them there instead of
// in 56 registers leaves room for 16 warps per SM.  The softmax runs over two
// chunks of key columns with a running max, exponentiates in fp32 and packs P
// straight into the A fragments of P.V; row sums come from an MMA against ones.
//
// Shared-memory layouts (64 bytes per pixel, four 16-byte chunks):
//  * SLIDE rows (Q, K, V): row r of a buffer starts at r * (W + 1) * 64 +
//    16 * (r & 3); any 4 consecutive rows x 2 adjacent pixels of one chunk
//    index fall in 8 distinct bank groups.
//  * DENSE group blocks (8 x 8 pixels): K / V chunk c of row t stored at
//    c ^ (t & 3); Q chunk c of slot s at c ^ ((s >> 1) & 3).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <set>

#include "na2d_device.cuh"
#include "na2d_launch.h"

namespace na2d {
namespace {

constexpr int KW = 7;                 // kernel size handled here
constexpr int NS = 3;                 // pipeline stages (steps in flight)
constexpr int kPixB = 64;             // bytes per pixel (D = 32, 16-bit)
constexpr float kMaskC = -1.0e30f;    // C-init of a masked score
constexpr int kTabPitch = 16;         // floats per bias-table row (13 used)
constexpr int kTabHead = 13 * kTabPitch;
constexpr int kDenseBlk = 64 * kPixB; // one 8 x 8 (7 x 7 + pad) group block of one tensor

// Counts bounded waits of this file's kernels that ran out.
__device__ unsigned int g_stream_timeouts;

struct StreamParams {
    const unsigned char *q, *k, *v;
    unsigned char *out;
    const void *rpb;
    int H, W, heads, d;
    int nsteps;      // DENSE: steps; SLIDE: query-row pairs (split over the CTAs)
    // SLIDE schedule
    int MX, SP, NP, SPI, NR;
    // DENSE schedule
    int GU;
    float c_log2;    // log2(e) / sqrt(D)
    float sqrt_d;    // sqrt(D)
    uint32_t off_k, off_v, off_tab, off_bar;   // byte offsets in dynamic shared memory (Q at 0)
};

// ---- mbarrier helpers ------------------------------------------------------
__device__ __forceinline__ void sb_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// One try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about 20 microseconds pass, instead of spinning.
__device__ __forceinline__ bool sb_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity: gives up after about 2^31
// SM clocks (about a second) and returns false.
__device__ __forceinline__ bool sb_wait(uint32_t bar, uint32_t parity) {
    if (sb_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!sb_try(bar, parity))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}
__device__ __forceinline__ void sb_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Arrives on the barrier once all of this thread's earlier cp.async copies
// have landed (the arrival is counted in the barrier's initial count).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}

// ---- programmatic dependent launch ------------------------------------------
// The kernels are launched with programmatic stream serialisation: a grid
// may be scheduled while the previous kernel on the stream finishes, runs its
// prologue (barriers, tensor-memory allocation), and reads no global memory
// before grid_dep_wait() returns, i.e. before that kernel has completed and
// its writes are visible.  grid_dep_launch() lets the next grid be scheduled.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- tensor memory (TMEM) helpers -------------------------------------------
constexpr int kTmemCols = 256;   // 4 column slots of 64, one per warp of a lane quarter

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem),
                 "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "n"(kTmemCols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
// 8 consecutive columns of this thread's lane
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
// 4 consecutive columns (one n-tile's C-init) of this thread's lane; complete
// after tmem_ld_wait()
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                 : "r"(taddr)
                 : "memory");
}

// ---- swizzled offsets --------------------------------------------------------
// K / V: pixel slot s of row `row` (pitch in slots); chunk keyed on row & 3.
__device__ __forceinline__ uint32_t kv_off(int row, int pitch, int slot, int ch) {
    return (uint32_t)((row * pitch + slot) * kPixB + ((ch ^ (row & 3)) << 4));
}
// Q: linear slot index; chunk keyed on (slot >> 1) & 3.
__device__ __forceinline__ uint32_t q_off(int slot, int ch) {
    return (uint32_t)(slot * kPixB + ((ch ^ ((slot >> 1) & 3)) << 4));
}

template <typename T> struct OnesBits;
template <> struct OnesBits<__half> { static constexpr uint32_t v = 0x3C003C00u; };
template <> struct OnesBits<__nv_bfloat16> { static constexpr uint32_t v = 0x3F803F80u; };

// exp2 of two fp32 arguments (fp32 ex2.approx, one MUFU op each), rounded
// and packed in the operand type T (low half = first argument).  A packed
// f16x2 / bf16x2 ex2 costs the same two MUFU ops plus repacking on sm_100.
template <typename T> struct Exp2Pair;
template <> struct Exp2Pair<__half> {
    __device__ __forceinline__ static uint32_t run(float lo, float hi) {
        const float a = ex2(lo), b = ex2(hi);
        uint32_t e;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(e) : "f"(b), "f"(a));
        return e;
    }
};
template <> struct Exp2Pair<__nv_bfloat16> {
    __device__ __forceinline__ static uint32_t run(float lo, float hi) {
        const float a = ex2(lo), b = ex2(hi);
        uint32_t e;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(e) : "f"(b), "f"(a));
        return e;
    }
};

// D = A * B + C with separate C (the C-init carries the bias).
template <typename T> struct MmaC;
template <> struct MmaC<__half> {
    __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4]) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};\n"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
              "f"(c[3]));
    }
};
template <> struct MmaC<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4]) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};\n"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
              "f"(c[3]));
    }
};

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// SLIDE geometry of query row y (or column): window start and halo start.
__device__ __forceinline__ int win_start(int y, int L) { return clampi(y - KW / 2, 0, L - KW); }

// Halo start of query-row pair p: the first of 8 consecutive key rows that
// hold both rows' clamped windows.
__device__ __forceinline__ int pair_halo(int pair, int H) { return min(win_start(2 * pair, H), H - 8); }

// SLIDE walk: the CTA's steps in order, with the K / V ring bookkeeping.
// A CTA owns a contiguous range of query-row pairs in (image, pair) order
// (global pair index bh * NP + pair), which may start and end inside an
// image; a step is up to SP consecutive pairs of one image.  Rows of one
// image are loaded in increasing order, each once, into consecutive ring
// rows; the next image continues after the last ring row of the previous
// one.  Producer and consumers run the same walk.  Only the image, the step's
// pairs and the ring row of the step's first key row are kept; the rest is
// recomputed from them.
struct SlideWalk {
    int bh;           // image
    int pa, pe;       // the step's first pair and one past its last
    int ge;           // end of the CTA's range (global pair index)
    int h;            // head of image bh
    int ring_lo;      // ring row of lo()
    __device__ __forceinline__ int p0(const StreamParams &) const { return pa; }
    __device__ __forceinline__ int plast(const StreamParams &) const { return pe - 1; }
    __device__ __forceinline__ int lo(const StreamParams &p) const { return pair_halo(pa, p.H); }
    __device__ __forceinline__ int hi(const StreamParams &p) const { return pair_halo(pe - 1, p.H) + 7; }
    __device__ __forceinline__ int step_end(const StreamParams &p) const {
        return min(pa + p.SP, min(p.NP, ge - bh * p.NP));
    }
    __device__ __forceinline__ void init(const StreamParams &p, int gb, int gend) {
        ge = gend;
        bh = gb / p.NP;
        pa = gb - bh * p.NP;
        pe = step_end(p);
        h = bh % p.heads;
        ring_lo = 0;
    }
    __device__ __forceinline__ static int wrap(int x, int NR) { return x >= NR ? x - NR : x; }
    __device__ __forceinline__ int ring(const StreamParams &p, int row) const {
        return wrap(ring_lo + row - lo(p), p.NR);
    }
    // Advances to the next step; returns the first row that step must load.
    __device__ __forceinline__ int next(const StreamParams &p) {
        const int old_lo = lo(p), old_hi = hi(p);
        const int hi_ring = wrap(ring_lo + old_hi - old_lo, p.NR);
        if (pe == p.NP) {
            ++bh;
            if (++h == p.heads) h = 0;
            pa = 0;
            pe = step_end(p);
            ring_lo = wrap(hi_ring + 1, p.NR);
            return lo(p);
        }
        pa = pe;
        pe = step_end(p);
        ring_lo = wrap(ring_lo + (lo(p) - old_lo), p.NR);
        return old_hi + 1;
    }
};

// Number of SLIDE steps in the pair range [gb, ge): per image, ceil(pairs / SP).
__device__ __forceinline__ int slide_steps(const StreamParams &p, int gb, int ge) {
    int n = 0;
    while (gb < ge) {
        const int bh = gb / p.NP, pa = gb - bh * p.NP, pe = min(p.NP, ge - bh * p.NP);
        n += (pe - pa + p.SP - 1) / p.SP;
        gb = bh * p.NP + pe;
    }
    return n;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void sb_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// Skewed row layout of the SLIDE buffers: row r of a buffer starts at
// r * pitch + 16 * (r & 3) bytes (pitch = (W + 1) * 64); pixels and their four
// 16-byte chunks are stored in order, so a whole image row lands with one bulk
// copy.  Any 4 consecutive rows x 2 adjacent pixels of one chunk index fall in
// 8 distinct bank groups.
__device__ __forceinline__ uint32_t row_base(int r, uint32_t pitch) { return (uint32_t)r * pitch + 16u * (r & 3); }

// ---------------------------------------------------------------------------
// The 16-query tile: QK^T (C-init = bias), softmax, P.V, store.
//   n-tiles are (R, J), R in {0, 1} (key rows 4R .. 4R+3), J < NJ (key
//   columns 2J, 2J+1); a P.V k-step takes the pair (0, J) + (1, J).
//   The key columns are processed in chunks [J0, J1) with an online softmax
//   (running max, rescaled sums), which bounds the live score registers.
//   tb: this warp's TMEM bias address for this lane; n-tile (R, J) holds its
//       four C-init values in columns (2J + R) * 4 .. + 3.
//   qa0, qa1: this lane's ldmatrix addresses of the Q fragments (k-steps 0, 1).
//   kb0, kb1: this lane's K address of n-tile (R, 0); n-tile (R, J) is + J*128.
//   dv: V address minus K address (same layout).
//   The stores go to out0 (row r) and out1 (row r + 8), or nowhere if null.
// ---------------------------------------------------------------------------
struct TileAcc {
    float o[4][4];   // O fragments, channel n-tiles 0..3
    float l[4];      // row sums (ones-MMA), all columns equal
    float m0, m1;    // running row max of rows r and r + 8 (raw accumulator units)
};

template <typename T, int J0, int J1, bool SKEW, bool FIRST>
__device__ __forceinline__ void tile_chunk(TileAcc &acc, const uint32_t (&qf)[2][4], uint32_t kb0, uint32_t kb1,
                                           uint32_t vsel, uint32_t tb, float c_log2) {
    constexpr int NC = J1 - J0;
    // ---- bias C-init of the chunk's n-tiles from TMEM
    float bias[2][NC][4];
#pragma unroll
    for (int j = 0; j < NC; ++j)
#pragma unroll
        for (int R = 0; R < 2; ++R) tmem_ld4(tb + (uint32_t)((2 * (J0 + j) + R) * 4), bias[R][j]);
    tmem_ld_wait();
    // ---- S = Q K^T + bias*sqrt(D) over the chunk's 2 * NC n-tiles
    float s[2][NC][4];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
#pragma unroll
        for (int R = 0; R < 2; ++R) {
            uint32_t kf[4];
            ldsm_x4(kf, (R ? kb1 : kb0) + (J0 + j) * 128);
            MmaC<T>::run(s[R][j], qf[0], kf[0], kf[1], bias[R][j]);
            Mma<T>::run(s[R][j], qf[1], kf[2], kf[3]);
        }
    }
    // ---- row max of the chunk, quad reduction, merge with the running max
    float c0 = s[0][0][0], c1 = s[0][0][2];
#pragma unroll
    for (int R = 0; R < 2; ++R)
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            c0 = max3(c0, s[R][j][0], s[R][j][1]);
            c1 = max3(c1, s[R][j][2], s[R][j][3]);
        }
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 1));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 1));
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 2));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 2));
    if constexpr (FIRST) {
        acc.m0 = c0;
        acc.m1 = c1;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc.l[i] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) acc.o[i][j] = 0.f;
        }
    } else {
        const float n0 = fmaxf(acc.m0, c0), n1 = fmaxf(acc.m1, c1);
        const float a0 = ex2((acc.m0 - n0) * c_log2), a1 = ex2((acc.m1 - n1) * c_log2);
        acc.m0 = n0;
        acc.m1 = n1;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc.o[i][0] *= a0; acc.o[i][1] *= a0;
            acc.o[i][2] *= a1; acc.o[i][3] *= a1;
        }
        acc.l[0] *= a0; acc.l[1] *= a0;
        acc.l[2] *= a1; acc.l[3] *= a1;
    }
    const float n0 = -acc.m0 * c_log2, n1 = -acc.m1 * c_log2;
    // ---- P = exp2((S - max) * log2(e) / sqrt(D)) straight into the A
    // fragments of the k-step (0, J) + (1, J); O += P V, l += P 1
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        uint32_t a[4];
        a[0] = Exp2Pair<T>::run(fmaf(s[0][j][0], c_log2, n0), fmaf(s[0][j][1], c_log2, n0));
        a[1] = Exp2Pair<T>::run(fmaf(s[0][j][2], c_log2, n1), fmaf(s[0][j][3], c_log2, n1));
        a[2] = Exp2Pair<T>::run(fmaf(s[1][j][0], c_log2, n0), fmaf(s[1][j][1], c_log2, n0));
        a[3] = Exp2Pair<T>::run(fmaf(s[1][j][2], c_log2, n1), fmaf(s[1][j][3], c_log2, n1));
        uint32_t v01[4], v23[4];
        // channel chunks 0/1, then 2/3: +32 bytes in the skewed layout; with the
        // XOR-swizzled layout (chunk c stored at c ^ (row & 3)) chunk bit 1 flips
        const uint32_t vaddr = vsel + (J0 + j) * 128;
        ldsm_x4_t(v01, vaddr);
        ldsm_x4_t(v23, SKEW ? vaddr + 32u : (vaddr ^ 32u));
        Mma<T>::run(acc.o[0], a, v01[0], v01[1]);
        Mma<T>::run(acc.o[1], a, v01[2], v01[3]);
        Mma<T>::run(acc.o[2], a, v23[0], v23[1]);
        Mma<T>::run(acc.o[3], a, v23[2], v23[3]);
        Mma<T>::run(acc.l, a, OnesBits<T>::v, OnesBits<T>::v);
    }
}

template <typename T, int NJ, bool SKEW>
__device__ __forceinline__ void tile_compute(uint32_t qa0, uint32_t qa1, uint32_t kb0, uint32_t kb1, uint32_t dv,
                                             uint32_t tb, float c_log2, int lane, unsigned char *out0,
                                             unsigned char *out1) {
    uint32_t qf[2][4];
    ldsm_x4(qf[0], qa0);
    ldsm_x4(qf[1], qa1);
    // V x4.trans lanes: 0-7 / 16-23 address key rows 0-3 (n-tile (0, J)), 8-15 /
    // 24-31 key rows 4-7 (n-tile (1, J)); lanes 16-31 take channel chunk + 1
    const uint32_t vsel = (((lane >> 3) & 1) ? kb1 : kb0) + dv;
    TileAcc acc;
    if constexpr (NJ == 7) {
        tile_chunk<T, 0, 4, SKEW, true>(acc, qf, kb0, kb1, vsel, tb, c_log2);
        tile_chunk<T, 4, 7, SKEW, false>(acc, qf, kb0, kb1, vsel, tb, c_log2);
    } else {
        tile_chunk<T, 0, NJ, SKEW, true>(acc, qf, kb0, kb1, vsel, tb, c_log2);
    }
    // ---- normalise and store: row r holds channels 8*cn + 2*(lane&3) (+1)
    float i0, i1;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(i0) : "f"(acc.l[0]));
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(i1) : "f"(acc.l[2]));
    const int cofs = 4 * (lane & 3);
    if (out0) {
#pragma unroll
        for (int cn = 0; cn < 4; ++cn)
            *reinterpret_cast<uint32_t *>(out0 + 16 * cn + cofs) =
                Elem<T>::pack2(acc.o[cn][0] * i0, acc.o[cn][1] * i0);
    }
    if (out1) {
#pragma unroll
        for (int cn = 0; cn < 4; ++cn)
            *reinterpret_cast<uint32_t *>(out1 + 16 * cn + cofs) =
                Elem<T>::pack2(acc.o[cn][2] * i1, acc.o[cn][3] * i1);
    }
}

// Writes one lane's bias C-init values (n-tile (R, J) at columns
// (2J + R) * 4 ..) into TMEM, 8 columns at a time.
template <int NJ>
__device__ __forceinline__ void tmem_store_bias(uint32_t tb, const float (&bias)[2][NJ][4]) {
#pragma unroll
    for (int J = 0; J < NJ; ++J) {
        const float v[8] = {bias[0][J][0], bias[0][J][1], bias[0][J][2], bias[0][J][3],
                            bias[1][J][0], bias[1][J][1], bias[1][J][2], bias[1][J][3]};
        tmem_st8(tb + (uint32_t)(8 * J), v);
    }
    tmem_st_wait();
}

// ---------------------------------------------------------------------------
// Kernel.
// ---------------------------------------------------------------------------
// Warps 0 .. NWC-1 consume; warp NWC produces (SLIDE: one thread issues one
// bulk copy per image row; DENSE: the warp issues 16-byte cp.async).  Each
// consumer warp owns a fixed tile position of every step (SLIDE: pair
// warp / MX of the step, column tile warp % MX; DENSE: group warp / 4 of the
// step, query-row pair warp % 4), so per-warp geometry is set up once.
template <typename T, bool DENSE, int NWC>
__global__ void __launch_bounds__((NWC + 1) * 32, 1) fwd_stream_kernel(const __grid_constant__ StreamParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's range: DENSE steps, or SLIDE query-row pairs (finer, so that
    // the CTAs' loads differ by at most one pair)
    const int s_begin = (int)((int64_t)p.nsteps * blockIdx.x / gridDim.x);
    const int s_end = (int)((int64_t)p.nsteps * (blockIdx.x + 1) / gridDim.x);
    grid_dep_launch();
    if (s_begin >= s_end) return;
    const int nst = DENSE ? s_end - s_begin : slide_steps(p, s_begin, s_end);
    constexpr int GPS = NWC / 4;   // DENSE groups per step

    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + p.off_bar, bar_empty = bar_full + 8 * NS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_bar + 16 * NS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_bar + 16 * NS + 4);
    // bias table, with 64 bytes of padding on either side for unclamped column reads
    float *tab = reinterpret_cast<float *>(smem + p.off_tab + 64);
    const uint32_t pitch = (uint32_t)(p.W + 1) * kPixB;   // SLIDE row pitch in bytes

    // ---- prologue: (DENSE) zero the staging blocks, whose pad pixels must
    // hold finite values; build the bias table; init the barriers; allocate TMEM.
    {
        if constexpr (DENSE) {
            uint4 *z = reinterpret_cast<uint4 *>(smem);
            const int n16 = (int)(p.off_tab / 16);
            for (int i = threadIdx.x; i < n16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
        }
        grid_dep_wait();   // first global read: the bias table
        const T *rpb = reinterpret_cast<const T *>(p.rpb);
        for (int i = threadIdx.x; i < p.heads * kTabHead; i += blockDim.x) {
            const int h = i / kTabHead, a = (i / kTabPitch) % 13, b = i % kTabPitch;
            float v = 0.f;
            if (rpb && b < 13) v = Elem<T>::to_f(rpb[(h * 13 + a) * 13 + b]) * p.sqrt_d;
            tab[i] = v;
        }
        if (threadIdx.x == 0) {
            for (int i = 0; i < NS; ++i) {
                // SLIDE: one expect_tx arrival per step; DENSE: one cp.async
                // arrival per producer lane
                sb_init(bar_full + 8 * i, DENSE ? 32 : 1);
                sb_init(bar_empty + 8 * i, NWC);
            }
            *abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        }
        if (warp == 0) tmem_alloc(smem_u32(tmem_slot));
        tmem_fence_before();
        __syncthreads();
        tmem_fence_after();
    }

    if (warp == NWC) {
        // =================== producer ===================
        if constexpr (!DENSE) {
            // one thread issues one bulk copy per image row: the step's new
            // K and V rows into the ring, its query rows into the stage
            if (lane == 0) {
                const uint32_t rowbytes = (uint32_t)p.W * kPixB;
                SlideWalk w;
                w.init(p, s_begin, s_end);
                int issued = 0;
                for (int i = 0; i < nst; ++i) {
                    const int stage = i % NS;
                    const int first = i ? w.next(p) : w.lo(p);
                    // ramp-up: each of the first NS steps is requested once
                    // the previous step's rows have landed, so that the first
                    // step's rows do not queue behind the next steps'; later,
                    // a step waits for its stage to be released
                    const bool ok = i >= NS ? sb_wait(bar_empty + 8 * stage, (uint32_t)(((i / NS) - 1) & 1))
                                            : (i == 0 || sb_wait(bar_full + 8 * (i - 1), 0u));
                    if (!ok) {
                        atomicAdd(&g_stream_timeouts, 1u);
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    const int hi = w.hi(p);
                    const int y0 = 2 * w.p0(p), y1 = min(2 * (w.plast(p) + 1), p.H);
                    const uint32_t bar = bar_full + 8 * stage;
                    sb_expect_tx(bar, (uint32_t)(2 * (hi - first + 1) + (y1 - y0)) * rowbytes);
                    for (int row = first; row <= hi; ++row) {
                        const uint32_t o = row_base(w.ring(p, row), pitch);
                        const size_t src = ((size_t)w.bh * p.H + row) * rowbytes;
                        bulk_g2s(sbase + p.off_k + o, p.k + src, rowbytes, bar);
                        bulk_g2s(sbase + p.off_v + o, p.v + src, rowbytes, bar);
                    }
                    for (int y = y0; y < y1; ++y)
                        bulk_g2s(sbase + row_base(stage * 2 * p.SP + (y - y0), pitch),
                                 p.q + ((size_t)w.bh * p.H + y) * rowbytes, rowbytes, bar);
                    ++issued;
                }
                // copies still in flight must land before the CTA's shared
                // memory is released (all of them, unless a wait ran out)
                for (int j = max(0, issued - NS); j < issued; ++j)
                    sb_wait(bar_full + 8 * (j % NS), (uint32_t)((j / NS) & 1));
            }
        } else {
            // GPS = 3 group-units per step, 16-byte cp.async per lane.  Lanes
            // 0-23 work: lane l copies chunk l & 3 of group (l >> 2) % 3 for
            // pixel 2t + (l >> 2) / 3 of the 7 x 7 group (row-major), so 12
            // adjacent lanes read 3 adjacent pixels where the groups are
            // adjacent.  Offsets are fixed per lane.
            static_assert(GPS == 3, "producer lane map assumes three groups per step");
            constexpr int NT = (49 + 1) / 2;
            const bool lane_on = lane < 24;
            const int ch = lane & 3, g = (lane >> 2) % 3, half = (lane >> 2) / 3;
            int src_off[NT];
            uint32_t dst_q[NT], dst_kv[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int px = min(2 * t + half, 48);
                const int jx = px % 7, ty = px / 7;
                src_off[t] = ((p.d * ty) * p.W + p.d * jx) * kPixB + (ch << 4);
                dst_q[t] = (uint32_t)(g * kDenseBlk) + q_off(ty * 8 + jx, ch);
                dst_kv[t] = (uint32_t)(g * kDenseBlk) + kv_off(ty, 8, jx, ch);
            }
            const int dd = p.d * p.d;
            for (int i = 0; i < nst; ++i) {
                const int s = s_begin + i, stage = i % NS;
                if (i >= NS && !sb_wait(bar_empty + 8 * stage, (uint32_t)(((i / NS) - 1) & 1))) {
                    if (lane == 0) {
                        atomicAdd(&g_stream_timeouts, 1u);
                        *abort_flag = 1;
                    }
                    break;
                }
                if (*abort_flag) break;
                // this lane's group: global byte offset of its first pixel
                const int gu = GPS * s + g;
                const bool gok = lane_on && gu < p.GU;
                const int bh = gu / dd, rem = gu - bh * dd, gy = rem / p.d, gx = rem - gy * p.d;
                const size_t gbase = (((size_t)bh * p.H + gy) * p.W + gx) * kPixB;
                const uint32_t sq = sbase + (uint32_t)(stage * GPS * kDenseBlk);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (gok && 2 * t + half < 49) {
                        const size_t src = gbase + src_off[t];
                        cp_async_16(sq + dst_q[t], p.q + src);
                        cp_async_16(sq + p.off_k + dst_kv[t], p.k + src);
                        cp_async_16(sq + p.off_v + dst_kv[t], p.v + src);
                    }
                }
                cp_async_arrive(bar_full + 8 * stage);
            }
            cp_async_wait<0>();
        }
    } else {
        // =================== consumers ===================
        const int r = lane >> 2, c = lane & 3;
        const int li = (lane & 7) >> 1, lj = lane & 1;   // this lane's key (row, col) in an n-tile
        const int lch = lane >> 3;                       // this lane's channel chunk for K loads
        constexpr int NJ = DENSE ? 4 : 7;
        // this warp's TMEM bias columns: lane quarter warp % 4, column slot warp / 4
        const uint32_t tb = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(64 * (warp >> 2));
        int bias_key = -1;
        if constexpr (!DENSE) {
            const int H = p.H, W = p.W;
            // fixed per warp: column tile, halo columns, this lane's query column
            const int pw = warp / p.MX, x0 = 8 * (warp - pw * p.MX);
            const bool active = warp < p.SP * p.MX;
            const int hx = min(win_start(x0, W), W - 14);
            const int qx = min(x0 + r, W - 1), sx = win_start(qx, W);
            const bool colok = x0 + r < W;
            // this lane's key columns hx + 2J + e: bias-table column b0 + 2J + e,
            // inside the query's window for the bits set in xmask
            const int b0 = hx - qx + 6;
            uint32_t xmask = 0;
#pragma unroll
            for (int t = 0; t < 2 * NJ; ++t) xmask |= ((unsigned)(hx + t - sx) < (unsigned)KW ? 1u : 0u) << t;
            const uint32_t kcol = (uint32_t)(hx + lj) * kPixB + 16u * lch;
            const uint32_t qcol = (uint32_t)min(x0 + (lane & 7), W - 1) * kPixB + 16u * (lane >> 4);
            const uint32_t dv = (p.off_v - p.off_k) + 16u * (uint32_t)((lane >> 4) - lch);
            const int qsel = (lane >> 3) & 1;
            SlideWalk w;
            w.init(p, s_begin, s_end);
            for (int i = 0; i < nst; ++i) {
                const int stage = i % NS;
                if (i) w.next(p);
                const int pair = w.p0(p) + pw;
                const bool work = active && pair <= w.plast(p);
                const int qy0 = 2 * pair, qy1 = min(qy0 + 1, H - 1);
                const int hy = pair_halo(pair, H);
                if (work) {
                    const int sy0 = win_start(qy0, H), sy1 = win_start(qy1, H);
                    // bias: rewritten when the head or the row geometry
                    // changes, before the wait for the step's rows (it needs
                    // none of them), so that it overlaps the copies
                    const int key = ((w.h * 8 + (qy0 - hy)) * 2 + (qy1 - qy0)) * 4 + (sy0 - hy) * 2 + (sy1 - hy);
                    if (key != bias_key) {
                        bias_key = key;
                        const float *th = tab + w.h * kTabHead;
                        float bias[2][NJ][4];
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            const int qy = m ? qy1 : qy0, sy = m ? sy1 : sy0;
#pragma unroll
                            for (int R = 0; R < 2; ++R) {
                                const int ky = hy + 4 * R + c;
                                // a key row outside the window masks the whole row
                                const uint32_t rmask = (unsigned)(ky - sy) < (unsigned)KW ? xmask : 0u;
                                // table row; columns b0 - 1 .. b0 + 13 stay inside the
                                // padded table, so the loads need no clamp
                                const float *row = th + clampi(ky - qy + 6, 0, 12) * kTabPitch + b0;
#pragma unroll
                                for (int J = 0; J < NJ; ++J)
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const float b = row[2 * J + e];
                                        bias[R][J][2 * m + e] = (rmask >> (2 * J + e)) & 1u ? b : kMaskC;
                                    }
                            }
                        }
                        tmem_store_bias<NJ>(tb, bias);
                    }
                }
                if (!sb_wait(bar_full + 8 * stage, (uint32_t)((i / NS) & 1))) {
                    if (lane == 0) {
                        atomicAdd(&g_stream_timeouts, 1u);
                        *abort_flag = 1;
                    }
                    break;
                }
                if (*abort_flag) break;
                if (work) {
                    // Q fragment addresses: lanes 0-7 / 16-23 row qy0, 8-15 /
                    // 24-31 row qy1; lanes 16-31 take the odd 16-byte chunk
                    const int qr = stage * 2 * p.SP + (qsel ? qy1 : qy0) - 2 * w.p0(p);
                    const uint32_t qa0 = sbase + row_base(qr, pitch) + qcol;
                    // K addresses of n-tiles (0, 0) and (1, 0); V (x4.trans)
                    // lanes address the same keys with chunk lane >> 4
                    const uint32_t kb0 = sbase + p.off_k + row_base(w.ring(p, hy + li), pitch) + kcol;
                    const uint32_t kb1 = sbase + p.off_k + row_base(w.ring(p, hy + 4 + li), pitch) + kcol;
                    unsigned char *o0 = nullptr, *o1 = nullptr;
                    if (colok) {
                        o0 = p.out + (((size_t)w.bh * H + qy0) * W + x0 + r) * kPixB;
                        if (qy0 + 1 < H) o1 = o0 + (size_t)W * kPixB;
                    }
                    tile_compute<T, NJ, true>(qa0, qa0 + 32u, kb0, kb1, dv, tb, p.c_log2, lane, o0, o1);
                }
                __syncwarp();
                if (lane == 0) sb_arrive(bar_empty + 8 * stage);
            }
        } else {
            const int g = warp >> 2, pp = warp & 3;
            const int qx = min(r, 6);
            const int qslot = (2 * pp + ((lane >> 3) & 1)) * 8 + (lane & 7);
            const uint32_t qoff0 = q_off(qslot, (lane >> 4)), qoff1 = q_off(qslot, 2 + (lane >> 4));
            const uint32_t koff0 = kv_off(li, 8, lj, lch), koff1 = kv_off(4 + li, 8, lj, lch);
            const uint32_t dv = (p.off_v - p.off_k) + (uint32_t)((((lane >> 4) ^ li) - (lch ^ li)) * 16);
            const int qy = 2 * pp;
            const int dd = p.d * p.d;
            // this warp's group of the first step, then advanced by GPS groups per step
            int gu = GPS * s_begin + g;
            int bh = gu / dd, rem = gu - bh * dd, gy = rem / p.d, gx = rem - gy * p.d;
            int h = bh % p.heads;
            for (int i = 0; i < nst; ++i) {
                const int stage = i % NS;
                if (i) {
                    gu += GPS;
                    gx += GPS;
                    while (gx >= p.d) {
                        gx -= p.d;
                        if (++gy == p.d) {
                            gy = 0;
                            ++bh;
                            if (++h == p.heads) h = 0;
                        }
                    }
                }
                if (!sb_wait(bar_full + 8 * stage, (uint32_t)((i / NS) & 1))) {
                    if (lane == 0) {
                        atomicAdd(&g_stream_timeouts, 1u);
                        *abort_flag = 1;
                    }
                    break;
                }
                if (*abort_flag) break;
                if (gu < p.GU) {
                    if (h != bias_key) {
                        bias_key = h;
                        const float *th = tab + h * kTabHead;
                        float bias[2][NJ][4];
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            const int qyy = min(2 * pp + m, 6);
#pragma unroll
                            for (int R = 0; R < 2; ++R) {
                                const int ky = 4 * R + c;
                                const float *row = th + clampi(ky - qyy + 6, 0, 12) * kTabPitch;
#pragma unroll
                                for (int J = 0; J < NJ; ++J)
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const int kx = 2 * J + e;
                                        const float b = row[clampi(kx - qx + 6, 0, 12)];
                                        bias[R][J][2 * m + e] = (ky < KW && kx < KW) ? b : kMaskC;
                                    }
                            }
                        }
                        tmem_store_bias<NJ>(tb, bias);
                    }
                    const uint32_t blk = sbase + (uint32_t)((stage * GPS + g) * kDenseBlk);
                    unsigned char *o0 = nullptr, *o1 = nullptr;
                    if (r < 7) {
                        o0 = p.out + ((((size_t)bh * p.H + gy + (size_t)p.d * qy) * p.W) + gx + (size_t)p.d * r) * kPixB;
                        if (qy + 1 < 7) o1 = o0 + (size_t)p.d * p.W * kPixB;
                    }
                    tile_compute<T, NJ, false>(blk + qoff0, blk + qoff1, blk + p.off_k + koff0, blk + p.off_k + koff1,
                                               dv, tb, p.c_log2, lane, o0, o1);
                }
                __syncwarp();
                if (lane == 0) sb_arrive(bar_empty + 8 * stage);
            }
        }
    }
    // ---- epilogue: TMEM released by the warp that took it, after every warp
    // is done with it
    tmem_fence_before();
    __syncthreads();
    if (warp == 0) {
        tmem_fence_after();
        tmem_dealloc(*tmem_slot);
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct StreamCache {
    std::mutex mu;
    std::map<int, std::pair<int, int>> dev;     // device -> (SMs, opt-in smem per block)
    std::set<std::pair<int, const void *>> attr;
};
StreamCache &scache() {
    static StreamCache c;
    return c;
}

cudaError_t stream_device(int *sms, int *smem_cap, const void *kern) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    StreamCache &c = scache();
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

template <typename T, bool DENSE, int NWC>
cudaError_t launch_stream_t(const StreamParams &sp, uint32_t smem, int grid, cudaStream_t st, bool *launched) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((NWC + 1) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fwd_stream_kernel<T, DENSE, NWC>, sp);
    *launched = true;
    return e != cudaSuccess ? e : cudaGetLastError();
}

// SLIDE plan for SP query-row pairs per step; returns the shared-memory bytes.
uint32_t plan_slide(StreamParams &sp, const Problem &pr, int SP) {
    sp.MX = (pr.W + 7) / 8;
    sp.SP = SP;
    sp.NP = (pr.H + 1) / 2;
    sp.SPI = (sp.NP + sp.SP - 1) / sp.SP;
    // K / V rows needed by NS consecutive steps: 2*SP per step plus a 6-row
    // halo for every image those steps touch
    const int images = std::min(NS, (NS - 2) / sp.SPI + 2);
    sp.NR = (int)align_up((uint32_t)(2 * sp.SP * NS + 6 * images), 4);
    // skewed rows: pitch (W + 1) * 64 bytes (see row_base)
    const uint32_t pitch = (uint32_t)(pr.W + 1) * kPixB;
    const uint32_t qbytes = (uint32_t)(NS * 2 * sp.SP) * pitch;
    const uint32_t ring = (uint32_t)sp.NR * pitch;
    sp.off_k = align_up(qbytes, 128);
    sp.off_v = sp.off_k + align_up(ring, 128);
    sp.off_tab = sp.off_v + align_up(ring, 128);
    sp.off_bar = align_up(sp.off_tab + 128 + (uint32_t)(pr.heads * kTabHead * 4), 16);
    return sp.off_bar + 16 * NS + 16;
}

template <typename T, int NWC>
cudaError_t launch_slide(StreamParams &sp, const Problem &pr, cudaStream_t st, bool *launched) {
    const void *kern = reinterpret_cast<const void *>(&fwd_stream_kernel<T, false, NWC>);
    int sms = 0, cap = 0;
    cudaError_t e = stream_device(&sms, &cap, kern);
    if (e != cudaSuccess) return e;
    const int MX = (pr.W + 7) / 8;
    for (int SP = std::max(1, NWC / MX); SP >= 1; --SP) {
        const uint32_t smem = plan_slide(sp, pr, SP);
        if ((int)smem > cap) continue;
        const int64_t npairs = pr.bh() * sp.NP;
        if (npairs >= INT32_MAX || npairs <= 0) return cudaSuccess;
        sp.nsteps = (int)npairs;
        // CTAs: one per SM with an even split of the pairs, or, when the
        // images fit on the SMs, a whole number c of CTAs per image, so that
        // every CTA's range lies inside one image (no second halo and no
        // second clamped image top, which cost about a step).  The aligned
        // split is taken while it gives a CTA at most one pair more.
        const int64_t images = pr.bh();
        int grid = (int)std::min<int64_t>(npairs, sms);
        if (images <= sms) {
            const int64_t c = std::min<int64_t>(sms / images, sp.NP);
            const int64_t aligned = (sp.NP + c - 1) / c, even = (npairs + sms - 1) / sms;
            if (aligned <= even + 1) grid = (int)(images * c);
        }
        return launch_stream_t<T, false, NWC>(sp, smem, grid, st, launched);
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_stream_impl(const Problem &pr, const void *q, const void *k, const void *v, const void *rpb,
                               void *out, cudaStream_t st, bool *launched) {
    StreamParams sp{};
    sp.q = static_cast<const unsigned char *>(q);
    sp.k = static_cast<const unsigned char *>(k);
    sp.v = static_cast<const unsigned char *>(v);
    sp.out = static_cast<unsigned char *>(out);
    sp.rpb = rpb;
    sp.H = pr.H; sp.W = pr.W; sp.heads = pr.heads; sp.d = pr.d;
    sp.c_log2 = kLog2e / std::sqrt((float)pr.D);
    sp.sqrt_d = std::sqrt((float)pr.D);
    const int64_t bh = pr.bh();
    const bool dense = (pr.H == KW * pr.d && pr.W == KW * pr.d);
    if (dense) {
        // 12 consumer warps (three 7 x 7 groups per step, one warp per
        // query-row pair of a group) and a producer warp
        constexpr int NWC = 12, GPS = NWC / 4;
        const void *kern = reinterpret_cast<const void *>(&fwd_stream_kernel<T, true, NWC>);
        int sms = 0, cap = 0;
        cudaError_t e = stream_device(&sms, &cap, kern);
        if (e != cudaSuccess) return e;
        const int64_t gu = bh * pr.d * pr.d;
        const int64_t nsteps = (gu + GPS - 1) / GPS;
        if (gu >= INT32_MAX || nsteps <= 0) return cudaSuccess;
        sp.GU = (int)gu;
        sp.nsteps = (int)nsteps;
        const uint32_t stage_bytes = GPS * kDenseBlk;
        sp.off_k = NS * stage_bytes;
        sp.off_v = 2 * NS * stage_bytes;
        sp.off_tab = 3 * NS * stage_bytes;
        sp.off_bar = align_up(sp.off_tab + 128 + (uint32_t)(pr.heads * kTabHead * 4), 16);
        const uint32_t smem = sp.off_bar + 16 * NS + 16;
        if ((int)smem > cap) return cudaSuccess;
        return launch_stream_t<T, true, NWC>(sp, smem, std::min(sp.nsteps, sms), st, launched);
    }
    // SLIDE: 14 consumer warps (SP query-row pairs of MX column tiles each)
    // and a producer warp; 15 warps keep 128 registers per thread
    return launch_slide<T, 14>(sp, pr, st, launched);
}

}  // namespace

bool stream_supported(const Problem &p) {
    if (p.dtype != DType::F16 && p.dtype != DType::BF16) return false;
    if (p.k != KW || p.D != 32 || p.heads > 64) return false;
    if (p.H == KW * p.d && p.W == KW * p.d) return true;            // dense groups
    return p.d == 1 && p.W >= 14 && p.W <= 64 && p.H >= 8;          // sliding rows
}

cudaError_t launch_forward_stream(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                  void *out, cudaStream_t st, bool *launched) {
    *launched = false;
    if (!stream_supported(p)) return cudaSuccess;
    if (p.dtype == DType::F16) return launch_stream_impl<__half>(p, q, k, v, rpb, out, st, launched);
    return launch_stream_impl<__nv_bfloat16>(p, q, k, v, rpb, out, st, launched);
}

cudaError_t read_stream_faults(unsigned int *count, cudaStream_t st) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_stream_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_stream_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace na2d
