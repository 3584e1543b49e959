// na2d_stream.cu -- streaming fused NA2D forward for k = 7 sliding windows on
// the tensor cores (f16 / bf16, D = 32, d = 1, 14 <= W <= 64, H >= 8).
//
// What it computes is the layer of "Dilated Neighborhood Attention
// Transformer" (gitcode DiNAT article, section "DiNAT 的核心思想":
// natten2dqkrpb -> softmax -> natten2dav), fused, with the NATTEN clamp rule
// for the window; this file only fixes how the work is scheduled and staged.
//
// Schedule: the map is walked in "steps" of up to SP query-row pairs of one
// image.  A query-row pair needs 8 consecutive key rows (the union of its two
// clamped windows), and consecutive pairs share 6 of them, so every K / V row
// is brought into a shared-memory ring once per CTA and reused by up to four
// pairs.  A CTA owns a contiguous range of pairs in (batch*head, pair) order:
// c CTAs per image when the images fit on the SMs (no range then crosses an
// image), else an even split over one CTA per SM.
//
// Loading, by a producer warp NS - 1 steps ahead through full / empty
// mbarriers: one thread issues one bulk copy (cp.async.bulk) per new image row
// of K, V and Q, with the byte count on the stage's full barrier.  In the
// ramp-up each of the first NS steps is requested once the previous step's
// rows have landed.  All waits are bounded.  The kernel is launched with
// programmatic stream serialisation and reads no global memory before the
// previous kernel on the stream has completed.
//
// Tiles: a consumer warp owns two 8-query tiles per step, each 2 query rows x
// 4 query columns.  The keys of a tile are the 8 x 10 halo of its clamped
// windows (80 keys for 49 useful).  Scores are computed transposed,
// S^T = K Q^T, as mma.sync.m16n8k16 with M = 16 keys (4 key rows x 2 key
// columns per 8 x 8 fragment, 5 such key groups cover the halo) and N = 8
// queries, so every query's scores sit in 10 registers of 8 lanes.  The
// relative-position bias (pre-multiplied by sqrt(D), masked keys at -1e30) is
// the C input of the first MMA, so adding it costs no instruction; each
// lane's 20 bias values per tile live in tensor memory (TMEM), rewritten only
// when the head or the tile's row geometry changes and read back with
// tcgen05.ld.  The row max is a register max plus three shuffles; P is
// exponentiated in fp32, packed, and transposed in registers (movmatrix) into
// the B operand of O^T = V^T P^T, whose A operand is loaded transposed from
// the V rows (ldmatrix.trans).  Row sums come from an MMA against ones; the
// output tile is transposed back with movmatrix and stored.
//
// Shared-memory layout of the rows (Q, K, V; 64 bytes per pixel, four 16-byte
// chunks): row r of a buffer starts at r * pitch + 16 * (r & 3), with image
// column x at pixel 3 + x and zero pixels on both sides (see row_base); any 4
// consecutive rows x 2 adjacent pixels of one chunk index fall in 8 distinct
// bank groups, which is the access pattern of every K and V fragment.  With
// the zero margins every tile's halo starts 3 columns left of the tile, so the
// two tiles of a warp always share their key groups (except at a ragged right
// edge).
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

namespace na2d {
namespace {

constexpr int KW = 7;                 // kernel size handled here
constexpr int NS = 3;                 // pipeline stages (steps in flight)
constexpr int kPixB = 64;             // bytes per pixel (D = 32, 16-bit)
constexpr float kMaskC = -1.0e30f;    // C-init of a masked score
constexpr int kTabPitch = 16;         // floats per bias-table row (13 used)
constexpr int kTabHead = 13 * kTabPitch;
constexpr int kTileCols = 4;          // query columns of a tile
constexpr int kHaloCols = kTileCols + KW - 1;   // 10 key columns per tile
constexpr int kKG = kHaloCols / 2;    // 5 key groups of 16 keys (8 rows x 2 columns)
constexpr int kMargin = KW / 2;       // zero pixels left of every shared-memory row
#ifndef NAT_NWC
#define NAT_NWC 14                    // consumer warps
#define NAT_NT 2                      // 4-column tiles per consumer warp and step
#endif

// Counts bounded waits of this file's kernels that ran out.
__device__ unsigned int g_stream_timeouts;

struct StreamParams {
    const unsigned char *q, *k, *v;
    unsigned char *out;
    const void *rpb;
    int H, W, heads, B;
    // byte strides (batch, head, row, pixel) of q, k, v (one set: the three
    // views of one tensor or three contiguous tensors) and of out
    int64_t in_sb, in_sh, in_sy, in_sx;
    int64_t out_sb, out_sh, out_sy, out_sx;
    int rows_contiguous;   // 1: an image row of q / k / v is one run of W * 64 bytes
    // limit of the data waits in SM clocks (kWaitLimit unless a test shortens
    // it); the final waits for copies in flight always use kWaitLimit
    long long wait_limit;
    int nsteps;      // query-row pairs (split over the CTAs)
    int MX, SP, NP, NR;
    // column bands (maps wider than 64): nb bands of whole 8-column warp
    // spans, band k of band_oct + (k < band_extra) spans; 1 band otherwise
    int nb, band_oct, band_extra;
    uint32_t pitch;  // bytes per shared-memory row: kMargin zero pixels, W pixels, kMargin zero pixels
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
// Bounded wait for the phase with the given parity: gives up after `limit`
// SM clocks (by default 2^31, about a second) and returns false.
constexpr long long kWaitLimit = 1LL << 31;
// Non-blocking test of the phase (no suspend).
__device__ __forceinline__ bool sb_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool sb_wait(uint32_t bar, uint32_t parity, long long limit = kWaitLimit) {
    if (limit < kWaitLimit) {
        // a shortened limit (tests of the error path): poll without the
        // suspend hint, which could outlast the limit
        const long long t0 = clock64();
        while (!sb_test(bar, parity))
            if (clock64() - t0 > limit) return false;
        return true;
    }
    if (sb_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!sb_try(bar, parity))
        if (clock64() - t0 > limit) return false;
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
// The kernel is launched with programmatic stream serialisation: a grid may
// be scheduled while the previous kernel on the stream finishes, runs its
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
// 4 consecutive columns of this thread's lane
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float (&v)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(taddr), "f"(v[0]),
                 "f"(v[1]), "f"(v[2]), "f"(v[3])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
// 16 and 4 consecutive columns of this thread's lane; complete after tmem_ld_wait()
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[kKG][4]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n"
        : "=f"(v[0][0]), "=f"(v[0][1]), "=f"(v[0][2]), "=f"(v[0][3]), "=f"(v[1][0]), "=f"(v[1][1]), "=f"(v[1][2]),
          "=f"(v[1][3]), "=f"(v[2][0]), "=f"(v[2][1]), "=f"(v[2][2]), "=f"(v[2][3]), "=f"(v[3][0]), "=f"(v[3][1]),
          "=f"(v[3][2]), "=f"(v[3][3])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                 : "r"(taddr)
                 : "memory");
}

// ldmatrix (x4, and x4.trans) at a compile-time byte offset from a base
// address: the offset goes into the instruction, so a tile's 20-odd
// fragment loads share one address register.
template <int OFF> __device__ __forceinline__ void ldsm_x4_at(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4+%5];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr), "n"(OFF));
}
template <int OFF> __device__ __forceinline__ void ldsm_x4_t_at(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4+%5];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr), "n"(OFF));
}
// 4-byte global store at a compile-time byte offset from a pointer.
template <int OFF> __device__ __forceinline__ void st_b32_at(unsigned char *ptr, uint32_t v) {
    asm volatile("st.global.b32 [%0+%1], %2;\n" ::"l"(ptr), "n"(OFF), "r"(v) : "memory");
}

// Transposes an 8 x 8 matrix of 16-bit elements held one row-pair per lane
// (the mma / ldmatrix fragment layout) across the warp.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

template <typename T> struct OnesBits;
template <> struct OnesBits<__half> { static constexpr uint32_t v = 0x3C003C00u; };
template <> struct OnesBits<__nv_bfloat16> { static constexpr uint32_t v = 0x3F803F80u; };

// exp2 of two fp32 arguments (fp32 ex2.approx, one MUFU op each), rounded
// and packed in the operand type T (low half = first argument).
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

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}


__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Window start of query row y (or column) on an axis of length L.
__device__ __forceinline__ int win_start(int y, int L) { return clampi(y - KW / 2, 0, L - KW); }

// Halo start of query-row pair p: the first of 8 consecutive key rows that
// hold both rows' clamped windows.
__device__ __forceinline__ int pair_halo(int pair, int H) { return min(win_start(2 * pair, H), H - 8); }


// The CTA's steps in order, with the K / V ring bookkeeping.  A CTA owns a
// contiguous range of query-row pairs in (image, pair) order (global pair
// index bh * NP + pair), which may start and end inside an image; a step is
// up to SP consecutive pairs of one image.  Rows of one image are loaded in
// increasing order, each once, into consecutive ring rows; the next image
// continues after the last ring row of the previous one.  Producer and
// consumers run the same walk.  Only the image, the step's pairs and the ring
// row of the step's first key row are kept; the rest is recomputed.
// Images are walked head-major (image index h * B + b, then the column band),
// so that a CTA's consecutive images share their head and its bias rows: with
// maps of a few pair-steps each (14 x 14), a batch-major walk would change
// the head, and rewrite the bias, at every step.
struct SlideWalk {
    int bh;           // image (a column band of one (head, batch) map when nb > 1)
    int pa, pe;       // the step's first pair and one past its last
    int ge;           // end of the CTA's range (global pair index)
    int h;            // head of image bh
    int b;            // batch of image bh
    int band;         // column band of image bh
    int ring_lo;      // ring row of lo()
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
        const int map = bh / p.nb;
        band = bh - map * p.nb;
        b = map % p.B;
        h = map / p.B;
        ring_lo = 0;
    }
    // byte offset of image (b, h) for the given batch / head strides
    __device__ __forceinline__ int64_t image(int64_t sb, int64_t sh) const { return (int64_t)b * sb + (int64_t)h * sh; }
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
            if (++band == p.nb) {
                band = 0;
                if (++b == p.B) {
                    b = 0;
                    ++h;
                }
            }
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

// Column band k: first image column and width (whole 8-column warp spans;
// the last band ends at the image's right edge).
__device__ __forceinline__ void band_cols(const StreamParams &p, int k, int &bx0, int &bw) {
    bx0 = 8 * (k * p.band_oct + min(k, p.band_extra));
    bw = min(8 * (p.band_oct + (k < p.band_extra ? 1 : 0)), p.W - bx0);
}

// Number of steps in the pair range [gb, ge): per image, ceil(pairs / SP).
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

// Skewed row layout: row r of a buffer starts at r * pitch + 16 * (r & 3)
// bytes; image column x is pixel kMargin + x of the row (pixels and their
// four 16-byte chunks in order), so a whole image row lands with one bulk
// copy.  The kMargin pixels on either side of the image are zeros, written
// once: every tile's 10-column halo starts at x0 - kMargin (clamped only for
// a last tile within 3 columns of the right edge), and halo columns outside
// the image read zero keys and values (their scores are masked by the bias).  Any 4 consecutive rows x 2 adjacent pixels of one chunk index
// fall in 8 distinct bank groups.  The skew makes a row overrun its pitch by
// up to 48 bytes, into the next row's left margin (zeros both ways); each
// buffer keeps 64 bytes of slack after its last row.
__device__ __forceinline__ uint32_t row_base(int r, uint32_t pitch) { return (uint32_t)r * pitch + 16u * (r & 3); }

// Fragment loads of key group G (compile time): K k-steps 0 / 1, V channels
// 0-15 / 16-31.
template <int G> __device__ __forceinline__ void ld_k(uint32_t (&k0)[4], uint32_t (&k1)[4], uint32_t base) {
    ldsm_x4_at<128 * G>(k0, base);
    ldsm_x4_at<128 * G + 32>(k1, base);
}
template <int G> __device__ __forceinline__ void ld_v(uint32_t (&v0)[4], uint32_t (&v1)[4], uint32_t base) {
    ldsm_x4_t_at<128 * G>(v0, base);
    ldsm_x4_t_at<128 * G + 32>(v1, base);
}
template <int G, int N, typename F> __device__ __forceinline__ void static_for(F &&f) {
    if constexpr (G < N) {
        f(std::integral_constant<int, G>{});
        static_for<G + 1, N>(f);
    }
}

// One P.V k-step of a tile: O^T += V^T P^T (channels 0-15 and 16-31) and the
// row sums l += 1^T P^T; `first` starts the accumulators at zero.
template <typename T>
__device__ __forceinline__ void pv_step(float (&o)[2][4], float (&l)[4], const uint32_t (&v0)[4], const uint32_t (&v1)[4],
                                        const uint32_t (&b)[2], const uint32_t (&ones)[4], bool first) {
    if (first) {
        Mma<T>::run0(o[0], v0, b[0], b[1]);
        Mma<T>::run0(o[1], v1, b[0], b[1]);
        Mma<T>::run0(l, ones, b[0], b[1]);
    } else {
        Mma<T>::run(o[0], v0, b[0], b[1]);
        Mma<T>::run(o[1], v1, b[0], b[1]);
        Mma<T>::run(l, ones, b[0], b[1]);
    }
}

// ---------------------------------------------------------------------------
// NT 8-query tiles (u < NT) of one warp: S^T = K Q^T + bias, softmax,
// O^T = V^T P^T, store.  Fragment roles, with g = lane / 4 and c = lane % 4:
//   key group t (16 keys): key m < 8 is halo row m / 2, column 2t + m % 2;
//     key m >= 8 is halo row 4 + (m - 8) / 2, column 2t + m % 2;
//   query n (8 per tile): tile row n / 4, tile column n % 4;
//   s[u][t][j] is the score of key g + 8 (j / 2) for query 2c + j % 2.
//   qa[u]: this lane's Q address (query lane % 8, chunk lane / 8);
//   ka[u]: K address of key group 0, k-step 0 (key lane % 16, chunk lane / 16);
//          group t is + 128 t bytes, k-step 1 is + 32;
//   va[u]: V address of key group 0, channels 0-15 (key lane % 8 + 8 (lane / 16),
//          chunk (lane / 8) % 2); channels 16-31 are + 32;
//   tb: this warp's TMEM bias columns (tile u at + 32 u);
//   out[u]: this lane's output pixel (query lane / 4 of tile u), or null.
// All exponentials of the tiles are issued before their P.V products, so the
// MUFU work of one warp forms one long independent run.
// ---------------------------------------------------------------------------
template <typename T, int NT, bool SHARED>
__device__ __forceinline__ void tile_run(const uint32_t (&qa)[NT], const uint32_t (&ka)[NT], const uint32_t (&va)[NT],
                                         uint32_t tb, float c_log2, unsigned char *const (&out)[NT], int lane) {
    // SHARED (NT = 2, halo columns of tile 1 = those of tile 0 + 4): the two
    // tiles' 14 halo columns are 7 key groups; tile 0 uses groups 0-4 and
    // tile 1 groups 2-6, so each K / V fragment is loaded once for both.
    static_assert(!SHARED || NT == 2, "shared key groups pair two adjacent tiles");
    constexpr int NG = SHARED ? kKG + 2 : kKG;   // key groups loaded per tile set
    float s[NT][kKG][4];
    uint32_t qb[NT][4];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        tmem_ld16(tb + 32u * u, *reinterpret_cast<float(*)[kKG][4]>(&s[u][0][0]));
        tmem_ld4(tb + 32u * u + 16u, s[u][4]);
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) ldsm_x4(qb[u], qa[u]);
    tmem_ld_wait();
    // ---- S^T = K Q^T + bias (C-init)
    if constexpr (SHARED) {
        static_for<0, NG>([&](auto G) {
            constexpr int gi = decltype(G)::value;
            uint32_t k0[4], k1[4];
            ld_k<gi>(k0, k1, ka[0]);
            if constexpr (gi < kKG) {
                Mma<T>::run(s[0][gi], k0, qb[0][0], qb[0][1]);
                Mma<T>::run(s[0][gi], k1, qb[0][2], qb[0][3]);
            }
            if constexpr (gi >= 2) {
                Mma<T>::run(s[1][gi - 2], k0, qb[1][0], qb[1][1]);
                Mma<T>::run(s[1][gi - 2], k1, qb[1][2], qb[1][3]);
            }
        });
    } else {
        static_for<0, kKG>([&](auto G) {
            constexpr int t = decltype(G)::value;
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                uint32_t k0[4], k1[4];
                ld_k<t>(k0, k1, ka[u]);
                Mma<T>::run(s[u][t], k0, qb[u][0], qb[u][1]);
                Mma<T>::run(s[u][t], k1, qb[u][2], qb[u][3]);
            }
        });
    }
    // ---- row max of queries 2c (m[u][0]) and 2c + 1 (m[u][1]): registers, then
    // the 8 lanes that hold the other keys of the same queries
    float m[NT][2];
#pragma unroll
    for (int u = 0; u < NT; ++u)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float x = max3(s[u][0][e], s[u][0][e + 2], s[u][1][e]);
            x = max3(x, s[u][1][e + 2], s[u][2][e]);
            x = max3(x, s[u][2][e + 2], s[u][3][e]);
            x = max3(x, s[u][3][e + 2], s[u][4][e]);
            m[u][e] = fmaxf(x, s[u][4][e + 2]);
        }
#pragma unroll
    for (int sh = 4; sh <= 16; sh <<= 1)
#pragma unroll
        for (int u = 0; u < NT; ++u)
#pragma unroll
            for (int e = 0; e < 2; ++e) m[u][e] = fmaxf(m[u][e], __shfl_xor_sync(0xffffffffu, m[u][e], sh));
    // ---- P = exp2((S - max) log2(e) / sqrt(D)), packed and transposed into
    // the B operands of the P.V k-steps
    uint32_t bp[NT][kKG][2];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        const float n0 = -m[u][0] * c_log2, n1 = -m[u][1] * c_log2;
#pragma unroll
        for (int t = 0; t < kKG; ++t) {
            float x0, x1, x2, x3;
            fma2(x0, x1, s[u][t][0], s[u][t][1], c_log2, n0, n1);
            fma2(x2, x3, s[u][t][2], s[u][t][3], c_log2, n0, n1);
            bp[u][t][0] = movm_t(Exp2Pair<T>::run(x0, x1));
            bp[u][t][1] = movm_t(Exp2Pair<T>::run(x2, x3));
        }
    }
    // ---- O^T += V^T P^T; l += 1^T P^T gives the row sums
    constexpr uint32_t ONE = OnesBits<T>::v;
    const uint32_t ones[4] = {ONE, ONE, ONE, ONE};
    float o[NT][2][4], l[NT][4];
    static_for<0, NG>([&](auto G) {
        constexpr int gi = decltype(G)::value;
        if constexpr (SHARED) {
            uint32_t v0[4], v1[4];
            ld_v<gi>(v0, v1, va[0]);
            if constexpr (gi < kKG) pv_step<T>(o[0], l[0], v0, v1, bp[0][gi], ones, gi == 0);
            if constexpr (gi >= 2) pv_step<T>(o[NT - 1], l[NT - 1], v0, v1, bp[NT - 1][gi - 2], ones, gi == 2);
        } else {
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                uint32_t v0[4], v1[4];
                ld_v<gi>(v0, v1, va[u]);
                pv_step<T>(o[u], l[u], v0, v1, bp[u][gi], ones, gi == 0);
            }
        }
    });
    // ---- normalise, transpose back (query lane / 4, channels 2c, 2c + 1 of
    // each 8-channel chunk) and store 4 bytes per chunk
    const uint32_t cofs = 4u * (uint32_t)(lane & 3);
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        float i0, i1;
        asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(i0) : "f"(l[u][0]));
        asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(i1) : "f"(l[u][1]));
        uint32_t y[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float a0, a1, a2, a3;
            mul2(a0, a1, o[u][h][0], o[u][h][1], i0, i1);
            mul2(a2, a3, o[u][h][2], o[u][h][3], i0, i1);
            y[2 * h] = movm_t(Elem<T>::pack2(a0, a1));
            y[2 * h + 1] = movm_t(Elem<T>::pack2(a2, a3));
        }
        if (out[u]) {
            unsigned char *op = out[u] + cofs;
            st_b32_at<0>(op, y[0]);
            st_b32_at<16>(op, y[1]);
            st_b32_at<32>(op, y[2]);
            st_b32_at<48>(op, y[3]);
        }
    }
}

// Named barrier among the consumer warps only (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void consumers_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;\n" ::"r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Kernel.  Warps 0 .. NWC-1 consume; warp NWC produces (one thread issues one
// bulk copy per image row).  Each consumer warp owns a fixed position in
// every step: pair warp / MX of the step and the 4 NT query columns starting
// at 4 NT (warp % MX), as NT 4-column tiles, so its column geometry (halo
// columns, the column part of its window masks and bias-table columns) is set
// up once.  The producer starts copying right after the barriers are set up;
// the consumers build the bias table and allocate tensor memory meanwhile.
// ---------------------------------------------------------------------------
template <typename T, int NWC, int NT, bool BANDED>
__global__ void __launch_bounds__((NWC + 1) * 32, 1) fwd_stream_kernel(const __grid_constant__ StreamParams p) {
    static_assert(32 * NT * ((NWC + 3) / 4) <= kTmemCols, "bias columns of all consumer warps fit in TMEM");
    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's range of query-row pairs (the CTAs' loads differ by at most one pair)
    // CTA b takes pairs [b * base + min(b, rem), ...): base = nsteps / grid,
    // the first rem = nsteps % grid CTAs one more
    const int base = p.nsteps / (int)gridDim.x, rem = p.nsteps - base * (int)gridDim.x;
    const int bx = (int)blockIdx.x;
    const int s_begin = bx * base + min(bx, rem), s_end = s_begin + base + (bx < rem ? 1 : 0);
    grid_dep_launch();
    if (s_begin >= s_end) return;
    const int nst = slide_steps(p, s_begin, s_end);

    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + p.off_bar, bar_empty = bar_full + 8 * NS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_bar + 16 * NS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_bar + 16 * NS + 4);
    // bias table, with 64 bytes of padding on either side for unclamped column reads
    float *tab = reinterpret_cast<float *>(smem + p.off_tab + 64);
    const uint32_t pitch = p.pitch;                        // row pitch in bytes
    constexpr uint32_t kLead = kMargin * kPixB;            // image column 0 within a row

    if (threadIdx.x == NWC * 32) {
        for (int i = 0; i < NS; ++i) {
            // bulk copies: one expect_tx arrival per step; strided rows: one
            // cp.async arrival per producer lane
            sb_init(bar_full + 8 * i, p.rows_contiguous ? 1 : 32);
            sb_init(bar_empty + 8 * i, NWC);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();

    if (warp == NWC && !p.rows_contiguous) {
        // =================== producer, strided rows ===================
        // the warp copies each new row's pixels as 16-byte pieces (cp.async),
        // every lane arriving on the stage's full barrier once its copies of
        // the step have landed
        grid_dep_wait();
        SlideWalk w;
        w.init(p, s_begin, s_end);
        for (int i = 0; i < nst; ++i) {
            const int stage = i % NS;
            const int first = i ? w.next(p) : w.lo(p);
            const bool ok = i >= NS ? sb_wait(bar_empty + 8 * stage, (uint32_t)(((i / NS) - 1) & 1), p.wait_limit)
                                    : (i == 0 || sb_wait(bar_full + 8 * (i - 1), 0u, p.wait_limit));
            if (!ok) {
                if (lane == 0) {
                    atomicAdd(&g_stream_timeouts, 1u);
                    *abort_flag = 1;
                }
                break;
            }
            if (*abort_flag) break;
            const int hi = w.hi(p);
            const int y0 = 2 * w.pa, y1 = min(2 * w.pe, p.H);
            const int64_t img = w.image(p.in_sb, p.in_sh);
            const int pieces = p.W * 4;
            for (int row = first; row <= hi; ++row) {
                const uint32_t o = row_base(w.ring(p, row), pitch) + kLead;
                const int64_t src = img + (int64_t)row * p.in_sy;
                for (int e = lane; e < pieces; e += 32) {
                    const int64_t so = src + (int64_t)(e >> 2) * p.in_sx + 16 * (e & 3);
                    const uint32_t d = o + (uint32_t)(e >> 2) * kPixB + 16u * (uint32_t)(e & 3);
                    cp_async_16(sbase + p.off_k + d, p.k + so);
                    cp_async_16(sbase + p.off_v + d, p.v + so);
                }
            }
            for (int y = y0; y < y1; ++y) {
                const uint32_t o = row_base(stage * 2 * p.SP + (y - y0), pitch) + kLead;
                const int64_t src = img + (int64_t)y * p.in_sy;
                for (int e = lane; e < pieces; e += 32)
                    cp_async_16(sbase + o + (uint32_t)(e >> 2) * kPixB + 16u * (uint32_t)(e & 3),
                                p.q + src + (int64_t)(e >> 2) * p.in_sx + 16 * (e & 3));
            }
            cp_async_arrive(bar_full + 8 * stage);
        }
        // every copy lands before the CTA's shared memory is released
        cp_async_wait<0>();
    } else if (warp == NWC) {
        // =================== producer ===================
        // one thread issues one bulk copy per image row: the step's new K and
        // V rows into the ring, its query rows into the stage.  Column bands
        // (BANDED): each copy takes the band's columns and 3 on either side
        // that lie on the map; in a band at the map's left or right edge the
        // warp first zeroes the ring rows' columns off the map.
        if constexpr (BANDED) {
            grid_dep_wait();   // no global read before the previous kernel completes
            const bool leader = lane == 0;
            // a banded row's pixels end one pixel short of its pitch, so the
            // 16 (r & 3) skew never reaches the next row's first pixel
            const int row16 = (int)(pitch / 16) - 4;
            SlideWalk w;
            w.init(p, s_begin, s_end);
            int issued = 0;
            for (int i = 0; i < nst; ++i) {
                const int stage = i % NS;
                const int first = i ? w.next(p) : w.lo(p);
                const bool ok_lane = i >= NS ? sb_wait(bar_empty + 8 * stage, (uint32_t)(((i / NS) - 1) & 1), p.wait_limit)
                                             : (i == 0 || sb_wait(bar_full + 8 * (i - 1), 0u, p.wait_limit));
                const bool ok = __all_sync(0xffffffffu, ok_lane);
                if (!ok) {
                    if (leader) {
                        atomicAdd(&g_stream_timeouts, 1u);
                        *abort_flag = 1;
                    }
                    break;
                }
                if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
                const int hi = w.hi(p);
                const int y0 = 2 * w.pa, y1 = min(2 * w.pe, p.H);
                int bx0, bw;
                band_cols(p, w.band, bx0, bw);
                const int cs = max(0, bx0 - kMargin), ce = min(p.W, bx0 + bw + kMargin);
                const uint32_t rowbytes = (uint32_t)(ce - cs) * kPixB;
                const uint32_t dcol = kLead + (uint32_t)(cs - bx0) * kPixB;   // shared column of image column cs
                // 16-byte pieces off the map: [0, zl) and [zr, row16) of each new row
                // (row16: the row's pixels, without the spare one)
                const int zl = bx0 == 0 ? 4 * kMargin : 0;
                const int zr = bx0 + bw == p.W ? 4 * (p.W - bx0 + kMargin) : row16;
                const int nz = zl + row16 - zr;
                for (int row = first; row <= hi; ++row) {
                    const uint32_t o = row_base(w.ring(p, row), pitch);
                    for (int t = lane; t < nz; t += 32) {
                        const uint32_t off = o + 16u * (uint32_t)(t < zl ? t : zr + t - zl);
                        *reinterpret_cast<uint4 *>(smem + p.off_k + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(smem + p.off_v + off) = make_uint4(0, 0, 0, 0);
                    }
                }
                __syncwarp();
                if (leader) {
                    const uint32_t bar = bar_full + 8 * stage;
                    const int64_t img = w.image(p.in_sb, p.in_sh) + (int64_t)cs * p.in_sx;
                    sb_expect_tx(bar, (uint32_t)(2 * (hi - first + 1) + (y1 - y0)) * rowbytes);
                    for (int row = first; row <= hi; ++row) {
                        const uint32_t o = row_base(w.ring(p, row), pitch) + dcol;
                        const int64_t src = img + (int64_t)row * p.in_sy;
                        bulk_g2s(sbase + p.off_k + o, p.k + src, rowbytes, bar);
                        bulk_g2s(sbase + p.off_v + o, p.v + src, rowbytes, bar);
                    }
                    for (int y = y0; y < y1; ++y)
                        bulk_g2s(sbase + row_base(stage * 2 * p.SP + (y - y0), pitch) + dcol,
                                 p.q + img + (int64_t)y * p.in_sy, rowbytes, bar);
                    ++issued;
                }
            }
            // copies still in flight must land before the CTA's shared
            // memory is released (all of them, unless a wait ran out)
            if (leader)
                for (int j = max(0, issued - NS); j < issued; ++j)
                    sb_wait(bar_full + 8 * (j % NS), (uint32_t)((j / NS) & 1));
        } else if (lane == 0) {
            grid_dep_wait();   // no global read before the previous kernel completes
            const uint32_t rowbytes = (uint32_t)p.W * kPixB;
            SlideWalk w;
            w.init(p, s_begin, s_end);
            int issued = 0;
            for (int i = 0; i < nst; ++i) {
                const int stage = i % NS;
                const int first = i ? w.next(p) : w.lo(p);
                // ramp-up: each of the first NS steps is requested once the
                // previous step's rows have landed, so that the first step's
                // rows do not queue behind the next steps'; later, a step
                // waits for its stage to be released
                const bool ok = i >= NS ? sb_wait(bar_empty + 8 * stage, (uint32_t)(((i / NS) - 1) & 1), p.wait_limit)
                                        : (i == 0 || sb_wait(bar_full + 8 * (i - 1), 0u, p.wait_limit));
                if (!ok) {
                    atomicAdd(&g_stream_timeouts, 1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int hi = w.hi(p);
                const int y0 = 2 * w.pa, y1 = min(2 * w.pe, p.H);
                const uint32_t bar = bar_full + 8 * stage;
                const int64_t img = w.image(p.in_sb, p.in_sh);
                sb_expect_tx(bar, (uint32_t)(2 * (hi - first + 1) + (y1 - y0)) * rowbytes);
                for (int row = first; row <= hi; ++row) {
                    const uint32_t o = row_base(w.ring(p, row), pitch) + kLead;
                    const int64_t src = img + (int64_t)row * p.in_sy;
                    bulk_g2s(sbase + p.off_k + o, p.k + src, rowbytes, bar);
                    bulk_g2s(sbase + p.off_v + o, p.v + src, rowbytes, bar);
                }
                for (int y = y0; y < y1; ++y)
                    bulk_g2s(sbase + row_base(stage * 2 * p.SP + (y - y0), pitch) + kLead,
                             p.q + img + (int64_t)y * p.in_sy, rowbytes, bar);
                ++issued;
            }
            // copies still in flight must land before the CTA's shared
            // memory is released (all of them, unless a wait ran out)
            for (int j = max(0, issued - NS); j < issued; ++j)
                sb_wait(bar_full + 8 * (j % NS), (uint32_t)((j / NS) & 1));
        }
    } else {
        // =================== consumers ===================
        // prologue (overlaps the first copies): bias table, zero margins,
        // tensor memory.  Each thread's first table entry is requested before
        // the zeroing, whose stores then cover the load's latency.
        {
            grid_dep_wait();   // first global read: the bias table
            const T *rpb = reinterpret_cast<const T *>(p.rpb);
            auto tab_entry = [&](int i) {
                const int h = i / kTabHead, a = (i / kTabPitch) % 13, b = i % kTabPitch;
                return (rpb && b < 13) ? Elem<T>::to_f(rpb[(h * 13 + a) * 13 + b]) * p.sqrt_d : 0.f;
            };
            const int ntab = p.heads * kTabHead;
            const float first = (int)threadIdx.x < ntab ? tab_entry(threadIdx.x) : 0.f;
            // zero the margins of every ring row of K and V (the copies write
            // only the image columns): one warp per row.  Banded rows get
            // their margins from the producer, band by band.
            const int lead16 = kMargin * 4, tail0 = lead16 + 4 * p.W, per_row = lead16 + (int)(pitch / 16) - tail0;
            for (int r = BANDED ? 2 * p.NR : warp; r < 2 * p.NR; r += NWC) {
                const uint32_t rowoff = r < p.NR ? p.off_k + row_base(r, pitch) : p.off_v + row_base(r - p.NR, pitch);
                for (int t = lane; t < per_row; t += 32)
                    *reinterpret_cast<uint4 *>(smem + rowoff + 16u * (uint32_t)(t < lead16 ? t : t - lead16 + tail0)) =
                        make_uint4(0, 0, 0, 0);
            }
            if ((int)threadIdx.x < ntab) tab[threadIdx.x] = first;
            for (int i = threadIdx.x + NWC * 32; i < ntab; i += NWC * 32) tab[i] = tab_entry(i);
            if (warp == 0) tmem_alloc(smem_u32(tmem_slot));
            tmem_fence_before();
            consumers_sync(NWC * 32);
            tmem_fence_after();
        }
        const int H = p.H, W = p.W;
        const int g = lane >> 2, c = lane & 3;
        // this warp's TMEM bias columns: lane quarter warp % 4, column slot warp / 4
        const uint32_t tb = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(32 * NT * (warp >> 2));
        // fixed per warp: its pair within the step and its NT 4-column tiles
        const int pw = warp / p.MX, x0 = kTileCols * NT * (warp - pw * p.MX);
        const bool active = warp < p.SP * p.MX;
        const int mk = lane & 15, mv = (lane & 7) + ((lane >> 4) << 3);
        const int krow = ((mk >> 3) << 2) + ((mk & 7) >> 1), vrow = ((mv >> 3) << 2) + ((mv & 7) >> 1);
        uint32_t qcol[NT], kcol[NT], vcol[NT];
        int xq[NT];
        // bias rewrite, column part: table column of key group 0 for this lane's
        // two queries (jlo = 0, 1), and which of the 10 (t, jlo) keys lie in
        // the query's window along x
        int cb[NT][2];
        uint32_t xin[NT];
        bool shared_cols = false;
        int bx0 = 0, bw = W;   // this warp's column band (the whole map unless BANDED)
        // column geometry of the warp's tiles in band k (image column x sits
        // at shared column x - bx0 + kMargin)
        auto set_band = [&](int k) {
            if constexpr (BANDED) band_cols(p, k, bx0, bw);
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                xq[u] = bx0 + x0 + kTileCols * u;
                // halo columns hx .. hx + 9: x0 - 3 .. x0 + 6, except for a last
                // tile that starts within 3 columns of the right edge, whose
                // queries all share the window W - 7 .. W - 1
                const int hx = min(xq[u] - kMargin, W - KW);
                qcol[u] = (uint32_t)(min(xq[u] + (lane & 3), W - 1) - bx0 + kMargin) * kPixB + 16u * (uint32_t)(lane >> 3);
                kcol[u] = (uint32_t)(hx - bx0 + kMargin + (mk & 1)) * kPixB + 16u * (uint32_t)(lane >> 4);
                vcol[u] = (uint32_t)(hx - bx0 + kMargin + (mv & 1)) * kPixB + 16u * (uint32_t)((lane >> 3) & 1);
                xin[u] = 0;
#pragma unroll
                for (int jlo = 0; jlo < 2; ++jlo) {
                    const int qx = min(xq[u] + 2 * (c & 1) + jlo, W - 1), sx = win_start(qx, W);
                    // kx - qx + 6 for key column kx = hx + 2t + (g & 1): within
                    // [0, 12]
                    cb[u][jlo] = hx + (g & 1) - qx + 6;
#pragma unroll
                    for (int t = 0; t < kKG; ++t) {
                        const int kx = hx + 2 * t + (g & 1);
                        xin[u] |= ((unsigned)(kx - sx) < (unsigned)KW ? 1u : 0u) << (2 * t + jlo);
                    }
                }
            }
            // the two tiles' halos are 4 columns apart (all but a warp that
            // holds a last tile starting within 3 columns of the right edge):
            // their key groups can be shared
            shared_cols = NT == 2 && min(xq[NT - 1] - kMargin, W - KW) == xq[0] - kMargin + kTileCols;
        };
        int cur_band = 0;
        set_band(0);
        const int qsel = (lane >> 2) & 1;
        // output pixel of this lane's epilogue query (lane / 4): tile row g / 4, column g % 4
        const int orow = g >> 2, ocol0 = g & 3;
        int bias_key = -1;
        // Geometry of one step for this warp, worked out one step early: right
        // after the previous step's tiles, while their last products and
        // stores drain.
        struct Geo {
            int pair, h, key, band;
            bool work;
            uint32_t qrow, krb, vrb;
            unsigned char *orow;   // output row of this lane's epilogue query, or null
        };
        auto geo_of = [&](const SlideWalk &w, int stage, Geo &e) {
            e.pair = w.pa + pw;
            e.band = w.band;
            e.work = active && e.pair < w.pe;
            if constexpr (BANDED) {
                int b0, bwk;
                band_cols(p, w.band, b0, bwk);
                e.work = e.work && x0 < bwk;   // a warp past a narrow last band has no tiles
            }
            e.h = w.h;
            const int qy0 = 2 * e.pair, qy1 = min(qy0 + 1, H - 1);
            const int hy = pair_halo(e.pair, H);
            e.key = (((w.h * 8 + (qy0 - hy)) * 2 + (qy1 - qy0)) * 4 + (win_start(qy0, H) - hy) * 2 +
                     (win_start(qy1, H) - hy)) * p.nb + w.band;
            e.qrow = sbase + row_base(stage * 2 * p.SP + (qsel ? qy1 : qy0) - 2 * w.pa, pitch);
            // ring rows of this lane's K and V fragment rows
            const int rb = w.ring_lo - w.lo(p) + hy;
            e.krb = sbase + p.off_k + row_base(SlideWalk::wrap(rb + krow, p.NR), pitch);
            e.vrb = sbase + p.off_v + row_base(SlideWalk::wrap(rb + vrow, p.NR), pitch);
            const int oy = orow ? qy0 + 1 : qy0;
            e.orow = (e.work && oy < H) ? p.out + w.image(p.out_sb, p.out_sh) + (int64_t)oy * p.out_sy : nullptr;
        };
        SlideWalk w;
        w.init(p, s_begin, s_end);
        Geo cur;
        geo_of(w, 0, cur);
        int stage = 0;
        uint32_t parity = 0;
        for (int i = 0; i < nst; ++i) {
            if constexpr (BANDED) {
                if (cur.band != cur_band) {
                    cur_band = cur.band;
                    set_band(cur_band);
                }
            }
            if (cur.work && cur.key != bias_key) {
                // bias: rewritten when the head or the row geometry changes,
                // before the wait for the step's rows (it needs none of them),
                // so that it overlaps the copies
                bias_key = cur.key;
                const int qy0 = 2 * cur.pair, qy1 = min(qy0 + 1, H - 1);
                const int hy = pair_halo(cur.pair, H);
                // this lane's queries 2c, 2c + 1 share tile row c / 2; its
                // keys lie on halo rows g / 2 (j < 2) and 4 + g / 2 (j >= 2)
                const int qy = (c >> 1) ? qy1 : qy0, sy = win_start(qy, H);
                const float *rows[2];
                bool yin[2];
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    const int ky = hy + 4 * jh + (g >> 1);
                    yin[jh] = (unsigned)(ky - sy) < (unsigned)KW;
                    rows[jh] = tab + cur.h * kTabHead + clampi(ky - qy + 6, 0, 12) * kTabPitch;
                }
#pragma unroll
                for (int u = 0; u < NT; ++u) {
                    float b[kKG][4];
#pragma unroll
                    for (int t = 0; t < kKG; ++t)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float v = rows[j >> 1][cb[u][j & 1] + 2 * t];
                            const bool in = yin[j >> 1] && ((xin[u] >> (2 * t + (j & 1))) & 1u);
                            b[t][j] = in ? v : kMaskC;
                        }
#pragma unroll
                    for (int t = 0; t < kKG; ++t) tmem_st4(tb + 32u * u + 4u * t, b[t]);
                }
                tmem_st_wait();
            }
            if (!sb_wait(bar_full + 8 * stage, parity, p.wait_limit)) {
                if (lane == 0) {
                    atomicAdd(&g_stream_timeouts, 1u);
                    *abort_flag = 1;
                }
                break;
            }
            // no per-step abort check: a producer that gave up never completes
            // this step's barrier, so the wait above runs out and ends the warp
            if (cur.work) {
                uint32_t qa[NT], ka[NT], va[NT];
                unsigned char *o[NT];
#pragma unroll
                for (int u = 0; u < NT; ++u) {
                    qa[u] = cur.qrow + qcol[u];
                    ka[u] = cur.krb + kcol[u];
                    va[u] = cur.vrb + vcol[u];
                    const int ox = xq[u] + ocol0;
                    o[u] = (cur.orow && ox < W) ? cur.orow + (int64_t)ox * p.out_sx : nullptr;
                }
                if (NT == 2 && shared_cols)
                    tile_run<T, NT, NT == 2>(qa, ka, va, tb, p.c_log2, o, lane);
                else
                    tile_run<T, NT, false>(qa, ka, va, tb, p.c_log2, o, lane);
            }
            __syncwarp();
            if (lane == 0) sb_arrive(bar_empty + 8 * stage);
            const int nstage = stage + 1 == NS ? 0 : stage + 1;
            parity ^= nstage == 0 ? 1u : 0u;
            stage = nstage;
            if (i + 1 < nst) {
                const int npe = w.pe + p.SP;
                if (w.pe - w.pa == p.SP && w.pa >= 2 && npe <= min(p.NP, w.ge - w.bh * p.NP) && 2 * npe <= H - 3) {
                    // this step and the next are full and interior (every
                    // pair's halo starts 3 rows above it, unclamped): the
                    // rows, the ring and the output advance by 2 SP rows and
                    // the bias key stays
                    w.pa = w.pe;
                    w.pe = npe;
                    w.ring_lo = SlideWalk::wrap(w.ring_lo + 2 * p.SP, p.NR);
                    cur.pair += p.SP;
                    cur.qrow = sbase + row_base(stage * 2 * p.SP + 2 * pw + qsel, pitch);
                    const int rb = w.ring_lo + 2 * pw;
                    cur.krb = sbase + p.off_k + row_base(SlideWalk::wrap(rb + krow, p.NR), pitch);
                    cur.vrb = sbase + p.off_v + row_base(SlideWalk::wrap(rb + vrow, p.NR), pitch);
                    if (cur.orow) cur.orow += (int64_t)(2 * p.SP) * p.out_sy;
                } else {
                    w.next(p);
                    geo_of(w, stage, cur);
                }
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

std::atomic<long long> &wait_limit_store() {
    static std::atomic<long long> v{0};
    return v;
}
long long stream_wait_limit() { return wait_limit_store().load(); }

template <typename T, int NWC, int NT, bool BANDED>
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
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fwd_stream_kernel<T, NWC, NT, BANDED>, sp);
    *launched = true;
    note_kernel("fwd_stream_kernel");
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Plan for SP query-row pairs per step; returns the shared-memory bytes.
// `aligned`: every CTA's range lies inside one image.
uint32_t plan_slide(StreamParams &sp, const Problem &pr, int SP, bool aligned) {
    sp.SP = SP;
    sp.NP = (pr.H + 1) / 2;
    const int spi = (sp.NP + sp.SP - 1) / sp.SP;   // steps per image
    // K / V rows needed by NS consecutive steps: 2*SP per step plus a 6-row
    // halo for every image those steps touch (one when no CTA crosses images)
    const int images = aligned ? 1 : std::min(NS, (NS - 2) / spi + 2);
    sp.NR = (int)align_up((uint32_t)(2 * sp.SP * NS + 6 * images), 4);
    // rows: kMargin zero pixels, the image, kMargin zero pixels.  A tile's
    // halo starts at min(x0 - 3, W - 7) >= -3 and spans 10 columns, so every
    // halo column lies in [-3, W + 2]; see row_base.  Banded rows hold a
    // band's MX spans of 8 columns and kMargin columns on either side, plus
    // one spare pixel that keeps the row skew off the next row's pixels.
    sp.pitch = sp.nb > 1 ? (uint32_t)(8 * sp.MX + 2 * kMargin + 1) * kPixB : (uint32_t)(pr.W + 2 * kMargin) * kPixB;
    const uint32_t qbytes = (uint32_t)(NS * 2 * sp.SP) * sp.pitch + 64;
    const uint32_t ring = (uint32_t)sp.NR * sp.pitch + 64;
    sp.off_k = align_up(qbytes, 128);
    sp.off_v = sp.off_k + align_up(ring, 128);
    sp.off_tab = sp.off_v + align_up(ring, 128);
    sp.off_bar = align_up(sp.off_tab + 128 + (uint32_t)(pr.heads * kTabHead * 4), 16);
    return sp.off_bar + 16 * NS + 16;
}

template <typename T, int NWC, int NT>
cudaError_t launch_slide(StreamParams &sp, const Problem &pr, cudaStream_t st, bool *launched) {
    const int span = kTileCols * NT;   // query columns per consumer warp
    // maps wider than 64 columns: column bands of whole spans, at most 56
    // columns each (7 warps per query-row pair), as even as whole spans allow
    const int spans = (pr.W + span - 1) / span;
    sp.nb = pr.W > 64 ? (pr.W + 55) / 56 : 1;
    sp.band_oct = spans / sp.nb;
    sp.band_extra = spans - sp.band_oct * sp.nb;
    sp.MX = sp.band_oct + (sp.band_extra ? 1 : 0);
    const bool banded = sp.nb > 1;
    const void *kern = banded ? reinterpret_cast<const void *>(&fwd_stream_kernel<T, NWC, NT, true>)
                              : reinterpret_cast<const void *>(&fwd_stream_kernel<T, NWC, NT, false>);
    int sms = 0, cap = 0;
    cudaError_t e = stream_device(&sms, &cap, kern);
    if (e != cudaSuccess) return e;
    sp.NP = (pr.H + 1) / 2;
    // an image of the walk is a column band of one (batch, head) map
    const int64_t images = pr.bh() * sp.nb;
    const int64_t npairs = images * sp.NP;
    if (npairs >= INT32_MAX || npairs <= 0) return cudaSuccess;
    sp.nsteps = (int)npairs;
    // CTAs: one per SM with an even split of the pairs, or, when the images
    // fit on the SMs, a whole number c of CTAs per image, so that every CTA's
    // range lies inside one image (no second halo and no second clamped image
    // top, which cost about a step).  The aligned split is taken while it
    // gives a CTA at most one pair more.
    int grid = (int)std::min<int64_t>(npairs, sms);
    bool aligned = false;
    if (images <= sms) {
        const int64_t c = std::min<int64_t>(sms / images, sp.NP);
        const int64_t per = (sp.NP + c - 1) / c, even = (npairs + sms - 1) / sms;
        if (per <= even + 1) {
            // per pairs per CTA when they divide an image's pairs (the ranges
            // then stay inside one image), else an even split over images * c
            aligned = sp.NP % per == 0;
            grid = (int)(images * (aligned ? sp.NP / per : c));
        }
    }
    for (int SP = std::max(1, NWC / sp.MX); SP >= 1; --SP) {
        const uint32_t smem = plan_slide(sp, pr, SP, aligned);
        if ((int)smem > cap) continue;
        return banded ? launch_stream_t<T, NWC, NT, true>(sp, smem, grid, st, launched)
                      : launch_stream_t<T, NWC, NT, false>(sp, smem, grid, st, launched);
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_stream_impl(const Problem &pr, const View &q, const View &k, const View &v, const void *rpb,
                               const View &out, cudaStream_t st, bool *launched) {
    StreamParams sp{};
    sp.q = static_cast<const unsigned char *>(q.p);
    sp.k = static_cast<const unsigned char *>(k.p);
    sp.v = static_cast<const unsigned char *>(v.p);
    sp.out = static_cast<unsigned char *>(const_cast<void *>(out.p));
    sp.rpb = rpb;
    const int64_t e = 2;   // f16 / bf16
    sp.in_sb = q.sb * e; sp.in_sh = q.sh * e; sp.in_sy = q.sy * e; sp.in_sx = q.sx * e;
    sp.out_sb = out.sb * e; sp.out_sh = out.sh * e; sp.out_sy = out.sy * e; sp.out_sx = out.sx * e;
    sp.rows_contiguous = (q.sx == 32 && q.sy == (int64_t)32 * pr.W) ? 1 : 0;
    if (pr.W > 64 && !sp.rows_contiguous) return cudaSuccess;   // bands copy contiguous row segments
    const long long lim = stream_wait_limit();
    sp.wait_limit = lim > 0 ? lim : kWaitLimit;
    sp.H = pr.H; sp.W = pr.W; sp.heads = pr.heads; sp.B = pr.B;
    sp.c_log2 = kLog2e / std::sqrt((float)pr.D);
    sp.sqrt_d = std::sqrt((float)pr.D);
    // NAT_NWC consumer warps (SP query-row pairs of MX column spans each)
    // and a producer warp
    return launch_slide<T, NAT_NWC, NAT_NT>(sp, pr, st, launched);
}

}  // namespace

bool stream_views_supported(const Problem &p, const View &q, const View &k, const View &v) {
    // q, k and v share one set of strides (three contiguous tensors, or the
    // three views of one fused tensor)
    return q.sb == k.sb && q.sh == k.sh && q.sy == k.sy && q.sx == k.sx && q.sb == v.sb && q.sh == v.sh &&
           q.sy == v.sy && q.sx == v.sx;
}

bool stream_supported(const Problem &p) {
    if (p.dtype != DType::F16 && p.dtype != DType::BF16) return false;
    if (p.k != KW || p.D != 32 || p.heads > 64) return false;
    return p.d == 1 && p.W >= 14 && p.H >= 8;                      // sliding rows (bands above 64 columns)
}

cudaError_t launch_forward_stream(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                  const View &out, cudaStream_t st, bool *launched) {
    *launched = false;
    if (!stream_supported(p) || !stream_views_supported(p, q, k, v)) return cudaSuccess;
    if (p.dtype == DType::F16) return launch_stream_impl<__half>(p, q, k, v, rpb, out, st, launched);
    return launch_stream_impl<__nv_bfloat16>(p, q, k, v, rpb, out, st, launched);
}

void set_stream_wait_limit(long long clocks) { wait_limit_store().store(clocks > 0 ? clocks : 0); }

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
