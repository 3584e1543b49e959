// na2d_tc.cu -- fused NA2D forward on the tensor cores (f16 / bf16, D = 32).
//
// What it computes ("Dilated Neighborhood Attention Transformer", gitcode DiNAT
// article, section "DiNAT 的核心思想": natten2dqkrpb -> softmax -> natten2dav,
// fused): for every query, scores q.key/sqrt(D) + rpb over its k x k dilated
// window (NATTEN clamp rule), softmax over the k*k scores, weighted sum of the
// values.  Nothing of size k*k reaches global memory.
//
// Design (B200, sm_100a):
//  * Persistent CTAs (8 warps), each owning a contiguous range of "blocks".  A
//    block is one (batch*head, row group gy) strip of TQY query rows (in
//    dilation-group coordinates) by BJ group columns, for BG column groups gx.
//    Working in group coordinates turns every dilation into plain NA on a
//    sub-grid (the d x d interleave), so one code path covers d = 1 and d > 1.
//  * The block's query tile and the union of its queries' windows (the K / V
//    halo) are staged in shared memory with 16-byte cp.async copies, double
//    buffered: block n+1 streams in while block n is computed.  Each pixel's
//    64-byte row is stored with a 2-bit XOR swizzle of its four 16-byte chunks
//    so ldmatrix reads are bank-conflict free.
//  * Each warp computes a 16-query tile (TQY x TQX, chosen per k so that its
//    halo is a whole number of 8-key MMA tiles: 8x2 queries / 14x8 keys at
//    k = 7).  QK^T and PV run on mma.sync m16n8k16 with fp32 accumulation;
//    the P fragments are re-packed in registers as the A operand of PV (no
//    shared-memory round trip), and one more MMA against an all-ones B
//    fragment gives the softmax row sums from the same rounded P.  The
//    softmax runs in registers; masking and the relative-position bias come
//    from one bank-conflict-free shared table lookup per score.
//  * Compile-time modes share that tile routine.  FULL: every dilation
//    group has at least NKR rows, so all NKR halo rows exist and the staged
//    halo has a fixed row stride (loads use immediate offsets, the tile body
//    has no branches).  DENSE (TMA path only, k <= 5 in practice): H = W =
//    k*d, every window is its whole k x k group.  GENERIC: everything else,
//    with run-time halo geometry.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <map>
#include <mutex>
#include <set>
#include <tuple>

#include "na2d_device.cuh"
#include "na2d_launch.h"

namespace na2d {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPix = 64;   // bytes per D = 32 row of a 16-bit type

enum Mode : int { kGeneric = 0, kFull = 1, kFullTma = 3, kDenseTma = 4 };

// Per-k warp tile: TQY x TQX queries (16), halo NKR = TQY + K - 1 rows by NKC
// columns (padded to a multiple of 8), processed in chunks of CH 8-key tiles;
// at most TILES warp tiles per block in FULL mode: 8, one per warp of the
// block (with 4 at k >= 9, half the warps idled through every block's tiles;
// the two stages of 8 tiles still fit, 219 KB at k = 13).
template <int K> struct Cfg;
// TILES_TMA: warp tiles per block on the TMA path (k <= 7 only).
template <> struct Cfg<3> { static constexpr int TQY = 4, TQX = 4, NKC = 8, CH = 6, TILES = 8, TILES_TMA = 7; };
template <> struct Cfg<5> { static constexpr int TQY = 4, TQX = 4, NKC = 8, CH = 8, TILES = 8, TILES_TMA = 7; };
template <> struct Cfg<7> { static constexpr int TQY = 8, TQX = 2, NKC = 8, CH = 14, TILES = 8, TILES_TMA = 7; };
template <> struct Cfg<9> { static constexpr int TQY = 2, TQX = 8, NKC = 16, CH = 10, TILES = 8, TILES_TMA = 0; };
template <> struct Cfg<11> { static constexpr int TQY = 4, TQX = 4, NKC = 16, CH = 14, TILES = 8, TILES_TMA = 0; };
template <> struct Cfg<13> { static constexpr int TQY = 4, TQX = 4, NKC = 16, CH = 16, TILES = 8, TILES_TMA = 0; };

constexpr int cround(int x, int m) { return (x + m - 1) / m * m; }

template <int K, int MODE> struct Geo {
    using C = Cfg<K>;
    static constexpr int TQY = C::TQY, TQX = C::TQX, NKC = C::NKC, TILES = C::TILES, TILES_TMA = C::TILES_TMA;
    static constexpr bool DENSE = MODE == kDenseTma;
    static constexpr bool FULL = MODE == kFull || MODE == kFullTma;
    static constexpr bool GENERIC = MODE == kGeneric;
    static constexpr bool TMA = MODE == kFullTma || MODE == kDenseTma;
    static constexpr int NKR = TQY + K - 1;                // halo rows of a warp tile
    static constexpr int HALF = NKC / 8;                   // 8-key tiles per halo row
    static constexpr int ROWS = DENSE ? K : NKR;           // halo rows that can hold keys
    static constexpr int NVALID = ROWS * HALF;             // 8-key tiles that can hold keys
    static constexpr int CH = NVALID <= 16 ? cround(NVALID, 2) : C::CH;
    static constexpr int NT = cround(NVALID, CH);          // 8-key tiles processed
    static constexpr int NCH = NT / CH;
    // staged halo row stride in pixel slots (0: chosen at run time)
    static constexpr int CCM = MODE == kFull      ? (TILES - 1) * TQX + NKC
                               : MODE == kFullTma ? (TILES_TMA > 0 ? TILES_TMA - 1 : 0) * TQX + NKC
                               : DENSE            ? NKC
                                                  : 0;
    static constexpr int RMAXC = FULL ? NKR : (DENSE ? K : 0);
    static constexpr int TPG = DENSE ? (K + TQX - 1) / TQX : 0;   // warp tiles per group (DENSE)
    // Bias tables: rows of 2K-1 bias columns plus a -inf column 2K-1, stored
    // as two planes by column parity; a plane row has PSTRIDE words (the
    // smallest 2 * odd >= K), so the 8 query rows x 4 column pairs a warp
    // reads fall in 32 distinct banks.  Table rows are halo rows relative to
    // the query's window start, from -(TQY-1) to NKR-1.
    static constexpr int RROWS = NKR + TQY - 1;
    static constexpr int PSTRIDE = ((K + 1) / 2) % 2 == 1 ? ((K + 1) / 2) * 2 : ((K + 1) / 2) * 2 + 2;
    static constexpr int RSTRIDE = 2 * PSTRIDE;
    static constexpr int TAB_FLOATS = K * RROWS * RSTRIDE;
    static_assert(TQY * TQX == 16, "a warp tile is one m16 MMA row block");
    static_assert(NT % CH == 0 && CH % 2 == 0, "chunks hold whole k16 steps");
    static_assert(8 % TQY == 0, "the two rows a thread owns share a query row");
    static_assert(PSTRIDE >= K && (PSTRIDE / 2) % 2 == 1, "plane stride");
};

struct Args {
    const void *q, *k, *v, *rpb;
    void *out;
    int heads, H, W, d;
    int qH, mH, qW, mW;            // H = qH*d + mH, W = qW*d + mW: group g has length q + (g < m)
    int BG, BJ, BJQ;               // column groups and group columns per block; Q slots per group
    int n_gxc, n_jc, n_rb;         // blocks along gx, group columns and group rows
    int RMAX, CCMAX;               // staged halo rows per group; slots per staged halo row
    int q_bytes, kv_bytes, stage_bytes, tab_bytes;
    int64_t nblocks;
    float scale_log2e;             // log2(e) / sqrt(D)
};

__device__ __forceinline__ int len_y(const Args &a, int g) { return a.qH + (g < a.mH ? 1 : 0); }
__device__ __forceinline__ int len_x(const Args &a, int g) { return a.qW + (g < a.mW ? 1 : 0); }

// Byte offset of 16-byte chunk c of pixel slot s, swizzled by the slot index.
// Used for the query tile (consecutive slots) and, with s = the column inside
// a halo row, for the halo (so the halo row stride can be anything).
__device__ __forceinline__ uint32_t swz(int s, int c) {
    return (uint32_t)s * kPix + ((uint32_t)(c ^ ((s >> 1) & 3)) << 4);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Position of a block in the walk order (bh, gy, rb, gxc, jc), innermost last.
// A CTA decodes its first block once and then steps with carries.
struct Walk {
    int64_t bh;
    int gy, rb, gxc, jc;
};

__device__ __forceinline__ Walk walk_at(const Args &a, int64_t blk) {
    Walk w;
    w.jc = (int)(blk % a.n_jc);
    int64_t t = blk / a.n_jc;
    w.gxc = (int)(t % a.n_gxc);
    t /= a.n_gxc;
    w.rb = (int)(t % a.n_rb);
    t /= a.n_rb;
    w.gy = (int)(t % a.d);
    w.bh = t / a.d;
    return w;
}

__device__ __forceinline__ void walk_next(const Args &a, Walk &w) {
    if (++w.jc < a.n_jc) return;
    w.jc = 0;
    if (++w.gxc < a.n_gxc) return;
    w.gxc = 0;
    if (++w.rb < a.n_rb) return;
    w.rb = 0;
    if (++w.gy < a.d) return;
    w.gy = 0;
    ++w.bh;
}

// Geometry of one block: query rows [i0, i0 + nrows) of row group gy, staged
// halo rows [hr0, hr0 + CR), column groups from gx0, group columns from j0.
struct Block {
    int64_t bh;
    int h, gy, i0, Lgy, nrows, hr0, CR, gx0, j0;
};

template <int K, int MODE>
__device__ __forceinline__ Block block_of(const Args &a, const Walk &w) {
    using G = Geo<K, MODE>;
    Block b;
    b.bh = w.bh;
    b.h = (int)(w.bh % a.heads);
    b.gy = w.gy;
    b.i0 = w.rb * G::TQY;
    b.Lgy = len_y(a, w.gy);
    b.nrows = min(G::TQY, b.Lgy - b.i0);   // <= 0: empty block
    if (G::FULL) {
        // all NKR halo rows exist: start early enough near the bottom edge
        b.hr0 = min(window_start(b.i0, b.Lgy, K), b.Lgy - G::NKR);
        b.CR = G::NKR;
    } else if (G::DENSE) {
        b.hr0 = 0;
        b.CR = K;
    } else {
        b.hr0 = b.nrows > 0 ? window_start(b.i0, b.Lgy, K) : 0;
        b.CR = min(G::NKR, b.Lgy - b.hr0);
    }
    b.gx0 = w.gxc * a.BG;
    b.j0 = w.jc * a.BJ;
    return b;
}

template <int K, int MODE> __device__ __forceinline__ int rmax(const Args &a) {
    return Geo<K, MODE>::RMAXC ? Geo<K, MODE>::RMAXC : a.RMAX;
}
template <int K, int MODE> __device__ __forceinline__ int ccmax(const Args &a) {
    return Geo<K, MODE>::CCM ? Geo<K, MODE>::CCM : a.CCMAX;
}

// Issue the cp.async copies that stage a block.  Work is split into segments
// of contiguous pixels (a query row, or a halo row, of one column group); a
// warp takes every 8th segment and its lanes take (pixel, 16-byte chunk).
// Offsets inside one (batch, head) plane fit in 32 bits (checked on the host).
template <typename T, int K, int MODE>
__device__ void stage_block(const Args &a, const Block &b, unsigned char *stage, int warp, int lane) {
    using G = Geo<K, MODE>;
    const size_t plane = (size_t)a.H * a.W * 32;
    const T *qg = static_cast<const T *>(a.q) + (size_t)b.bh * plane;
    const T *kg = static_cast<const T *>(a.k) + (size_t)b.bh * plane;
    const T *vg = static_cast<const T *>(a.v) + (size_t)b.bh * plane;
    const uint32_t qs = smem_u32(stage);
    const uint32_t ks = qs + a.q_bytes;
    const uint32_t vs = ks + a.kv_bytes;
    const int chunk = lane & 3, px = lane >> 2;
    const int pstep = 8 * a.d * 32;                  // 8 pixels of one group row, in elements
    const int lsrc = px * a.d * 32 + chunk * 8;      // this lane's first element
    const int RM = rmax<K, MODE>(a), CM = ccmax<K, MODE>(a);
    // query rows: segments (gxl, qr), qr fastest
    {
        int gxl = 0, qr = warp;
        while (qr >= b.nrows && gxl < a.BG) { qr -= b.nrows; ++gxl; }
        while (gxl < a.BG) {
            const int gx = b.gx0 + gxl;
            if (gx >= a.d) break;
            const int ncols = min(a.BJ, len_x(a, gx) - b.j0);
            const int y = b.gy + a.d * (b.i0 + qr);
            const T *row = qg + (y * a.W + gx + a.d * b.j0) * 32 + lsrc;
            for (int c = px, off = 0; c < ncols; c += 8, off += pstep)
                cp_async_16(qs + swz((gxl * a.BJQ + c) * G::TQY + qr, chunk), row + off);
            qr += kWarps;
            while (qr >= b.nrows && gxl < a.BG) { qr -= b.nrows; ++gxl; }
        }
    }
    // halo rows: segments (gxl, rho), rho fastest; the chunk swizzle is keyed
    // on the column, so it is a per-lane constant
    {
        const uint32_t ldst = swz(px, chunk);
        int gxl = 0, rho = warp;
        while (rho >= b.CR && gxl < a.BG) { rho -= b.CR; ++gxl; }
        while (gxl < a.BG) {
            const int gx = b.gx0 + gxl;
            if (gx >= a.d) break;
            const int Lgx = len_x(a, gx);
            if (b.j0 < Lgx) {
                const int hc0 = window_start(b.j0, Lgx, K);
                const int CC = min(a.BJ + K - 1, Lgx - hc0);
                const int y = b.gy + a.d * (b.hr0 + rho);
                const int src0 = (y * a.W + gx + a.d * hc0) * 32 + lsrc;
                const uint32_t dst0 = (uint32_t)((gxl * RM + rho) * CM) * kPix + ldst;
                for (int c = px, off = 0, doff = 0; c < CC; c += 8, off += pstep, doff += 8 * kPix) {
                    cp_async_16(ks + dst0 + doff, kg + src0 + off);
                    cp_async_16(vs + dst0 + doff, vg + src0 + off);
                }
            }
            rho += kWarps;
            while (rho >= b.CR && gxl < a.BG) { rho -= b.CR; ++gxl; }
        }
    }
}

// Bias / mask tables for head h.  Table o (o = 0..K-1) serves queries whose
// window starts o - (K-1) rows from them (o = K/2 in the interior).  Row
// rr = rho' + TQY - 1 of table o, for a key row rho' rows after the window
// start, holds rpb[h][rho' + o][col] * log2(e) when 0 <= rho' < K (the key row
// is in the window) and -inf otherwise; column 2K-1 is -inf everywhere and is
// used for keys outside the query's window columns.  One lookup therefore
// gives "bias, or masked" for any score of a warp tile.  Column c of a row is
// stored at word (c & 1) * PSTRIDE + (c >> 1).  NTHREADS threads build it.
template <typename T, int K, int NTHREADS>
__device__ void build_tables(const Args &a, int h, float *tab) {
    using G = Geo<K, kGeneric>;
    const int nb = 2 * K - 1;
    const T *rpb = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int pr = warp; pr < K * G::RROWS; pr += NTHREADS / 32) {   // one (table, row) per warp
        const int o = pr / G::RROWS;
        const int rr = pr - o * G::RROWS - (G::TQY - 1);             // key row relative to window start
        const bool rin = rr >= 0 && rr < K;
        for (int w = lane; w < G::RSTRIDE; w += 32) {
            const int col = (w >= G::PSTRIDE ? 1 : 0) + 2 * (w >= G::PSTRIDE ? w - G::PSTRIDE : w);
            float val = -INFINITY;
            if (rin && col < nb) val = rpb ? Elem<T>::to_f(rpb[(rr + o) * nb + col]) * kLog2e : 0.f;
            tab[pr * G::RSTRIDE + w] = val;
        }
    }
}

// Swizzle-key offset of halo row rho in a TMA box whose rows are CCM pixels.
template <class G> __device__ __forceinline__ constexpr int kr_of(int rho) { return ((G::CCM / 2) * rho) & 3; }

template <typename T> struct Ones;
template <> struct Ones<__half> { static constexpr uint32_t v = 0x3C003C00u; };
template <> struct Ones<__nv_bfloat16> { static constexpr uint32_t v = 0x3F803F80u; };

// One warp computes one 16-query tile: TQY group rows [i0, i0+TQY) by TQX group
// columns [jt0, jt0+TQX) of column group gx.
// The staged query tile is column-major ([group][column][row], qw == 0) when
// cp.async staged it, or row-major ([group][row][qw columns], qg pixels per
// group) when a TMA box did.
template <typename T, int K, int MODE>
__device__ __forceinline__ void compute_tile(const Args &a, const Block &b, const unsigned char *stage,
                                             const float *tab, int gxl, int jt, int lane, int qw = 0, int qg = 0) {
    using G = Geo<K, MODE>;
    const int gx = b.gx0 + gxl;
    if (gx >= a.d) return;
    const int Lgx = len_x(a, gx);
    const int jt0 = b.j0 + jt * G::TQX;
    if (jt0 >= Lgx) return;
    const int hc0 = window_start(b.j0, Lgx, K);
    const int wc0 = window_start(jt0, Lgx, K);
    const int coff = wc0 - hc0;   // warp halo column 0 inside the staged halo

    const uint32_t qs = smem_u32(stage);
    const uint32_t ks = qs + a.q_bytes;
    const uint32_t vs = ks + a.kv_bytes;

    // ---- A operand: the 16 queries (m = qc * TQY + qr), D = 32 as two k16 steps
    uint32_t qa[2][4];
    {
        const int m = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int slot = qw ? gxl * qg + (m % G::TQY) * qw + (jt0 - b.j0) + m / G::TQY
                            : (gxl * a.BJQ + (jt0 - b.j0)) * G::TQY + m;
        ldsm_x4(qa[0], qs + swz(slot, (lane >> 4)));
        ldsm_x4(qa[1], qs + swz(slot, (lane >> 4) + 2));
    }

    // ---- this thread's queries: rows g and g+8 of the tile share query row qr
    const int g = lane >> 2, c4 = lane & 3;
    const int qr = g % G::TQY;
    const int qc0 = g / G::TQY, qc1 = qc0 + 8 / G::TQY;
    const int iq = min(b.i0 + qr, b.Lgy - 1);   // clamped: padding rows stay finite
    const int sy = window_start(iq, b.Lgy, K);
    const int trow = (sy - iq + K - 1) * G::RROWS + (b.hr0 - sy) + (G::TQY - 1);
    int boff[2][G::HALF][2];   // [query column][halo column half][even/odd key]: table word
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int jq = min(jt0 + (s ? qc1 : qc0), Lgx - 1);
        const int sx = window_start(jq, Lgx, K);
#pragma unroll
        for (int hh = 0; hh < G::HALF; ++hh)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kc = wc0 + hh * 8 + 2 * c4 + e;   // key group column
                const bool in = (unsigned)(kc - sx) < (unsigned)K;
                const int col = in ? kc - jq + K - 1 : 2 * K - 1;
                boff[s][hh][e] = trow * G::RSTRIDE + (col & 1) * G::PSTRIDE + (col >> 1);
            }
    }

    // ---- per-lane ldmatrix addressing of the staged K / V halo.  cp.async
    // staging keys the chunk swizzle on the column; a TMA box keys it on the
    // pixel's linear index rho * CCM + c, i.e. on c plus kr(rho) = (CCM/2 *
    // rho) mod 4, so a lane keeps one address per value of kr.
    const uint32_t rowstride = (uint32_t)ccmax<K, MODE>(a) * kPix;
    const uint32_t gofs = (uint32_t)(gxl * rmax<K, MODE>(a)) * rowstride;
    const uint32_t kbase = ks + gofs, vbase = vs + gofs;
    constexpr int NKR_PAT = G::TMA ? 4 : 1;
    uint32_t klane[G::HALF][NKR_PAT];
    uint32_t vlane[G::HALF][2][NKR_PAT];
#pragma unroll
    for (int hh = 0; hh < G::HALF; ++hh) {
        const int c = coff + hh * 8 + (lane & 7);
#pragma unroll
        for (int kr = 0; kr < NKR_PAT; ++kr) {
            const int key = ((c >> 1) + kr) & 3;
            klane[hh][kr] = kbase + c * kPix + (((lane >> 3) ^ key) << 4);
#pragma unroll
            for (int x = 0; x < 2; ++x) vlane[hh][x][kr] = vbase + c * kPix + ((((lane >> 4) + 2 * x) ^ key) << 4);
        }
    }
    const int vsel = (lane >> 3) & 1;

    float m_run[2] = {-INFINITY, -INFINITY};
    float o[5][4];   // d-tiles 0..3 and, in tile 4, the row sums (P times a ones matrix)
#pragma unroll
    for (int dt = 0; dt < 5; ++dt)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[dt][r] = 0.f;

#pragma unroll
    for (int ch = 0; ch < G::NCH; ++ch) {
        float s[G::CH][4];
        // ---- scores: S = Q K^T (fp32), then * log2(e)/sqrt(D) + bias-or-mask
#pragma unroll
        for (int jj = 0; jj < G::CH; ++jj) {
            const int j = ch * G::CH + jj;
            const int rho = j / G::HALF, hh = j % G::HALF;
            const bool live = j < G::NVALID && (!G::GENERIC || rho < b.CR);
            if (live) {
                uint32_t kb[4];
                ldsm_x4(kb, klane[hh][G::TMA ? kr_of<G>(rho) : 0] + rho * rowstride);
                float acc[4];
                Mma<T>::run0(acc, qa[0], kb[0], kb[1]);
                Mma<T>::run(acc, qa[1], kb[2], kb[3]);
                const float *tr = tab + rho * G::RSTRIDE;   // halo row -> table row
                s[jj][0] = fmaf(acc[0], a.scale_log2e, tr[boff[0][hh][0]]);
                s[jj][1] = fmaf(acc[1], a.scale_log2e, tr[boff[0][hh][1]]);
                s[jj][2] = fmaf(acc[2], a.scale_log2e, tr[boff[1][hh][0]]);
                s[jj][3] = fmaf(acc[3], a.scale_log2e, tr[boff[1][hh][1]]);
            } else {
                s[jj][0] = s[jj][1] = s[jj][2] = s[jj][3] = -INFINITY;
            }
        }
        // ---- softmax over the chunk (log2 domain), rescaling earlier chunks
        float mx[2] = {m_run[0], m_run[1]};
#pragma unroll
        for (int jj = 0; jj < G::CH; ++jj) {
            if (ch * G::CH + jj >= G::NVALID) continue;
            mx[0] = max3(mx[0], s[jj][0], s[jj][1]);
            mx[1] = max3(mx[1], s[jj][2], s[jj][3]);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        }
        float base[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            base[r] = mx[r] == -INFINITY ? 0.f : mx[r];   // a row with no key yet
            if (G::NCH > 1) {
                const float corr = ex2(m_run[r] - base[r]);
#pragma unroll
                for (int dt = 0; dt < 5; ++dt) {
                    o[dt][2 * r] *= corr;
                    o[dt][2 * r + 1] *= corr;
                }
            }
            m_run[r] = mx[r];
        }
#pragma unroll
        for (int jj = 0; jj < G::CH; ++jj) {
            if (ch * G::CH + jj < G::NVALID) {
                s[jj][0] = ex2(s[jj][0] - base[0]);
                s[jj][1] = ex2(s[jj][1] - base[0]);
                s[jj][2] = ex2(s[jj][2] - base[1]);
                s[jj][3] = ex2(s[jj][3] - base[1]);
            } else {
                s[jj][0] = s[jj][1] = s[jj][2] = s[jj][3] = 0.f;
            }
        }
        // ---- O += P V and l += P 1: the score fragments of 8-key tiles 2t and
        // 2t+1 are the A fragment of one k16 step
#pragma unroll
        for (int t = 0; t < G::CH / 2; ++t) {
            const int j0t = ch * G::CH + 2 * t;
            if (j0t >= G::NVALID) continue;
            if (G::GENERIC && j0t / G::HALF >= b.CR) continue;
            uint32_t pa[4];
            pa[0] = Elem<T>::pack2(s[2 * t][0], s[2 * t][1]);
            pa[1] = Elem<T>::pack2(s[2 * t][2], s[2 * t][3]);
            pa[2] = Elem<T>::pack2(s[2 * t + 1][0], s[2 * t + 1][1]);
            pa[3] = Elem<T>::pack2(s[2 * t + 1][2], s[2 * t + 1][3]);
            const int jv = j0t + vsel;
            // an 8-key tile past the halo has P = 0: read any valid row for it
            const int rho = G::GENERIC ? min(jv / G::HALF, b.CR - 1) : min(jv / G::HALF, G::ROWS - 1);
            const int hh = jv % G::HALF;
            uint32_t vb[4], vb2[4];
            const int kr = G::TMA ? kr_of<G>(rho) : 0;
            ldsm_x4_t(vb, vlane[hh][0][kr] + rho * rowstride);
            ldsm_x4_t(vb2, vlane[hh][1][kr] + rho * rowstride);
            Mma<T>::run(o[0], pa, vb[0], vb[1]);
            Mma<T>::run(o[1], pa, vb[2], vb[3]);
            Mma<T>::run(o[2], pa, vb2[0], vb2[1]);
            Mma<T>::run(o[3], pa, vb2[2], vb2[3]);
            Mma<T>::run(o[4], pa, Ones<T>::v, Ones<T>::v);
        }
    }

    // ---- normalise by the row sums and store (rounded to nearest even)
    if (b.i0 + qr >= b.Lgy) return;
    const size_t plane = (size_t)a.H * a.W * 32;
    T *og = static_cast<T *>(a.out) + (size_t)b.bh * plane;
    const int y = b.gy + a.d * (b.i0 + qr);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int jq = jt0 + (r ? qc1 : qc0);
        if (jq >= Lgx) continue;
        const float inv = 1.f / o[4][2 * r];
        T *dst = og + (y * a.W + gx + a.d * jq) * 32 + 2 * c4;
#pragma unroll
        for (int dt = 0; dt < 4; ++dt)
            *reinterpret_cast<uint32_t *>(dst + 8 * dt) = Elem<T>::pack2(o[dt][2 * r] * inv, o[dt][2 * r + 1] * inv);
    }
}

// Two resident CTAs per SM where the k*k score fragments fit in 128 registers
// (k <= 7), one otherwise.
template <typename T, int K, int MODE>
__global__ void __launch_bounds__(kThreads, (K <= 7 ? 2 : 1)) fwd_tc_kernel(const Args a) {
    using G = Geo<K, MODE>;
    extern __shared__ __align__(1024) unsigned char smem[];
    float *tab = reinterpret_cast<float *>(smem);
    unsigned char *stages = smem + a.tab_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t first = (int64_t)blockIdx.x * a.nblocks / gridDim.x;
    const int64_t last = (int64_t)(blockIdx.x + 1) * a.nblocks / gridDim.x;
    if (first >= last) return;

    // Padding slots are never loaded; zero them once so every value an MMA
    // reads is finite.
    for (int i = threadIdx.x * 16; i < 2 * a.stage_bytes; i += kThreads * 16)
        *reinterpret_cast<uint4 *>(stages + i) = make_uint4(0, 0, 0, 0);
    __syncthreads();

    Walk w = walk_at(a, first);
    Block cur = block_of<K, MODE>(a, w);
    if (cur.nrows > 0) stage_block<T, K, MODE>(a, cur, stages, warp, lane);
    cp_async_commit();
    int cur_h = -1;
    const int tpg = G::DENSE ? G::TPG : a.BJ / G::TQX;   // warp tiles per column group
    const int ntiles = a.BG * tpg;

    for (int64_t n = first; n < last; ++n) {
        unsigned char *st = stages + ((n - first) & 1) * a.stage_bytes;
        Block nxt;
        if (n + 1 < last) {
            walk_next(a, w);
            nxt = block_of<K, MODE>(a, w);
            if (nxt.nrows > 0)
                stage_block<T, K, MODE>(a, nxt, stages + ((n + 1 - first) & 1) * a.stage_bytes, warp, lane);
        }
        cp_async_commit();
        if (cur.nrows > 0 && cur.h != cur_h) {
            build_tables<T, K, kThreads>(a, cur.h, tab);
            cur_h = cur.h;
        }
        cp_async_wait<1>();
        __syncthreads();
        if (cur.nrows > 0) {
            for (int t = warp; t < ntiles; t += kWarps) {
                if constexpr (MODE == kFull)
                    compute_tile<T, K, MODE>(a, cur, st, tab, 0, t, lane);
                else
                    compute_tile<T, K, MODE>(a, cur, st, tab, t / tpg, t % tpg, lane);
            }
        }
        __syncthreads();
        if (n + 1 < last) cur = nxt;
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// TMA path (k <= 7, FULL and DENSE modes, H and W multiples of d).
//
// Two CTAs per SM, each with one warp per warp tile of a block (7 for the
// FULL k = 7 blocks, 8 for two dense k = 7 groups).  A CTA owns an equal share
// [t0, t1) of all warp tiles in block order and walks its blocks in step:
// while block n is computed, the tensor copies (cp.async.bulk.tensor, 64-byte
// swizzle) of block n+1 land in the other stage and complete on its mbarrier;
// a CTA barrier ends each block.  With two CTAs per SM one CTA keeps the SM
// busy while the other waits at its barrier.
// ---------------------------------------------------------------------------
template <int K, int MODE> struct SyncGeo {
    using G = Geo<K, MODE>;
    static constexpr int GROUPS = G::FULL ? 1 : (G::TILES_TMA + G::TPG) / G::TPG;   // column groups per block
    static constexpr int NWC = G::FULL ? G::TILES_TMA : GROUPS * G::TPG;           // warps = tiles per block
    // Query-box width in pixels: at least the block's query columns, and such
    // that the 8 pixels an ldmatrix reads down one column land in 8 distinct
    // bank groups under the 64-byte swizzle (odd for TQY = 8, 2 mod 8 for TQY = 4).
    static constexpr int QCOLS = G::FULL ? G::TILES_TMA * G::TQX : G::TPG * G::TQX;
    static constexpr int QW = cround(QCOLS, 8) + (G::TQY == 8 ? 1 : 2);
    static constexpr int QBOX = QW * G::TQY * kPix;
    static constexpr int KCOLS = G::CCM;
    static constexpr int KROWS = G::FULL ? G::NKR : K;
    static constexpr int KBOX = KCOLS * KROWS * kPix;
    static constexpr int QREG = GROUPS * QBOX;
    static constexpr int KREG = GROUPS * KBOX;
    static constexpr int STAGE = QREG + 2 * KREG;
    static constexpr int TAB = cround(G::TAB_FLOATS * 4, 512);
    static constexpr int CTRL = 512;                // two barriers
    static constexpr int SMEM = TAB + CTRL + 2 * STAGE;
    static_assert(QBOX % 512 == 0 && KBOX % 512 == 0, "boxes start on 512-byte swizzle atoms");
    static_assert(G::CCM % 2 == 0, "halo rows hold whole swizzle pairs");
};

struct TmaArgs {
    CUtensorMap tq, tk, tv;   // 5-D maps (D, gx, j', gy, bh*H/d + i') of q, k, v
    Args a;
    int64_t ntiles;           // warp tiles over all blocks
    int tpb;                  // warp tiles per block
};

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the barrier's current phase (parity of its phase index);
// gives up after about 2^31 SM clocks (about a second).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > (1LL << 31)) return false;
    return true;
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c1, int c2,
                                            int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5, %6}], [%7];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}

// Counts bounded waits that ran out (read and cleared by na2d_device_faults).
__device__ unsigned int g_wait_timeouts;

// Thread 0 arms the stage's barrier with the block's byte count and issues its
// tensor copies.
template <int K, int MODE>
__device__ void tma_copy(const TmaArgs &t, const Block &b, uint32_t st, uint32_t bar) {
    using G = Geo<K, MODE>;
    using R = SyncGeo<K, MODE>;
    const Args &a = t.a;
    const int r0 = (int)(b.bh * a.qH);   // merged (batch*head, group row) coordinate of group row 0
    if (G::FULL) {
        const int hc0 = window_start(b.j0, len_x(a, b.gx0), K);
        mbar_expect_tx(bar, R::QBOX + 2 * R::KBOX);
        tma_load_5d(st, &t.tq, bar, b.gx0, b.j0, b.gy, r0 + b.i0);
        tma_load_5d(st + R::QREG, &t.tk, bar, b.gx0, hc0, b.gy, r0 + b.hr0);
        tma_load_5d(st + R::QREG + R::KREG, &t.tv, bar, b.gx0, hc0, b.gy, r0 + b.hr0);
    } else {
        const int ng = min(a.BG, a.d - b.gx0);
        mbar_expect_tx(bar, ng * (R::QBOX + 2 * R::KBOX));
        for (int g = 0; g < ng; ++g) {
            tma_load_5d(st + g * R::QBOX, &t.tq, bar, b.gx0 + g, 0, b.gy, r0 + b.i0);
            tma_load_5d(st + R::QREG + g * R::KBOX, &t.tk, bar, b.gx0 + g, 0, b.gy, r0);
            tma_load_5d(st + R::QREG + R::KREG + g * R::KBOX, &t.tv, bar, b.gx0 + g, 0, b.gy, r0);
        }
    }
}

template <typename T, int K, int MODE>
__global__ void __launch_bounds__(SyncGeo<K, MODE>::NWC * 32, 2) fwd_sync_kernel(const __grid_constant__ TmaArgs t) {
    using G = Geo<K, MODE>;
    using R = SyncGeo<K, MODE>;
    const Args &a = t.a;
    extern __shared__ __align__(1024) unsigned char smem[];
    float *tab = reinterpret_cast<float *>(smem);
    const uint32_t bars = smem_u32(smem + R::TAB);
    unsigned char *stage_ptr = smem + R::TAB + R::CTRL;
    const uint32_t stages = smem_u32(stage_ptr);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t t0 = (int64_t)blockIdx.x * t.ntiles / gridDim.x;
    const int64_t t1 = (int64_t)(blockIdx.x + 1) * t.ntiles / gridDim.x;
    if (t0 >= t1) return;
    const int64_t b0 = t0 / t.tpb, b1 = (t1 - 1) / t.tpb;

    if (threadIdx.x == 0) {
        mbar_init(bars, 1);
        mbar_init(bars + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();

    Walk w = walk_at(a, b0);
    Block cur = block_of<K, MODE>(a, w);
    if (threadIdx.x == 0) tma_copy<K, MODE>(t, cur, stages, bars);
    int cur_h = -1;
    bool fault = false;
    int64_t fault_b = 0;
    for (int64_t bi = b0; bi <= b1; ++bi) {
        const int s = (int)((bi - b0) & 1);
        const uint32_t parity = (uint32_t)(((bi - b0) >> 1) & 1);
        Block nxt;
        if (bi < b1) {
            walk_next(a, w);
            nxt = block_of<K, MODE>(a, w);
            // the other stage was released by the barrier that ended block bi-1
            if (threadIdx.x == 0) tma_copy<K, MODE>(t, nxt, stages + (s ^ 1) * R::STAGE, bars + 8 * (s ^ 1));
        }
        if (cur.h != cur_h) {
            build_tables<T, K, R::NWC * 32>(a, cur.h, tab);
            cur_h = cur.h;
        }
        const bool ok = mbar_wait(bars + 8 * s, parity);
        if (__syncthreads_or(!ok)) {   // also publishes a rebuilt table
            fault = true;
            fault_b = bi;
            break;
        }
        const int64_t lo = t0 - bi * t.tpb, hi = t1 - bi * t.tpb;
        if (warp < t.tpb && warp >= lo && warp < hi) {
            const unsigned char *st = stage_ptr + s * R::STAGE;
            if constexpr (G::FULL)
                compute_tile<T, K, MODE>(a, cur, st, tab, 0, warp, lane, R::QW, 0);
            else
                compute_tile<T, K, MODE>(a, cur, st, tab, warp / G::TPG, warp % G::TPG, lane, R::QW,
                                         R::QW * G::TQY);
        }
        __syncthreads();
        if (bi < b1) cur = nxt;
    }
    if (fault && threadIdx.x == 0) {
        atomicAdd(&g_wait_timeouts, 1u);
        // let copies still in flight (blocks fault_b and fault_b + 1) land before
        // the CTA's shared memory is released; these waits are bounded too
        for (int64_t bi = fault_b; bi <= min(fault_b + 1, b1); ++bi)
            mbar_wait(bars + 8 * (int)((bi - b0) & 1), (uint32_t)(((bi - b0) >> 1) & 1));
    }
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Per-device facts and per-(device, kernel, smem) occupancy, queried once and
// cached, so steady-state launches (and launches under stream capture) make
// no attribute or occupancy queries.
struct LaunchCache {
    std::mutex mu;
    std::map<int, std::pair<int, int>> dev;                       // device -> (SMs, max opt-in smem)
    std::set<std::pair<int, const void *>> smem_set;              // kernels with the smem limit raised
    std::map<std::tuple<int, const void *, int>, int> occ;        // (device, kernel, smem) -> CTAs per SM
};

LaunchCache &cache() {
    static LaunchCache c;
    return c;
}

// (SMs, max opt-in shared memory per block) of the current device.
cudaError_t device_facts(int *dev_out, std::pair<int, int> *facts) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    LaunchCache &c = cache();
    std::lock_guard<std::mutex> lock(c.mu);
    auto it = c.dev.find(dev);
    if (it == c.dev.end()) {
        int n = 0, m = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&m, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
        it = c.dev.emplace(dev, std::make_pair(n, m)).first;
    }
    *dev_out = dev;
    *facts = it->second;
    return cudaSuccess;
}

cudaError_t launch_geometry(const void *kern, int smem, int *sms, int *occ, int threads = kThreads) {
    int dev = 0;
    std::pair<int, int> f;
    cudaError_t e = device_facts(&dev, &f);
    if (e != cudaSuccess) return e;
    *sms = f.first;
    if (smem > f.second) return cudaErrorInvalidConfiguration;
    LaunchCache &c = cache();
    std::lock_guard<std::mutex> lock(c.mu);
    if (!c.smem_set.count({dev, kern})) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, f.second);
        if (e != cudaSuccess) return e;
        c.smem_set.insert({dev, kern});
    }
    auto key = std::make_tuple(dev, kern, smem);
    auto oc = c.occ.find(key);
    if (oc == c.occ.end()) {
        int n = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem)) != cudaSuccess) return e;
        oc = c.occ.emplace(key, std::max(n, 1)).first;
    }
    *occ = oc->second;
    return cudaSuccess;
}

// (Maps whose groups are all exactly k long take the TMA block kernel for
// k <= 7 and the tcgen05 group kernel for k >= 9; should either decline, the
// GENERIC geometry covers them.)
template <int K> int pick_mode(const Problem &p) {
    if (p.H / p.d >= Geo<K, kFull>::NKR) return kFull;
    return kGeneric;
}

// Block shapes.  FULL: one column group per block, the group's warp-tile
// columns split into n_jc equal chunks of at most TILES tiles.  GENERIC: BJ group
// columns by BG column groups, the first candidate (widest BJ first, then the
// most column groups) whose two stages plus bias tables fit in shared memory.
// Returns the shared-memory bytes, or -1 if nothing fits.
template <int K>
int plan_blocks(const Problem &p, Args &a, int mode, int smem_cap) {
    using GG = Geo<K, kGeneric>;
    const int Lgx_max = (p.W + p.d - 1) / p.d;
    const int Lgy_max = (p.H + p.d - 1) / p.d;
    a.tab_bytes = round_up(GG::TAB_FLOATS * 4, 128);
    a.n_rb = (Lgy_max + GG::TQY - 1) / GG::TQY;
    bool ok = false;
    if (mode == kFull) {
        using G = Geo<K, kFull>;
        const int ntx = (Lgx_max + G::TQX - 1) / G::TQX;   // warp-tile columns per group
        a.n_jc = (ntx + G::TILES - 1) / G::TILES;
        a.BJ = (ntx + a.n_jc - 1) / a.n_jc * G::TQX;
        a.BG = 1;
        a.BJQ = G::TILES * G::TQX;
        a.RMAX = G::NKR;
        a.CCMAX = G::CCM;
        a.q_bytes = a.BJQ * G::TQY * kPix;
        a.kv_bytes = G::NKR * G::CCM * kPix;
        ok = a.tab_bytes + 2 * (a.q_bytes + 2 * a.kv_bytes) <= smem_cap;
    } else {
        a.RMAX = std::min(GG::NKR, Lgy_max);
        for (int bj = std::min(round_up(Lgx_max, GG::TQX), 8 * GG::TQX); bj >= GG::TQX && !ok; bj -= GG::TQX) {
            for (int bg = std::max(1, std::min(p.d, kWarps / (bj / GG::TQX))); bg >= 1; --bg) {
                a.BJ = a.BJQ = bj;
                a.BG = bg;
                a.CCMAX = std::min(a.BJ - GG::TQX, Lgx_max - K) + GG::NKC;
                a.q_bytes = a.BG * a.BJQ * GG::TQY * kPix;
                a.kv_bytes = a.BG * a.RMAX * a.CCMAX * kPix;
                ok = a.tab_bytes + 2 * (a.q_bytes + 2 * a.kv_bytes) <= smem_cap;
                if (ok) break;
            }
        }
        a.n_jc = (Lgx_max + a.BJ - 1) / a.BJ;
    }
    if (!ok) return -1;
    a.stage_bytes = a.q_bytes + 2 * a.kv_bytes;
    a.n_gxc = (p.d + a.BG - 1) / a.BG;
    a.nblocks = p.bh() * p.d * a.n_rb * a.n_gxc * a.n_jc;
    return a.tab_bytes + 2 * a.stage_bytes;
}

template <typename T, int K, int MODE>
cudaError_t launch_mode(const Args &a, int smem, cudaStream_t st) {
    auto kern = fwd_tc_kernel<T, K, MODE>;
    int sms = 0, occ = 1;
    cudaError_t e = launch_geometry(reinterpret_cast<const void *>(kern), smem, &sms, &occ);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(a.nblocks, (int64_t)sms * occ);
    kern<<<(unsigned)grid, kThreads, smem, st>>>(a);
    note_kernel(MODE == kFull ? "fwd_tc_kernel/full" : "fwd_tc_kernel/generic");
    return cudaGetLastError();
}

// cuTensorMapEncodeTiled, fetched once through the runtime (no link against
// the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// 5-D view (D, gx, j', gy, bh*H/d + i') of a [B*heads, H, W, 32] tensor with
// H and W multiples of d: pixel (gy + d*i', gx + d*j') of plane bh.  Strides
// are non-decreasing, each the product of the previous extent and stride.
bool encode_map(CUtensorMap *m, const void *base, DType dt, int64_t bh, int H, int W, int d, int box_cols,
                int box_rows, int box_gx = 1) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[5] = {32, (cuuint64_t)d, (cuuint64_t)(W / d), (cuuint64_t)d, (cuuint64_t)bh * (H / d)};
    const cuuint64_t strides[4] = {64, 64ull * d, 64ull * W, 64ull * W * d};
    const cuuint32_t box[5] = {32, (cuuint32_t)box_gx, (cuuint32_t)box_cols, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = enc(m, dt == DType::F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                           const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The TMA path takes k <= 7 problems whose dilation groups all have the same
// length (H, W multiples of d) and are either exactly k long (DENSE) or at
// least NKR long (FULL); the merged row coordinate must fit in 32 bits.
template <int K> int pick_tma_mode(const Problem &p) {
    if (Cfg<K>::TILES_TMA == 0 || p.H % p.d || p.W % p.d) return -1;
    if (p.bh() * (p.H / p.d) >= ((int64_t)1 << 31)) return -1;
    if (!tensor_map_encoder()) return -1;
    if (p.H == K * p.d && p.W == K * p.d) return kDenseTma;
    if (p.H / p.d >= Geo<K, kFullTma>::NKR) return kFullTma;
    return -1;
}

template <typename T, int K, int MODE>
cudaError_t launch_tma(const Problem &p, const Args &base, cudaStream_t st, bool *launched) {
    using G = Geo<K, MODE>;
    using R = SyncGeo<K, MODE>;
    *launched = false;
    TmaArgs t;
    t.a = base;
    Args &a = t.a;
    const int Lgx = p.W / p.d, Lgy = p.H / p.d;
    if (G::FULL) {
        const int ntx = (Lgx + G::TQX - 1) / G::TQX;     // warp-tile columns per group
        a.n_jc = (ntx + G::TILES_TMA - 1) / G::TILES_TMA;
        a.BJ = (ntx + a.n_jc - 1) / a.n_jc * G::TQX;     // equal column chunks
        a.BG = 1;
        t.tpb = a.BJ / G::TQX;
    } else {
        a.BJ = G::TPG * G::TQX;
        a.n_jc = 1;
        a.BG = std::min(R::GROUPS, p.d);
        t.tpb = a.BG * G::TPG;
    }
    a.BJQ = R::QW;
    a.n_gxc = (p.d + a.BG - 1) / a.BG;
    a.n_rb = (Lgy + G::TQY - 1) / G::TQY;
    a.RMAX = G::RMAXC;
    a.CCMAX = G::CCM;
    a.q_bytes = R::QREG;
    a.kv_bytes = R::KREG;
    a.stage_bytes = R::STAGE;
    a.tab_bytes = R::TAB;
    a.nblocks = p.bh() * p.d * a.n_rb * a.n_gxc * a.n_jc;
    t.ntiles = a.nblocks * t.tpb;
    if (!encode_map(&t.tq, a.q, p.dtype, p.bh(), p.H, p.W, p.d, R::QW, G::TQY) ||
        !encode_map(&t.tk, a.k, p.dtype, p.bh(), p.H, p.W, p.d, R::KCOLS, R::KROWS) ||
        !encode_map(&t.tv, a.v, p.dtype, p.bh(), p.H, p.W, p.d, R::KCOLS, R::KROWS))
        return cudaSuccess;   // not launched: the caller takes the cp.async path
    auto kern = fwd_sync_kernel<T, K, MODE>;
    int sms = 0, occ = 1;
    cudaError_t e = launch_geometry(reinterpret_cast<const void *>(kern), R::SMEM, &sms, &occ, R::NWC * 32);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>((t.ntiles + t.tpb - 1) / t.tpb, (int64_t)sms * occ);
    kern<<<(unsigned)grid, R::NWC * 32, R::SMEM, st>>>(t);
    *launched = true;
    note_kernel(MODE == kFullTma ? "fwd_sync_kernel/full_tma" : "fwd_sync_kernel/dense_tma");
    return cudaGetLastError();
}

template <typename T, int K>
cudaError_t launch_impl(const Problem &p, const void *q, const void *k, const void *v, const void *rpb, void *out,
                        cudaStream_t st) {
    Args a;
    a.q = q; a.k = k; a.v = v; a.rpb = rpb; a.out = out;
    a.heads = p.heads; a.H = p.H; a.W = p.W; a.d = p.d;
    a.qH = p.H / p.d; a.mH = p.H % p.d; a.qW = p.W / p.d; a.mW = p.W % p.d;
    a.scale_log2e = kLog2e / sqrtf((float)p.D);
    int dev = 0;
    std::pair<int, int> f;
    cudaError_t e = device_facts(&dev, &f);
    if (e != cudaSuccess) return e;
    if constexpr (Cfg<K>::TILES_TMA > 0) {
        const int tma_mode = pick_tma_mode<K>(p);
        if (tma_mode >= 0) {
            bool launched = false;
            e = tma_mode == kFullTma ? launch_tma<T, K, kFullTma>(p, a, st, &launched)
                                     : launch_tma<T, K, kDenseTma>(p, a, st, &launched);
            if (e != cudaSuccess || launched) return e;
        }
    }
    int mode = pick_mode<K>(p);
    int smem = plan_blocks<K>(p, a, mode, f.second);
    if (smem < 0 && mode != kGeneric) smem = plan_blocks<K>(p, a, mode = kGeneric, f.second);
    if (smem < 0) return cudaErrorInvalidConfiguration;
    if (mode == kFull) return launch_mode<T, K, kFull>(a, smem, st);
    return launch_mode<T, K, kGeneric>(a, smem, st);
}

template <typename T>
cudaError_t launch_t(const Problem &p, const void *q, const void *k, const void *v, const void *rpb, void *out,
                     cudaStream_t st) {
    switch (p.k) {
    case 3: return launch_impl<T, 3>(p, q, k, v, rpb, out, st);
    case 5: return launch_impl<T, 5>(p, q, k, v, rpb, out, st);
    case 7: return launch_impl<T, 7>(p, q, k, v, rpb, out, st);
    case 9: return launch_impl<T, 9>(p, q, k, v, rpb, out, st);
    case 11: return launch_impl<T, 11>(p, q, k, v, rpb, out, st);
    default: return launch_impl<T, 13>(p, q, k, v, rpb, out, st);
    }
}

}  // namespace

cudaError_t read_device_faults(unsigned int *count, cudaStream_t st) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_wait_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_wait_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

bool encode_group_map(CUtensorMap *map, const void *base, DType dt, int64_t bh, int H, int W, int d, int box_cols,
                      int box_rows, int box_gx) {
    return encode_map(map, base, dt, bh, H, W, d, box_cols, box_rows, box_gx);
}

bool tc_supported(const Problem &p) {
    // every dilation group at least k long (no padded map)
    return (p.dtype == DType::F16 || p.dtype == DType::BF16) && p.D == 32 && p.k >= 3 && p.k <= 13 && (p.k & 1) &&
           (int64_t)p.k * p.d <= p.H && (int64_t)p.k * p.d <= p.W;
}

cudaError_t launch_forward_tc(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                              void *out, cudaStream_t st) {
    if (p.dtype == DType::F16) return launch_t<__half>(p, q, k, v, rpb, out, st);
    return launch_t<__nv_bfloat16>(p, q, k, v, rpb, out, st);
}

}  // namespace na2d
