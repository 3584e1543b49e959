// na2d_bwd.cu -- backward of the fused NA2D forward: dq, dk, dv and the
// relative-position-bias gradient.
//
// The layer is trained end to end ("Dilated Neighborhood Attention
// Transformer", gitcode DiNAT article, section "微调示例：加载预训练权重继续训练";
// the HF tests described under "源码与测试导览" run forward and backward), so
// its gradients are the chain rule through scores -> softmax -> (dropout ->)
// weighted sum.  For a query with scores s_n, weights p_n, dropout factors
// z_n (0 or 1 / (1 - p_drop); 1 without dropout) and output gradient g:
//     dP_n = z_n (g . v_n),   delta = sum_n p_n dP_n,   ds_n = p_n (dP_n - delta),
//     dq  = sum_n ds_n k_n / sqrt(D),   dk_n += ds_n q / sqrt(D),
//     dv_n += z_n p_n g,    drpb[h, key' - i' + k - 1] += ds_n.
//
// Three passes on the caller's stream (fp32 arithmetic throughout), on
// tensors given by element strides, any D in {16, 32, 64, 128}, and maps
// shorter than k*d treated as zero-padded (padded keys have zero q, k and
// v; padded queries are not outputs, so they carry no gradient):
//  1. bwd_query_kernel, one warp per real query: recomputes the scores and
//     the softmax (lane t holds neighbours t, t + 32, ...), writes dq, and
//     stores the query's log-sum-exp and delta in the workspace; a block
//     covers queries of one (batch, head) image and sums its bias gradient in
//     shared memory before one atomic add per table entry into the
//     workspace's fp32 table.
//  2. bwd_key_kernel, one warp per real key: walks the key's inverse
//     neighbourhood (the queries whose clamped window holds it: per axis a
//     contiguous range of group positions, up to 2k - 1 long) 8 queries at a
//     time (4 lanes per query, a quarter of the channels each), recomputes
//     p = exp(s - lse) and ds from the stored statistics and accumulates dk
//     and dv in registers; no atomics.
//  3. bwd_rpb_kernel rounds the fp32 bias gradient to the bias dtype.
// The workspace is [lse, delta] per query (8 bytes per query and head) plus
// the fp32 table (heads * (2k-1)^2 floats), zeroed by bwd_zero_kernel first.
#include <cuda_runtime.h>

#include <cfloat>
#include <map>
#include <mutex>

#include "na2d_device.cuh"
#include "na2d_launch.h"

namespace na2d {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kQPB = 128;                 // queries per block in the query pass
constexpr int kMaxPerLane = (13 * 13 + 31) / 32;
constexpr int kMaxTab = 25 * 25;          // (2k-1)^2 for k <= 13

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// a . row over D channels: a from shared memory (fp32), the row from global
// memory in 16-byte pieces (the row start is 16-byte aligned).
template <typename T, int D> __device__ __forceinline__ float dot_s(const float *a, const T *row) {
    constexpr int kPer16 = 16 / sizeof(T);
    const uint4 *p4 = reinterpret_cast<const uint4 *>(row);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < D / kPer16; ++c) {
        const uint4 u = __ldg(p4 + c);
        const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
        for (int t = 0; t < kPer16; ++t) s = fmaf(a[c * kPer16 + t], Elem<T>::to_f(e[t]), s);
    }
    return s;
}

struct BwdArgs {
    View q, k, v, g, dq, dk, dv;
    const void *rpb;
    void *drpb;
    float *lse, *delta, *tab;    // workspace
    int heads, H, W, Hp, Wp, K, d;
    int64_t nq;                  // B * heads * H * W (real queries)
    int qblocks;                 // query-pass blocks per image
    float scale;                 // 1 / sqrt(D)
    bool dropout;
    uint32_t drop_thresh;
    float drop_scale;
    uint64_t seed, offset;
};

template <typename T> __device__ __forceinline__ const T *at(const View &x, int64_t b, int h, int y, int xx) {
    return static_cast<const T *>(x.p) + b * x.sb + h * x.sh + y * x.sy + xx * x.sx;
}

// ---------------------------------------------------------------------------
__global__ void bwd_zero_kernel(float *tab, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) tab[i] = 0.f;
}

// ---------------------------------------------------------------------------
// Pass 1: block (image bh, chunk) takes real queries [chunk * kQPB, +kQPB) of
// image bh, one warp per query at a time.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_query_kernel(const BwdArgs a) {
    __shared__ float bins[kMaxTab];
    __shared__ float qs[kWarps][D], gs[kWarps][D];
    constexpr int NC = (D + 31) / 32;
    const int K = a.K, d = a.d, H = a.H, W = a.W, KK = K * K, nb = 2 * K - 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = blockIdx.x / a.qblocks;
    const int chunk = (int)(blockIdx.x - bh * a.qblocks);
    const int64_t b = bh / a.heads;
    const int h = (int)(bh % a.heads);
    for (int i = threadIdx.x; i < nb * nb; i += blockDim.x) bins[i] = 0.f;
    __syncthreads();
    const T *bias = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
    const int q_end = min(H * W, (chunk + 1) * kQPB);
    for (int qi = chunk * kQPB + warp; qi < q_end; qi += kWarps) {
        const int i = qi / W, j = qi - (qi / W) * W;
        const int gy = i % d, iy = i / d, sy = window_start(iy, group_len(a.Hp, d, gy), K);
        const int gx = j % d, ix = j / d, sx = window_start(ix, group_len(a.Wp, d, gx), K);
        // neighbour rows ty < nty and columns tx < ntx lie on the real map
        // (the rest are zero padding): gy + d (sy + ty) < H
        const int nty = min(K, (H - 1 - gy) / d - sy + 1), ntx = min(K, (W - 1 - gx) / d - sx + 1);
        const T *qp = at<T>(a.q, b, h, i, j), *gp = at<T>(a.g, b, h, i, j);
        for (int c = lane; c < D; c += 32) {
            qs[warp][c] = Elem<T>::to_f(qp[c]);
            gs[warp][c] = Elem<T>::to_f(gp[c]);
        }
        __syncwarp();
        const int64_t qlin = bh * H * W + qi;
        float s[kMaxPerLane], dp[kMaxPerLane];
        int tys[kMaxPerLane], txs[kMaxPerLane];
        float m = -FLT_MAX;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            s[r] = -FLT_MAX;
            dp[r] = 0.f;
            tys[r] = n / K;
            txs[r] = n - tys[r] * K;
            if (n < KK) {
                const int ty = tys[r], tx = txs[r];
                const int ky = gy + d * (sy + ty), kx = gx + d * (sx + tx);
                float dot = 0.f;
                if (ty < nty && tx < ntx) {
                    dot = dot_s<T, D>(qs[warp], at<T>(a.k, b, h, ky, kx));
                    dp[r] = dot_s<T, D>(gs[warp], at<T>(a.v, b, h, ky, kx));
                }
                float sv = dot * a.scale;
                if (bias) sv += Elem<T>::to_f(bias[(sy + ty - iy + K - 1) * nb + (sx + tx - ix + K - 1)]);
                s[r] = sv;
                if (a.dropout)
                    dp[r] = dropout_keep((uint64_t)qlin * KK + n, a.seed, a.offset, a.drop_thresh) ? dp[r] * a.drop_scale
                                                                                                   : 0.f;
                m = fmaxf(m, sv);
            }
        }
        m = warp_max(m);
        float l = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            s[r] = lane + 32 * r < KK ? __expf(s[r] - m) : 0.f;
            l += s[r];
        }
        l = warp_sum(l);
        const float inv = 1.f / l;
        float pdp = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            s[r] *= inv;                 // p_n
            pdp = fmaf(s[r], dp[r], pdp);
        }
        const float delta = warp_sum(pdp);
        // ds_n, the bias gradient, then dq (lane = channel)
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            dp[r] = s[r] * (dp[r] - delta);      // ds_n
            if (n < KK) atomicAdd(&bins[(sy + tys[r] - iy + K - 1) * nb + (sx + txs[r] - ix + K - 1)], dp[r]);
        }
        // dq = sum_n ds_n k_n, lane = channel: the neighbours in order, each
        // ds from its lane; the key pointer steps along the window
        float acc[NC];
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) acc[jj] = 0.f;
        const int64_t stx = (int64_t)d * a.k.sx, sty = (int64_t)d * a.k.sy;
        const T *krow = at<T>(a.k, b, h, gy + d * sy, gx + d * sx) + lane, *kp = krow;
        int ty = 0, tx = 0;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            if (32 * r >= KK) break;
            const int cnt = min(32, KK - 32 * r);
            for (int tl = 0; tl < cnt; ++tl) {
                const float dsn = __shfl_sync(0xffffffffu, dp[r], tl);
                if (ty < nty && tx < ntx) {
#pragma unroll
                    for (int jj = 0; jj < NC; ++jj)
                        if (lane + 32 * jj < D) acc[jj] = fmaf(dsn, Elem<T>::to_f(kp[32 * jj]), acc[jj]);
                }
                kp += stx;
                if (++tx == K) {
                    tx = 0;
                    ++ty;
                    krow += sty;
                    kp = krow;
                }
            }
        }
        T *dqp = const_cast<T *>(at<T>(a.dq, b, h, i, j));
#pragma unroll
        for (int jj = 0; jj < NC; ++jj)
            if (lane + 32 * jj < D) dqp[lane + 32 * jj] = Elem<T>::from_f(acc[jj] * a.scale);
        if (lane == 0) {
            a.lse[qlin] = m + __logf(l);
            a.delta[qlin] = delta;
        }
        __syncwarp();   // the next query overwrites this warp's staged rows
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb * nb; i += blockDim.x)
        if (bins[i] != 0.f) atomicAdd(&a.tab[(size_t)h * nb * nb + i], bins[i]);
}

// ---------------------------------------------------------------------------
// The group positions of the queries whose clamped window holds key position
// jp (group coordinates, group length Lg): a contiguous range [lo, hi].
// With window starts s(ip) = clamp(ip - K/2, 0, Lg - K) (non-decreasing):
// hi is the last ip with s(ip) <= jp, i.e. Lg - 1 once jp reaches the last
// start Lg - K, else jp + K/2; lo is the first ip with s(ip) + K > jp, i.e. 0
// while jp < K, else jp - K/2.
__device__ __forceinline__ void inverse_range(int jp, int Lg, int K, int *lo, int *hi) {
    *hi = jp >= Lg - K ? Lg - 1 : jp + K / 2;
    *lo = jp < K ? 0 : jp - K / 2;
}

// Pass 2: one warp per real key pixel (b, head, y, x).  The key's inverse
// neighbourhood (up to (2k - 1)^2 queries) is walked 8 queries at a time:
// lanes 4s .. 4s + 3 take query slot s, each lane a quarter of the channels
// (D / 4), so a query's dot products need two shuffle rounds.  Each lane
// accumulates its quarter of dk and dv for its slot's queries; the 8 slots
// are summed at the end (three shuffle rounds) and slot 0 writes.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_key_kernel(const BwdArgs a) {
    constexpr int QC = D / 4;                      // channels per lane
    const int K = a.K, d = a.d, H = a.H, W = a.W, nb = 2 * K - 1, KK = K * K;
    const int lane = threadIdx.x & 31, slot = lane >> 2, quarter = lane & 3;
    const int c0 = quarter * QC;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t idx = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; idx < a.nq; idx += nwarps) {
        int x, y, h;
        int64_t bh, b;
        split_pixel(idx, W, H, a.heads, x, y, bh, b, h);
        const T *bias = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
        const int gy = y % d, jy = y / d, Lgy = group_len(a.Hp, d, gy);
        const int gx = x % d, jx = x / d, Lgx = group_len(a.Wp, d, gx);
        int ylo, yhi, xlo, xhi;
        inverse_range(jy, Lgy, K, &ylo, &yhi);
        inverse_range(jx, Lgx, K, &xlo, &xhi);
        // real queries only: the padded rows / columns come last in each range
        yhi = min(yhi, (H - 1 - gy) / d);
        xhi = min(xhi, (W - 1 - gx) / d);
        const int nx = xhi - xlo + 1, cnt = (yhi - ylo + 1) * nx;
        const T *kp = at<T>(a.k, b, h, y, x) + c0, *vp = at<T>(a.v, b, h, y, x) + c0;
        float kc[QC], vc[QC], dk[QC], dv[QC];
#pragma unroll
        for (int c = 0; c < QC; ++c) {
            kc[c] = Elem<T>::to_f(kp[c]);
            vc[c] = Elem<T>::to_f(vp[c]);
            dk[c] = dv[c] = 0.f;
        }
        // slot s takes queries s, s + 8, ... of the range in row-major order;
        // two rounds are in flight at a time
        int iy = ylo, ix = xlo + slot;
        while (ix > xhi) {
            ix -= nx;
            ++iy;
        }
        auto round = [&](bool on, int ry, int rx) {
            if (!on) {   // a slot past the range reads the first query, and adds nothing
                ry = ylo;
                rx = xlo;
            }
            const int qy = gy + d * ry, qx = gx + d * rx;
            const T *qp = at<T>(a.q, b, h, qy, qx) + c0, *gp = at<T>(a.g, b, h, qy, qx) + c0;
            const int64_t qlin = bh * H * W + (int64_t)qy * W + qx;
            const float lse = a.lse[qlin], dlt = a.delta[qlin];
            float qc[QC], gc[QC], sdot = 0.f, pdot = 0.f;
#pragma unroll
            for (int c = 0; c < QC; ++c) {
                qc[c] = Elem<T>::to_f(qp[c]);
                gc[c] = Elem<T>::to_f(gp[c]);
                sdot = fmaf(qc[c], kc[c], sdot);
                pdot = fmaf(gc[c], vc[c], pdot);
            }
            sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
            pdot += __shfl_xor_sync(0xffffffffu, pdot, 1);
            sdot += __shfl_xor_sync(0xffffffffu, sdot, 2);
            pdot += __shfl_xor_sync(0xffffffffu, pdot, 2);
            float sv = sdot * a.scale;
            if (bias) sv += Elem<T>::to_f(bias[(jy - ry + K - 1) * nb + (jx - rx + K - 1)]);
            const float p = on ? __expf(sv - lse) : 0.f;
            float z = 1.f;
            if (a.dropout && on) {
                const int n = (jy - window_start(ry, Lgy, K)) * K + (jx - window_start(rx, Lgx, K));
                z = dropout_keep((uint64_t)qlin * KK + n, a.seed, a.offset, a.drop_thresh) ? a.drop_scale : 0.f;
            }
            const float ds = on ? p * (z * pdot - dlt) : 0.f;
            const float pz = p * z;
#pragma unroll
            for (int c = 0; c < QC; ++c) {
                dv[c] = fmaf(pz, gc[c], dv[c]);
                dk[c] = fmaf(ds, qc[c], dk[c]);
            }
        };
        auto advance = [&]() {
            ix += 8;
            while (ix > xhi) {
                ix -= nx;
                ++iy;
            }
        };
        for (int t0 = 0; t0 < cnt; t0 += 16) {
            const int y0 = iy, x0 = ix;
            advance();
            const int y1 = iy, x1 = ix;
            advance();
            round(t0 + slot < cnt, y0, x0);
            if (t0 + 8 < cnt) round(t0 + 8 + slot < cnt, y1, x1);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1)
#pragma unroll
            for (int c = 0; c < QC; ++c) {
                dk[c] += __shfl_xor_sync(0xffffffffu, dk[c], o);
                dv[c] += __shfl_xor_sync(0xffffffffu, dv[c], o);
            }
        if (slot == 0) {
            T *dkp = const_cast<T *>(at<T>(a.dk, b, h, y, x)) + c0, *dvp = const_cast<T *>(at<T>(a.dv, b, h, y, x)) + c0;
#pragma unroll
            for (int c = 0; c < QC; ++c) {
                dkp[c] = Elem<T>::from_f(dk[c] * a.scale);
                dvp[c] = Elem<T>::from_f(dv[c]);
            }
        }
    }
}

// Pass 3: the fp32 bias gradient, rounded to the bias dtype.
template <typename T> __global__ void bwd_rpb_kernel(const float *tab, T *drpb, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        drpb[i] = Elem<T>::from_f(tab[i]);
}

int grid_for(int64_t threads) {
    const int64_t g = (threads + kThreads - 1) / kThreads;
    const int64_t cap = 148LL * 64;
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

template <typename T, int D> cudaError_t launch_bwd_t(const BwdArgs &a, int64_t bh, cudaStream_t st) {
    const int ntab = a.heads * (2 * a.K - 1) * (2 * a.K - 1);
    bwd_zero_kernel<<<grid_for(ntab), kThreads, 0, st>>>(a.tab, ntab);
    bwd_query_kernel<T, D><<<(unsigned)(bh * a.qblocks), kThreads, 0, st>>>(a);
    bwd_key_kernel<T, D><<<grid_for(a.nq * 32), kThreads, 0, st>>>(a);
    if (a.drpb) bwd_rpb_kernel<T><<<grid_for(ntab), kThreads, 0, st>>>(a.tab, static_cast<T *>(a.drpb), ntab);
    note_kernel("bwd_query_kernel+bwd_key_kernel");
    return cudaGetLastError();
}

template <typename T> cudaError_t launch_bwd_d(const BwdArgs &a, int D, int64_t bh, cudaStream_t st) {
    switch (D) {
    case 16: return launch_bwd_t<T, 16>(a, bh, st);
    case 32: return launch_bwd_t<T, 32>(a, bh, st);
    case 64: return launch_bwd_t<T, 64>(a, bh, st);
    default: return launch_bwd_t<T, 128>(a, bh, st);
    }
}

// ---------------------------------------------------------------------------
// Built-in scratch for na2d_backward_noalloc: the same workspace as above
// ([lse, delta] per query and head, then the fp32 bias table), held in a
// fixed array that every GPU loading the library keeps until the process
// exits, for callers that cannot allocate device memory themselves.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocAddrs {
    std::mutex mu;
    std::map<int, void *> dev;   // device -> device address of g_bwd_noalloc_scratch
};
NoAllocAddrs &noalloc_addrs() {
    static NoAllocAddrs a;
    return a;
}

}  // namespace

size_t backward_workspace_bytes(const Problem &p) {
    const size_t nq = (size_t)p.bh() * p.H * p.W;
    const size_t ntab = (size_t)p.heads * (2 * p.k - 1) * (2 * p.k - 1);
    return (2 * nq + ntab) * sizeof(float);
}

cudaError_t launch_backward_views(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                  const View &dout, const View &dq, const View &dk, const View &dv, void *drpb,
                                  const Dropout &drop, void *workspace, cudaStream_t st) {
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = dout; a.dq = dq; a.dk = dk; a.dv = dv;
    a.rpb = rpb; a.drpb = drpb;
    a.nq = p.bh() * p.H * p.W;
    float *ws = static_cast<float *>(workspace);
    a.lse = ws;
    a.delta = ws + a.nq;
    a.tab = ws + 2 * a.nq;
    a.heads = p.heads; a.H = p.H; a.W = p.W; a.Hp = p.Hp(); a.Wp = p.Wp(); a.K = p.k; a.d = p.d;
    a.qblocks = (p.H * p.W + kQPB - 1) / kQPB;
    a.scale = 1.0f / sqrtf((float)p.D);
    a.dropout = drop.p > 0.f;
    const double th = (double)drop.p * 4294967296.0;
    a.drop_thresh = th >= 4294967295.0 ? 0xFFFFFFFFu : (uint32_t)(th + 0.5);
    a.drop_scale = a.dropout ? 1.0f / (1.0f - drop.p) : 1.0f;
    a.seed = drop.seed;
    a.offset = drop.offset;
    if (p.bh() * a.qblocks >= INT32_MAX) return cudaErrorInvalidConfiguration;
    switch (p.dtype) {
    case DType::F32: return launch_bwd_d<float>(a, p.D, p.bh(), st);
    case DType::F16: return launch_bwd_d<__half>(a, p.D, p.bh(), st);
    default: return launch_bwd_d<__nv_bfloat16>(a, p.D, p.bh(), st);
    }
}

cudaError_t launch_backward(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                            const void *dout, void *dq, void *dk, void *dv, void *drpb, void *workspace,
                            cudaStream_t st) {
    return launch_backward_views(p, View::contiguous(q, p), View::contiguous(k, p), View::contiguous(v, p), rpb,
                                 View::contiguous(dout, p), View::contiguous(dq, p), View::contiguous(dk, p),
                                 View::contiguous(dv, p), drpb, Dropout{0.f, 0, 0}, workspace, st);
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// The array's name is only a host-side stand-in in host code; its device
// address is looked up once per device, with that device current, on the
// first call there.
cudaError_t launch_backward_noalloc(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                    const void *dout, void *dq, void *dk, void *dv, void *drpb, cudaStream_t st) {
    if (backward_workspace_bytes(p) > kNoAllocScratchBytes) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    void *scratch = nullptr;
    {
        NoAllocAddrs &a = noalloc_addrs();
        std::lock_guard<std::mutex> lock(a.mu);
        auto it = a.dev.find(dev);
        if (it == a.dev.end()) {
            e = cudaGetSymbolAddress(&scratch, g_bwd_noalloc_scratch);
            if (e != cudaSuccess) return e;
            it = a.dev.emplace(dev, scratch).first;
        }
        scratch = it->second;
    }
    return launch_backward(p, q, k, v, rpb, dout, dq, dk, dv, drpb, scratch, st);
}

}  // namespace na2d
