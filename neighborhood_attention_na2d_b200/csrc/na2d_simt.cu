// na2d_simt.cu -- CUDA-core kernels: the fused forward for fp32 (and any k the
// tensor-core kernel does not cover) and the three split-path stages
// (natten2dqkrpb -> softmax -> natten2dav, "Dilated Neighborhood Attention
// Transformer", gitcode DiNAT article, section "DiNAT 的核心思想").
//
// All arithmetic is fp32.  The window rule is the NATTEN clamp rule: per axis
// g = i mod d, i' = i / d, s' = clamp(i' - k/2, 0, Lg - k), keys g + d (s' + t).
#include <cuda_runtime.h>

#include <cfloat>

#include "na2d_device.cuh"
#include "na2d_launch.h"

namespace na2d {
namespace {

constexpr int kHeadDim = 32;
constexpr int kThreads = 256;

// Loads one D = 32 row (16-byte aligned) into fp32 registers.
template <typename T> __device__ __forceinline__ void load_row(const T *p, float (&x)[kHeadDim]) {
    constexpr int kPer16 = 16 / sizeof(T);
    const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int c = 0; c < kHeadDim / kPer16; ++c) {
        uint4 u = __ldg(p4 + c);
        const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
        for (int t = 0; t < kPer16; ++t) x[c * kPer16 + t] = Elem<T>::to_f(e[t]);
    }
}

template <typename T> __device__ __forceinline__ float dot_row(const float (&qf)[kHeadDim], const T *p) {
    float kf[kHeadDim];
    load_row<T>(p, kf);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kHeadDim; ++c) s = fmaf(qf[c], kf[c], s);
    return s;
}

struct QueryWin {
    int gy, iy, sy, gx, ix, sx;
};

__device__ __forceinline__ QueryWin query_window(int i, int j, int H, int W, int K, int d) {
    QueryWin w;
    w.gy = i % d;
    w.iy = i / d;
    w.sy = window_start(w.iy, group_len(H, d, w.gy), K);
    w.gx = j % d;
    w.ix = j / d;
    w.sx = window_start(w.ix, group_len(W, d, w.gx), K);
    return w;
}

// ---------------------------------------------------------------------------
// Fused forward, one warp per (b, head, i, j) query.  Scores: lane t takes
// neighbours n = t, t + 32, ... (n = ty * k + tx, up to six per lane for
// k <= 13), each a full D = 32 dot product.  The row max and sum are warp
// reductions.  Weighted values: lane c accumulates channel c over the
// neighbours in order, each probability taken from its lane by a shuffle, so
// the value rows are read coalesced.
// ---------------------------------------------------------------------------
constexpr int kMaxPerLane = (13 * 13 + 31) / 32;

template <typename T>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                            const T *__restrict__ v, const T *__restrict__ rpb,
                                                            T *__restrict__ out, int heads, int H, int W, int K,
                                                            int d, int64_t nq, float scale) {
    const int nb = 2 * K - 1, KK = K * K;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t idx = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; idx < nq; idx += nwarps) {
        const int j = (int)(idx % W);
        const int64_t t = idx / W;
        const int i = (int)(t % H);
        const int64_t bh = t / H;
        const int h = (int)(bh % heads);
        const QueryWin w = query_window(i, j, H, W, K, d);
        const size_t base = (size_t)bh * H * W;
        const T *bias = rpb ? rpb + (size_t)h * nb * nb : nullptr;
        float qf[kHeadDim];
        load_row<T>(q + (size_t)idx * kHeadDim, qf);

        float sc[kMaxPerLane];
        float m = -FLT_MAX;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            sc[r] = -FLT_MAX;
            if (n < KK) {
                const int ty = n / K, tx = n - ty * K;
                const int ky = w.gy + d * (w.sy + ty), kx = w.gx + d * (w.sx + tx);
                float sv = dot_row<T>(qf, k + (base + (size_t)ky * W + kx) * kHeadDim) * scale;
                if (bias) sv += Elem<T>::to_f(bias[(w.sy + ty - w.iy + K - 1) * nb + (w.sx + tx - w.ix + K - 1)]);
                sc[r] = sv;
                m = fmaxf(m, sv);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            sc[r] = lane + 32 * r < KK ? expf(sc[r] - m) : 0.f;
            l += sc[r];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            if (32 * r >= KK) break;
            const int cnt = min(32, KK - 32 * r);
            for (int tl = 0; tl < cnt; ++tl) {
                const int n = 32 * r + tl;
                const float pn = __shfl_sync(0xffffffffu, sc[r], tl);
                const int ty = n / K, tx = n - ty * K;
                const int ky = w.gy + d * (w.sy + ty), kx = w.gx + d * (w.sx + tx);
                acc = fmaf(pn, Elem<T>::to_f(v[(base + (size_t)ky * W + kx) * kHeadDim + lane]), acc);
            }
        }
        out[(size_t)idx * kHeadDim + lane] = Elem<T>::from_f(acc / l);
    }
}

// ---------------------------------------------------------------------------
// Split path, stage 1: one thread per (query, neighbour n = ty*k + tx).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads) qk_rpb_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                          const T *__restrict__ rpb, float *__restrict__ attn,
                                                          int heads, int H, int W, int K, int d, int64_t total,
                                                          float scale) {
    const int KK = K * K, nb = 2 * K - 1;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(idx % KK);
        const int64_t qi = idx / KK;
        const int j = (int)(qi % W);
        const int64_t t = qi / W;
        const int i = (int)(t % H);
        const int64_t bh = t / H;
        const int h = (int)(bh % heads);
        const QueryWin w = query_window(i, j, H, W, K, d);
        const int ty = n / K, tx = n % K;
        const int ky = w.gy + d * (w.sy + ty), kx = w.gx + d * (w.sx + tx);
        float qf[kHeadDim];
        load_row<T>(q + (size_t)qi * kHeadDim, qf);
        float s = dot_row<T>(qf, k + ((size_t)bh * H * W + (size_t)ky * W + kx) * kHeadDim) * scale;
        if (rpb)
            s += Elem<T>::to_f(rpb[((size_t)h * nb + (w.sy + ty - w.iy + K - 1)) * nb + (w.sx + tx - w.ix + K - 1)]);
        attn[idx] = s;
    }
}

// Split path, stage 2: softmax over the last axis, one warp per query row.
__global__ void __launch_bounds__(kThreads) softmax_kernel(float *__restrict__ attn, int KK, int64_t rows) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        float *row = attn + r * KK;
        float m = -FLT_MAX;
        for (int n = lane; n < KK; n += 32) m = fmaxf(m, row[n]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.f;
        for (int n = lane; n < KK; n += 32) s += expf(row[n] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float inv = 1.f / s;
        for (int n = lane; n < KK; n += 32) row[n] = expf(row[n] - m) * inv;
    }
}

// Split path, stage 3: one thread per (query, channel); a warp covers one query.
template <typename T>
__global__ void __launch_bounds__(kThreads) av_kernel(const float *__restrict__ attn, const T *__restrict__ v,
                                                      T *__restrict__ out, int H, int W, int K, int d,
                                                      int64_t total) {
    const int KK = K * K;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % kHeadDim);
        const int64_t qi = idx / kHeadDim;
        const int j = (int)(qi % W);
        const int64_t t = qi / W;
        const int i = (int)(t % H);
        const int64_t bh = t / H;
        const QueryWin w = query_window(i, j, H, W, K, d);
        const float *p = attn + qi * KK;
        const T *vb = v + (size_t)bh * H * W * kHeadDim + c;
        float acc = 0.f;
        for (int ty = 0; ty < K; ++ty) {
            const int ky = w.gy + d * (w.sy + ty);
            for (int tx = 0; tx < K; ++tx) {
                const int kx = w.gx + d * (w.sx + tx);
                acc = fmaf(p[ty * K + tx], Elem<T>::to_f(vb[((size_t)ky * W + kx) * kHeadDim]), acc);
            }
        }
        out[idx] = Elem<T>::from_f(acc);
    }
}

int grid_for(int64_t work) {
    int64_t g = (work + kThreads - 1) / kThreads;
    const int64_t cap = 148LL * 64;   // grid-stride beyond a few waves
    return (int)(g < cap ? (g > 0 ? g : 1) : cap);
}

template <typename T>
cudaError_t fwd_simt_impl(const Problem &p, const void *q, const void *k, const void *v, const void *rpb, void *out,
                          cudaStream_t st) {
    const int64_t nq = p.bh() * p.H * p.W;
    fwd_simt_kernel<T><<<grid_for(nq * 32), kThreads, 0, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v),
        static_cast<const T *>(rpb), static_cast<T *>(out), p.heads, p.H, p.W, p.k, p.d, nq,
        1.0f / sqrtf((float)p.D));
    note_kernel("fwd_simt_kernel");
    return cudaGetLastError();
}

template <typename T>
cudaError_t qk_rpb_impl(const Problem &p, const void *q, const void *k, const void *rpb, float *attn,
                        cudaStream_t st) {
    const int64_t total = p.bh() * p.H * p.W * p.k * p.k;
    qk_rpb_kernel<T><<<grid_for(total), kThreads, 0, st>>>(static_cast<const T *>(q), static_cast<const T *>(k),
                                                           static_cast<const T *>(rpb), attn, p.heads, p.H, p.W,
                                                           p.k, p.d, total, 1.0f / sqrtf((float)p.D));
    return cudaGetLastError();
}

template <typename T>
cudaError_t av_impl(const Problem &p, const float *attn, const void *v, void *out, cudaStream_t st) {
    const int64_t total = p.bh() * p.H * p.W * kHeadDim;
    av_kernel<T><<<grid_for(total), kThreads, 0, st>>>(attn, static_cast<const T *>(v), static_cast<T *>(out), p.H,
                                                       p.W, p.k, p.d, total);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_simt(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                void *out, cudaStream_t st) {
    switch (p.dtype) {
    case DType::F32: return fwd_simt_impl<float>(p, q, k, v, rpb, out, st);
    case DType::F16: return fwd_simt_impl<__half>(p, q, k, v, rpb, out, st);
    default: return fwd_simt_impl<__nv_bfloat16>(p, q, k, v, rpb, out, st);
    }
}

cudaError_t launch_qk_rpb(const Problem &p, const void *q, const void *k, const void *rpb, float *attn,
                          cudaStream_t st) {
    switch (p.dtype) {
    case DType::F32: return qk_rpb_impl<float>(p, q, k, rpb, attn, st);
    case DType::F16: return qk_rpb_impl<__half>(p, q, k, rpb, attn, st);
    default: return qk_rpb_impl<__nv_bfloat16>(p, q, k, rpb, attn, st);
    }
}

cudaError_t launch_softmax(const Problem &p, float *attn, cudaStream_t st) {
    const int64_t rows = p.bh() * p.H * p.W;
    const int warps_per_block = kThreads / 32;
    int64_t g = (rows + warps_per_block - 1) / warps_per_block;
    const int64_t cap = 148LL * 64;
    softmax_kernel<<<(int)(g < cap ? (g > 0 ? g : 1) : cap), kThreads, 0, st>>>(attn, p.k * p.k, rows);
    return cudaGetLastError();
}

cudaError_t launch_av(const Problem &p, const float *attn, const void *v, void *out, cudaStream_t st) {
    switch (p.dtype) {
    case DType::F32: return av_impl<float>(p, attn, v, out, st);
    case DType::F16: return av_impl<__half>(p, attn, v, out, st);
    default: return av_impl<__nv_bfloat16>(p, attn, v, out, st);
    }
}

}  // namespace na2d
