// na2d_simt.cu -- CUDA-core kernels: the generic fused forward and the three
// split-path stages (natten2dqkrpb -> softmax -> natten2dav, "Dilated
// Neighborhood Attention Transformer", gitcode DiNAT article, section
// "DiNAT 的核心思想").
//
// Generic means: any dtype, head dim D in {16, 32, 64, 128}, tensors given by
// element strides (channels contiguous), and maps shorter than k*d.  Such a
// map is treated as padded with zero pixels (q = k = v = 0) at the bottom and
// right up to k*d, as the HF DiNAT layer pads its feature map before
// attention ("maybe_pad"); the window rule runs on the padded size and only
// the real queries are written.  A padded key scores its bias alone and
// contributes a zero value.  The fused forward can also write the attention
// weights (after dropout, as the layer returns them with output_attentions)
// and apply attention dropout between the softmax and the weighted sum.
//
// All arithmetic is fp32.  The window rule is the NATTEN clamp rule: per axis
// g = i mod d, i' = i / d, s' = clamp(i' - k/2, 0, Lg - k), keys g + d (s' + t).
#include <cuda_runtime.h>

#include <cfloat>

#include "na2d_device.cuh"
#include "na2d_launch.h"

namespace na2d {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxPerLane = (13 * 13 + 31) / 32;

struct FwdArgs {
    View q, k, v, out;
    const void *rpb;
    float *attn;                 // [B, heads, H, W, k*k] fp32, or null
    int heads, H, W, Hp, Wp, K, d;
    int64_t nq;                  // B * heads * H * W (real queries)
    float scale;                 // 1 / sqrt(D)
    uint32_t drop_thresh;        // keep a weight when its Philox word >= this
    float drop_scale;            // 1 / (1 - p)
    uint64_t seed, offset;
    bool dropout;
};

// q . key over D channels: q from shared memory (fp32), the key row from
// global memory in 16-byte pieces (the row start is 16-byte aligned).
template <typename T, int D> __device__ __forceinline__ float dot_q(const float *qs, const T *kp) {
    constexpr int kPer16 = 16 / sizeof(T);
    const uint4 *p4 = reinterpret_cast<const uint4 *>(kp);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < D / kPer16; ++c) {
        const uint4 u = __ldg(p4 + c);
        const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
        for (int t = 0; t < kPer16; ++t) s = fmaf(qs[c * kPer16 + t], Elem<T>::to_f(e[t]), s);
    }
    return s;
}

struct Win {
    int g, ip, s;
};
__device__ __forceinline__ Win axis_win(int i, int Lp, int K, int d) {
    Win w;
    w.g = i % d;
    w.ip = i / d;
    w.s = window_start(w.ip, group_len(Lp, d, w.g), K);
    return w;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---------------------------------------------------------------------------
// Fused forward, one warp per real query.  The query row is staged in shared
// memory (fp32).  Scores: lane t takes neighbours n = t, t + 32, ...
// (n = ty * k + tx), each a full D-channel dot product.  The row max and sum
// are warp reductions.  Weighted values: lane c accumulates channels
// c, c + 32, ... over the neighbours in order, each weight taken from its
// lane by a shuffle, so the value rows are read coalesced.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(const FwdArgs a) {
    __shared__ float qsh[kWarps][D];
    constexpr int NC = (D + 31) / 32;
    const int K = a.K, d = a.d, KK = K * K, nb = 2 * K - 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    for (int64_t idx = blockIdx.x * (int64_t)kWarps + warp; idx < a.nq; idx += nwarps) {
        int j, i, h;
        int64_t bh, b;
        split_pixel(idx, a.W, a.H, a.heads, j, i, bh, b, h);
        const T *qp = static_cast<const T *>(a.q.p) + b * a.q.sb + h * a.q.sh + i * a.q.sy + j * a.q.sx;
        for (int c = lane; c < D; c += 32) qsh[warp][c] = Elem<T>::to_f(qp[c]);
        __syncwarp();
        const Win wy = axis_win(i, a.Hp, K, d), wx = axis_win(j, a.Wp, K, d);
        // neighbour rows ty < nty and columns tx < ntx lie on the real map
        // (the rest are zero padding): wy.g + d (wy.s + ty) < H
        const int nty = min(K, (a.H - 1 - wy.g) / d - wy.s + 1), ntx = min(K, (a.W - 1 - wx.g) / d - wx.s + 1);
        const T *kb = static_cast<const T *>(a.k.p) + b * a.k.sb + h * a.k.sh;
        const T *vb = static_cast<const T *>(a.v.p) + b * a.v.sb + h * a.v.sh;
        const T *bias = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
        float sc[kMaxPerLane];
        float m = -FLT_MAX;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            sc[r] = -FLT_MAX;
            if (n < KK) {
                const int ty = n / K, tx = n - ty * K;
                const int ky = wy.g + d * (wy.s + ty), kx = wx.g + d * (wx.s + tx);
                float dot = 0.f;
                if (ty < nty && tx < ntx) dot = dot_q<T, D>(qsh[warp], kb + ky * a.k.sy + kx * a.k.sx);
                float sv = dot * a.scale;
                if (bias) sv += Elem<T>::to_f(bias[(wy.s + ty - wy.ip + K - 1) * nb + (wx.s + tx - wx.ip + K - 1)]);
                sc[r] = sv;
                m = fmaxf(m, sv);
            }
        }
        m = warp_max(m);
        float l = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            sc[r] = lane + 32 * r < KK ? __expf(sc[r] - m) : 0.f;
            l += sc[r];
        }
        const float inv = 1.f / warp_sum(l);
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            float pn = sc[r] * inv;
            if (n < KK) {
                if (a.dropout)
                    pn = dropout_keep((uint64_t)idx * KK + n, a.seed, a.offset, a.drop_thresh) ? pn * a.drop_scale : 0.f;
                if (a.attn) a.attn[idx * KK + n] = pn;
            }
            sc[r] = pn;
        }
        float acc[NC];
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) acc[jj] = 0.f;
        // lane = channel: the neighbours in order, each weight from its lane;
        // the value pointer steps along the window
        const int64_t stx = (int64_t)d * a.v.sx, sty = (int64_t)d * a.v.sy;
        const T *vrow = vb + (int64_t)(wy.g + d * wy.s) * a.v.sy + (int64_t)(wx.g + d * wx.s) * a.v.sx + lane;
        const T *vp = vrow;
        int ty = 0, tx = 0;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            if (32 * r >= KK) break;
            const int cnt = min(32, KK - 32 * r);
            for (int tl = 0; tl < cnt; ++tl) {
                const float pn = __shfl_sync(0xffffffffu, sc[r], tl);
                if (pn != 0.f && ty < nty && tx < ntx) {
#pragma unroll
                    for (int jj = 0; jj < NC; ++jj)
                        if (lane + 32 * jj < D) acc[jj] = fmaf(pn, Elem<T>::to_f(vp[32 * jj]), acc[jj]);
                }
                vp += stx;
                if (++tx == K) {
                    tx = 0;
                    ++ty;
                    vrow += sty;
                    vp = vrow;
                }
            }
        }
        T *op = static_cast<T *>(const_cast<void *>(a.out.p)) + b * a.out.sb + h * a.out.sh + i * a.out.sy +
                j * a.out.sx;
#pragma unroll
        for (int jj = 0; jj < NC; ++jj)
            if (lane + 32 * jj < D) op[lane + 32 * jj] = Elem<T>::from_f(acc[jj]);
        __syncwarp();   // the next query overwrites this warp's staged row
    }
}

// ---------------------------------------------------------------------------
// Split path (contiguous tensors).  Stage 1: one thread per (real query,
// neighbour n = ty * k + tx); a padded neighbour scores its bias alone.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) qk_rpb_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                          const T *__restrict__ rpb, float *__restrict__ attn,
                                                          int heads, int H, int W, int Hp, int Wp, int K, int d,
                                                          int64_t total, float scale) {
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
        const Win wy = axis_win(i, Hp, K, d), wx = axis_win(j, Wp, K, d);
        const int ty = n / K, tx = n % K;
        const int ky = wy.g + d * (wy.s + ty), kx = wx.g + d * (wx.s + tx);
        float s = 0.f;
        if (ky < H && kx < W) {
            const T *qp = q + (size_t)qi * D, *kp = k + ((size_t)bh * H * W + (size_t)ky * W + kx) * D;
            for (int c = 0; c < D; ++c) s = fmaf(Elem<T>::to_f(qp[c]), Elem<T>::to_f(kp[c]), s);
        }
        s *= scale;
        if (rpb) s += Elem<T>::to_f(rpb[((size_t)h * nb + (wy.s + ty - wy.ip + K - 1)) * nb + (wx.s + tx - wx.ip + K - 1)]);
        attn[idx] = s;
    }
}

// Stage 2: softmax over the last axis, one warp per query row.
__global__ void __launch_bounds__(kThreads) softmax_kernel(float *__restrict__ attn, int KK, int64_t rows) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        float *row = attn + r * KK;
        float m = -FLT_MAX;
        for (int n = lane; n < KK; n += 32) m = fmaxf(m, row[n]);
        m = warp_max(m);
        float s = 0.f;
        for (int n = lane; n < KK; n += 32) s += expf(row[n] - m);
        s = warp_sum(s);
        const float inv = 1.f / s;
        for (int n = lane; n < KK; n += 32) row[n] = expf(row[n] - m) * inv;
    }
}

// Stage 3: one thread per (real query, channel); padded neighbours carry a
// zero value.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) av_kernel(const float *__restrict__ attn, const T *__restrict__ v,
                                                      T *__restrict__ out, int H, int W, int Hp, int Wp, int K, int d,
                                                      int64_t total) {
    const int KK = K * K;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % D);
        const int64_t qi = idx / D;
        const int j = (int)(qi % W);
        const int64_t t = qi / W;
        const int i = (int)(t % H);
        const int64_t bh = t / H;
        const Win wy = axis_win(i, Hp, K, d), wx = axis_win(j, Wp, K, d);
        const float *p = attn + qi * KK;
        const T *vb = v + (size_t)bh * H * W * D + c;
        float acc = 0.f;
        for (int ty = 0; ty < K; ++ty) {
            const int ky = wy.g + d * (wy.s + ty);
            if (ky >= H) continue;
            for (int tx = 0; tx < K; ++tx) {
                const int kx = wx.g + d * (wx.s + tx);
                if (kx < W) acc = fmaf(p[ty * K + tx], Elem<T>::to_f(vb[((size_t)ky * W + kx) * D]), acc);
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

template <typename T, int D>
cudaError_t fwd_simt_impl(const FwdArgs &a, cudaStream_t st) {
    fwd_simt_kernel<T, D><<<grid_for(a.nq * 32), kThreads, 0, st>>>(a);
    note_kernel("fwd_simt_kernel");
    return cudaGetLastError();
}

template <typename T> cudaError_t fwd_simt_d(const FwdArgs &a, int D, cudaStream_t st) {
    switch (D) {
    case 16: return fwd_simt_impl<T, 16>(a, st);
    case 32: return fwd_simt_impl<T, 32>(a, st);
    case 64: return fwd_simt_impl<T, 64>(a, st);
    default: return fwd_simt_impl<T, 128>(a, st);
    }
}

template <typename T, int D>
cudaError_t qk_rpb_impl(const Problem &p, const void *q, const void *k, const void *rpb, float *attn,
                        cudaStream_t st) {
    const int64_t total = p.bh() * p.H * p.W * p.k * p.k;
    qk_rpb_kernel<T, D><<<grid_for(total), kThreads, 0, st>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(rpb), attn, p.heads, p.H, p.W,
        p.Hp(), p.Wp(), p.k, p.d, total, 1.0f / sqrtf((float)p.D));
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t av_impl(const Problem &p, const float *attn, const void *v, void *out, cudaStream_t st) {
    const int64_t total = p.bh() * p.H * p.W * D;
    av_kernel<T, D><<<grid_for(total), kThreads, 0, st>>>(attn, static_cast<const T *>(v), static_cast<T *>(out),
                                                          p.H, p.W, p.Hp(), p.Wp(), p.k, p.d, total);
    return cudaGetLastError();
}

template <typename T>
cudaError_t qk_rpb_t(const Problem &p, const void *q, const void *k, const void *rpb, float *attn, cudaStream_t st) {
    switch (p.D) {
    case 16: return qk_rpb_impl<T, 16>(p, q, k, rpb, attn, st);
    case 32: return qk_rpb_impl<T, 32>(p, q, k, rpb, attn, st);
    case 64: return qk_rpb_impl<T, 64>(p, q, k, rpb, attn, st);
    default: return qk_rpb_impl<T, 128>(p, q, k, rpb, attn, st);
    }
}

template <typename T>
cudaError_t av_t(const Problem &p, const float *attn, const void *v, void *out, cudaStream_t st) {
    switch (p.D) {
    case 16: return av_impl<T, 16>(p, attn, v, out, st);
    case 32: return av_impl<T, 32>(p, attn, v, out, st);
    case 64: return av_impl<T, 64>(p, attn, v, out, st);
    default: return av_impl<T, 128>(p, attn, v, out, st);
    }
}

}  // namespace

cudaError_t launch_forward_simt(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                const View &out, float *attn, const Dropout &drop, cudaStream_t st) {
    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.out = out;
    a.rpb = rpb;
    a.attn = attn;
    a.heads = p.heads; a.H = p.H; a.W = p.W; a.Hp = p.Hp(); a.Wp = p.Wp(); a.K = p.k; a.d = p.d;
    a.nq = p.bh() * p.H * p.W;
    a.scale = 1.0f / sqrtf((float)p.D);
    a.dropout = drop.p > 0.f;
    const double th = (double)drop.p * 4294967296.0;
    a.drop_thresh = th >= 4294967295.0 ? 0xFFFFFFFFu : (uint32_t)(th + 0.5);
    a.drop_scale = a.dropout ? 1.0f / (1.0f - drop.p) : 1.0f;
    a.seed = drop.seed;
    a.offset = drop.offset;
    switch (p.dtype) {
    case DType::F32: return fwd_simt_d<float>(a, p.D, st);
    case DType::F16: return fwd_simt_d<__half>(a, p.D, st);
    default: return fwd_simt_d<__nv_bfloat16>(a, p.D, st);
    }
}

cudaError_t launch_qk_rpb(const Problem &p, const void *q, const void *k, const void *rpb, float *attn,
                          cudaStream_t st) {
    switch (p.dtype) {
    case DType::F32: return qk_rpb_t<float>(p, q, k, rpb, attn, st);
    case DType::F16: return qk_rpb_t<__half>(p, q, k, rpb, attn, st);
    default: return qk_rpb_t<__nv_bfloat16>(p, q, k, rpb, attn, st);
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
    case DType::F32: return av_t<float>(p, attn, v, out, st);
    case DType::F16: return av_t<__half>(p, attn, v, out, st);
    default: return av_t<__nv_bfloat16>(p, attn, v, out, st);
    }
}

}  // namespace na2d
