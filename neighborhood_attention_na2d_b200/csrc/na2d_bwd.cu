// na2d_bwd.cu -- backward of the fused NA2D forward: dq, dk, dv and the
// relative-position-bias gradient.
//
// The layer is trained end to end ("Dilated Neighborhood Attention
// Transformer", gitcode DiNAT article, section "微调示例：加载预训练权重继续训练";
// the HF tests described under "源码与测试导览" run forward and backward), so
// its gradients are the chain rule through scores -> softmax -> weighted sum.
// For a query with scores s_n, weights p_n and output gradient g:
//     dp_n = g . v_n,   delta = sum_n p_n dp_n,   ds_n = p_n (dp_n - delta),
//     dq  = sum_n ds_n k_n / sqrt(D),   dk_n += ds_n q / sqrt(D),
//     dv_n += p_n g,    drpb[h, key' - i' + k - 1] += ds_n.
//
// Three passes on the caller's stream (fp32 arithmetic throughout):
//  1. bwd_query_kernel, one warp per query: recomputes the scores and the
//     softmax (lane t holds neighbours t, t + 32, ...), writes dq, and stores
//     the query's log-sum-exp and delta in the workspace; a block covers
//     queries of one (batch, head) image and sums its bias gradient in shared
//     memory before one atomic add per table entry into the workspace's fp32
//     table.
//  2. bwd_key_kernel, one warp per key (lane = channel): walks the key's
//     inverse neighbourhood (the queries whose clamped window holds it: per
//     axis a contiguous range of group positions, up to k + k/2 long at the
//     edges), recomputes p = exp(s - lse) and ds from the stored statistics
//     and accumulates dk and dv in registers; no atomics.
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

constexpr int kD = 32;                    // head dim
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kQPB = 128;                 // queries per block in the query pass
constexpr int kMaxPerLane = (13 * 13 + 31) / 32;
constexpr int kMaxTab = 25 * 25;          // (2k-1)^2 for k <= 13

template <typename T> __device__ __forceinline__ void load_row(const T *p, float (&x)[kD]) {
    constexpr int kPer16 = 16 / sizeof(T);
    const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int c = 0; c < kD / kPer16; ++c) {
        uint4 u = __ldg(p4 + c);
        const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
        for (int t = 0; t < kPer16; ++t) x[c * kPer16 + t] = Elem<T>::to_f(e[t]);
    }
}

template <typename T> __device__ __forceinline__ float dot_row(const float (&a)[kD], const T *p) {
    float b[kD];
    load_row<T>(p, b);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kD; ++c) s = fmaf(a[c], b[c], s);
    return s;
}

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

struct BwdArgs {
    const void *q, *k, *v, *rpb, *dout;
    void *dq, *dk, *dv, *drpb;
    float *lse, *delta, *tab;    // workspace
    int heads, H, W, K, d;
    int64_t nq;                  // B * heads * H * W
    int qblocks;                 // query-pass blocks per image
    float scale;                 // 1 / sqrt(D)
};

// ---------------------------------------------------------------------------
__global__ void bwd_zero_kernel(float *tab, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) tab[i] = 0.f;
}

// ---------------------------------------------------------------------------
// Pass 1: block (image bh, chunk) takes queries [chunk * kQPB, +kQPB) of
// image bh, one warp per query at a time.
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_query_kernel(const BwdArgs a) {
    __shared__ float bins[kMaxTab];
    const int K = a.K, d = a.d, H = a.H, W = a.W, KK = K * K, nb = 2 * K - 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = blockIdx.x / a.qblocks;
    const int chunk = (int)(blockIdx.x - bh * a.qblocks);
    const int h = (int)(bh % a.heads);
    for (int i = threadIdx.x; i < nb * nb; i += blockDim.x) bins[i] = 0.f;
    __syncthreads();
    const T *q = static_cast<const T *>(a.q), *k = static_cast<const T *>(a.k), *v = static_cast<const T *>(a.v);
    const T *g = static_cast<const T *>(a.dout);
    const T *bias = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
    const size_t plane = (size_t)bh * H * W;
    const int q_end = min(H * W, (chunk + 1) * kQPB);
    for (int qi = chunk * kQPB + warp; qi < q_end; qi += kWarps) {
        const int i = qi / W, j = qi - (qi / W) * W;
        const int gy = i % d, iy = i / d, sy = window_start(iy, group_len(H, d, gy), K);
        const int gx = j % d, ix = j / d, sx = window_start(ix, group_len(W, d, gx), K);
        float qf[kD], gf[kD];
        load_row<T>(q + (plane + qi) * kD, qf);
        load_row<T>(g + (plane + qi) * kD, gf);
        float s[kMaxPerLane], dp[kMaxPerLane];
        float m = -FLT_MAX;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            const int n = lane + 32 * r;
            s[r] = -FLT_MAX;
            dp[r] = 0.f;
            if (n < KK) {
                const int ty = n / K, tx = n - ty * K;
                const size_t key = plane + (size_t)(gy + d * (sy + ty)) * W + (gx + d * (sx + tx));
                float sv = dot_row<T>(qf, k + key * kD) * a.scale;
                if (bias) sv += Elem<T>::to_f(bias[(sy + ty - iy + K - 1) * nb + (sx + tx - ix + K - 1)]);
                s[r] = sv;
                dp[r] = dot_row<T>(gf, v + key * kD);
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
            if (n < KK) {
                const int ty = n / K, tx = n - ty * K;
                atomicAdd(&bins[(sy + ty - iy + K - 1) * nb + (sx + tx - ix + K - 1)], dp[r]);
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxPerLane; ++r) {
            if (32 * r >= KK) break;
            const int cnt = min(32, KK - 32 * r);
            for (int tl = 0; tl < cnt; ++tl) {
                const int n = 32 * r + tl;
                const float dsn = __shfl_sync(0xffffffffu, dp[r], tl);
                const int ty = n / K, tx = n - ty * K;
                const size_t key = plane + (size_t)(gy + d * (sy + ty)) * W + (gx + d * (sx + tx));
                acc = fmaf(dsn, Elem<T>::to_f(k[key * kD + lane]), acc);
            }
        }
        static_cast<T *>(a.dq)[(plane + qi) * kD + lane] = Elem<T>::from_f(acc * a.scale);
        if (lane == 0) {
            a.lse[plane + qi] = m + __logf(l);
            a.delta[plane + qi] = delta;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb * nb; i += blockDim.x)
        if (bins[i] != 0.f) atomicAdd(&a.tab[(size_t)h * nb * nb + i], bins[i]);
}

// ---------------------------------------------------------------------------
// The group positions of the queries whose clamped window holds key position
// jp (group coordinates, group length Lg): a contiguous range [lo, hi].
__device__ __forceinline__ void inverse_range(int jp, int Lg, int K, int *lo, int *hi) {
    int a = INT32_MAX, b = -1;
    for (int ip = max(0, jp - K + 1); ip <= min(Lg - 1, jp + K - 1); ++ip) {
        const int s = window_start(ip, Lg, K);
        if (s <= jp && jp < s + K) {
            a = min(a, ip);
            b = ip;
        }
    }
    *lo = a;
    *hi = b;
}

// Pass 2: one warp per key pixel (b, head, y, x), lane = channel.
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_key_kernel(const BwdArgs a) {
    const int K = a.K, d = a.d, H = a.H, W = a.W, nb = 2 * K - 1;
    const int lane = threadIdx.x & 31;
    const T *q = static_cast<const T *>(a.q), *k = static_cast<const T *>(a.k), *v = static_cast<const T *>(a.v);
    const T *g = static_cast<const T *>(a.dout);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t idx = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; idx < a.nq; idx += nwarps) {
        const int x = (int)(idx % W);
        const int64_t t = idx / W;
        const int y = (int)(t % H);
        const int64_t bh = t / H;
        const int h = (int)(bh % a.heads);
        const T *bias = a.rpb ? static_cast<const T *>(a.rpb) + (size_t)h * nb * nb : nullptr;
        const size_t plane = (size_t)bh * H * W;
        const int gy = y % d, jy = y / d, Lgy = group_len(H, d, gy);
        const int gx = x % d, jx = x / d, Lgx = group_len(W, d, gx);
        int ylo, yhi, xlo, xhi;
        inverse_range(jy, Lgy, K, &ylo, &yhi);
        inverse_range(jx, Lgx, K, &xlo, &xhi);
        const float kc = Elem<T>::to_f(k[idx * kD + lane]), vc = Elem<T>::to_f(v[idx * kD + lane]);
        float dk = 0.f, dv = 0.f;
        for (int iy = ylo; iy <= yhi; ++iy) {
            const int qy = gy + d * iy;
            const int by = jy - iy + K - 1;
            for (int ix = xlo; ix <= xhi; ++ix) {
                const size_t qi = plane + (size_t)qy * W + (gx + d * ix);
                const float qc = Elem<T>::to_f(q[qi * kD + lane]), gc = Elem<T>::to_f(g[qi * kD + lane]);
                float sdot = qc * kc, pdot = gc * vc;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
                    pdot += __shfl_xor_sync(0xffffffffu, pdot, o);
                }
                float sv = sdot * a.scale;
                if (bias) sv += Elem<T>::to_f(bias[by * nb + (jx - ix + K - 1)]);
                const float p = __expf(sv - a.lse[qi]);
                const float ds = p * (pdot - a.delta[qi]);
                dv = fmaf(p, gc, dv);
                dk = fmaf(ds, qc, dk);
            }
        }
        static_cast<T *>(a.dk)[idx * kD + lane] = Elem<T>::from_f(dk * a.scale);
        static_cast<T *>(a.dv)[idx * kD + lane] = Elem<T>::from_f(dv);
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

template <typename T> cudaError_t launch_bwd_t(const BwdArgs &a, int64_t bh, cudaStream_t st) {
    const int ntab = a.heads * (2 * a.K - 1) * (2 * a.K - 1);
    bwd_zero_kernel<<<grid_for(ntab), kThreads, 0, st>>>(a.tab, ntab);
    bwd_query_kernel<T><<<(unsigned)(bh * a.qblocks), kThreads, 0, st>>>(a);
    bwd_key_kernel<T><<<grid_for(a.nq * 32), kThreads, 0, st>>>(a);
    if (a.drpb) bwd_rpb_kernel<T><<<grid_for(ntab), kThreads, 0, st>>>(a.tab, static_cast<T *>(a.drpb), ntab);
    note_kernel("bwd_query_kernel+bwd_key_kernel");
    return cudaGetLastError();
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

cudaError_t launch_backward(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                            const void *dout, void *dq, void *dk, void *dv, void *drpb, void *workspace,
                            cudaStream_t st) {
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.rpb = rpb; a.dout = dout;
    a.dq = dq; a.dk = dk; a.dv = dv; a.drpb = drpb;
    a.nq = p.bh() * p.H * p.W;
    float *ws = static_cast<float *>(workspace);
    a.lse = ws;
    a.delta = ws + a.nq;
    a.tab = ws + 2 * a.nq;
    a.heads = p.heads; a.H = p.H; a.W = p.W; a.K = p.k; a.d = p.d;
    a.qblocks = (p.H * p.W + kQPB - 1) / kQPB;
    a.scale = 1.0f / sqrtf((float)p.D);
    if (p.bh() * a.qblocks >= INT32_MAX) return cudaErrorInvalidConfiguration;
    switch (p.dtype) {
    case DType::F32: return launch_bwd_t<float>(a, p.bh(), st);
    case DType::F16: return launch_bwd_t<__half>(a, p.bh(), st);
    default: return launch_bwd_t<__nv_bfloat16>(a, p.bh(), st);
    }
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
