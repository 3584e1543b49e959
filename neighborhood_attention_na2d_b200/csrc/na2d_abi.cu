// na2d_abi.cu -- the extern "C" entry points declared in include/na2d.h:
// host-side argument checks, then one launch on the caller's stream.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "../../include/na2d.h"
#include "na2d_launch.h"

namespace {

using na2d::DType;
using na2d::Dropout;
using na2d::Problem;
using na2d::View;

constexpr int64_t kMaxTotal = (int64_t)1 << 62;
constexpr int64_t kMaxPlane = ((int64_t)1 << 31) - 1;

size_t elem_size(na2d_dtype t) { return t == NA2D_F32 ? 4 : 2; }

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Checks the problem description itself.  On success fills `out` and reports
// whether the problem is empty (B or heads zero: nothing to launch).
na2d_status check_problem(const na2d_problem *p, Problem *out, bool *empty) {
    if (!p) return NA2D_ERR_NULL;
    if (p->dtype != NA2D_F32 && p->dtype != NA2D_F16 && p->dtype != NA2D_BF16) return NA2D_ERR_DTYPE;
    if (p->k < 1 || p->k > 13 || (p->k % 2) == 0) return NA2D_ERR_KERNEL;
    if (p->d < 1) return NA2D_ERR_DILATION;
    if (p->B < 0 || p->heads < 0 || p->H < 1 || p->W < 1) return NA2D_ERR_SHAPE;
    if (p->D != 16 && p->D != 32 && p->D != 64 && p->D != 128) return NA2D_ERR_SHAPE;
    // maps shorter than k*d are padded (up to k*d), which bounds the padded size
    if ((int64_t)p->k * p->d > kMaxPlane) return NA2D_ERR_SHAPE;
    const int64_t Hp = p->H > (int64_t)p->k * p->d ? p->H : (int64_t)p->k * p->d;
    const int64_t Wp = p->W > (int64_t)p->k * p->d ? p->W : (int64_t)p->k * p->d;
    const int64_t inner = (int64_t)(p->D > p->k * p->k ? p->D : p->k * p->k);
    const int64_t plane = Hp * Wp * inner;
    if (plane > kMaxPlane) return NA2D_ERR_SHAPE;
    const int64_t bh = (int64_t)p->B * p->heads;
    if (bh > 0 && bh > kMaxTotal / plane) return NA2D_ERR_SHAPE;
    *out = Problem{p->B, p->heads, p->H, p->W, p->D, p->k, p->d, static_cast<DType>(p->dtype)};
    *empty = (bh == 0);
    return NA2D_OK;
}

size_t tensor_bytes(const na2d_problem *p) {
    return (size_t)p->B * p->heads * p->H * p->W * p->D * elem_size(p->dtype);
}
size_t attn_bytes(const na2d_problem *p) { return (size_t)p->B * p->heads * p->H * p->W * p->k * p->k * 4; }
// Chunks of the batch for na2d_forward_host: at most kHostChunks of cb
// batch elements each (the last one shorter), and two workspace slots of q,
// k, v and out (one when there is a single chunk), each tensor 256-byte
// aligned within the workspace, then the bias table.
constexpr int kHostChunks = 8;
struct HostPlan {
    int cb = 0, nchunk = 0, slots = 0;
    size_t batch_bytes = 0;   // one batch element of one tensor
    size_t per = 0;           // one tensor of one slot, rounded up to 256 bytes
    size_t rpb_off = 0, ws = 0;
};
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
HostPlan host_plan(const na2d_problem *p);
size_t rpb_bytes(const na2d_problem *p) {
    return (size_t)p->heads * (2 * p->k - 1) * (2 * p->k - 1) * elem_size(p->dtype);
}

bool rpb_aligned(const na2d_problem *p, const void *rpb) {
    return !rpb || (reinterpret_cast<uintptr_t>(rpb) % elem_size(p->dtype)) == 0;
}

// A strided tensor argument: 16-byte aligned data, strides (in elements) that
// keep every pixel row 16-byte aligned, and non-negative.
na2d_status check_tensor(const na2d_problem *p, const na2d_tensor *t, View *v) {
    if (!t || !t->data) return NA2D_ERR_NULL;
    const long long st[4] = {t->stride_b, t->stride_h, t->stride_y, t->stride_x};
    const size_t e = elem_size(p->dtype);
    for (long long x : st)
        if (x < 0 || ((size_t)x * e) % 16 != 0) return NA2D_ERR_ALIGN;
    if (!aligned16(t->data)) return NA2D_ERR_ALIGN;
    *v = View{t->data, st[0], st[1], st[2], st[3]};
    return NA2D_OK;
}

// [first byte, one past the last byte] a view can touch.
void view_span(const na2d_problem *p, const View &v, uintptr_t *lo, uintptr_t *hi) {
    const size_t e = elem_size(p->dtype);
    const int64_t last = (int64_t)(p->B - 1) * v.sb + (int64_t)(p->heads - 1) * v.sh + (int64_t)(p->H - 1) * v.sy +
                         (int64_t)(p->W - 1) * v.sx + p->D;
    *lo = reinterpret_cast<uintptr_t>(v.p);
    *hi = *lo + (size_t)last * e;
}
bool spans_overlap(uintptr_t a0, uintptr_t a1, uintptr_t b0, uintptr_t b1) { return a0 < b1 && b0 < a1; }

// An output view whose pixels do not overlap one another: sorted by stride,
// each dimension steps past the whole extent of the smaller ones.
bool view_disjoint(const na2d_problem *p, const View &v) {
    int64_t st[4] = {v.sb, v.sh, v.sy, v.sx}, ex[4] = {p->B, p->heads, p->H, p->W};
    for (int i = 0; i < 4; ++i)
        for (int j = i + 1; j < 4; ++j)
            if (st[j] < st[i]) {
                int64_t t = st[i]; st[i] = st[j]; st[j] = t;
                t = ex[i]; ex[i] = ex[j]; ex[j] = t;
            }
    int64_t span = p->D;   // channels are contiguous
    for (int i = 0; i < 4; ++i) {
        if (ex[i] <= 1) continue;
        if (st[i] < span) return false;
        span = st[i] * (ex[i] - 1) + span;
    }
    return true;
}

// Two views that cannot touch a common element: their address spans are
// apart, or they have the same strides and interleave block by block (the
// q / k / v or dq / dk / dv views of one fused channels-last buffer).  The
// block of a view is its D channels, or the heads * D channels of a pixel when
// the head stride is D; the views must start at least a block apart and end
// a block before the next pixel (the smallest stride beyond the block).
bool views_disjoint(const na2d_problem *p, const View &a, const View &b) {
    uintptr_t a0, a1, b0, b1;
    view_span(p, a, &a0, &a1);
    view_span(p, b, &b0, &b1);
    if (!spans_overlap(a0, a1, b0, b1)) return true;
    if (a.sb != b.sb || a.sh != b.sh || a.sy != b.sy || a.sx != b.sx) return false;
    const int64_t e = (int64_t)elem_size(p->dtype);
    const int64_t diff = (int64_t)(reinterpret_cast<uintptr_t>(b.p) - reinterpret_cast<uintptr_t>(a.p));
    if (diff % e) return false;
    const int64_t delta = diff < 0 ? -diff / e : diff / e;
    const bool heads_packed = a.sh == p->D && p->heads > 1;
    const int64_t block = heads_packed ? (int64_t)p->heads * p->D : p->D;
    int64_t next = INT64_MAX;
    const int64_t st[4] = {a.sb, heads_packed ? INT64_MAX : a.sh, a.sy, a.sx};
    const int64_t ex[4] = {p->B, p->heads, p->H, p->W};
    for (int i = 0; i < 4; ++i)
        if (ex[i] > 1 && st[i] < next) next = st[i];
    return delta >= block && delta + block <= next;
}

// Name of the kernel the calling thread's last forward call launched.
thread_local const char *t_last_kernel = nullptr;

na2d_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return NA2D_OK;
    cudaGetLastError();   // clear a sticky launch error for the caller's next call
    return NA2D_ERR_CUDA;
}

}  // namespace

namespace na2d {
void note_kernel(const char *name) { t_last_kernel = name; }
}  // namespace na2d

namespace {

HostPlan host_plan(const na2d_problem *p) {
    HostPlan h;
    if (p->B <= 0 || p->heads <= 0) return h;
    const int n = p->B < kHostChunks ? p->B : kHostChunks;
    h.cb = (p->B + n - 1) / n;
    h.nchunk = (p->B + h.cb - 1) / h.cb;
    h.slots = h.nchunk > 1 ? 2 : 1;
    h.batch_bytes = (size_t)p->heads * p->H * p->W * p->D * elem_size(p->dtype);
    h.per = round256(h.batch_bytes * (size_t)h.cb);
    h.rpb_off = 4 * (size_t)h.slots * h.per;
    h.ws = h.rpb_off + round256(rpb_bytes(p));
    return h;
}

}  // namespace

extern "C" {

na2d_status na2d_forward(const na2d_problem *p, const void *q, const void *k, const void *v, const void *rpb,
                         void *out, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!q || !k || !v || !out) return NA2D_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !rpb_aligned(p, rpb))
        return NA2D_ERR_ALIGN;
    const size_t n = tensor_bytes(p);
    if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, rpb, rpb_bytes(p)))
        return NA2D_ERR_ALIAS;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    t_last_kernel = nullptr;
    if (na2d::tc_supported(pr)) {
        bool launched = false;
        cudaError_t e = na2d::launch_forward_umma(pr, q, k, v, rpb, out, st, &launched);
        if (e != cudaSuccess || launched) return from_cuda(e);
        e = na2d::launch_forward_ugrp(pr, q, k, v, rpb, out, st, &launched);
        if (e != cudaSuccess || launched) return from_cuda(e);
        e = na2d::launch_forward_stream(pr, View::contiguous(q, pr), View::contiguous(k, pr), View::contiguous(v, pr),
                                        rpb, View::contiguous(out, pr), st, &launched);
        if (e != cudaSuccess || launched) return from_cuda(e);
        return from_cuda(na2d::launch_forward_tc(pr, q, k, v, rpb, out, st));
    }
    return from_cuda(na2d::launch_forward_simt(pr, View::contiguous(q, pr), View::contiguous(k, pr),
                                               View::contiguous(v, pr), rpb, View::contiguous(out, pr), nullptr,
                                               Dropout{0.f, 0, 0}, st));
}

na2d_status na2d_forward_host_workspace_size(const na2d_problem *p, size_t *bytes) {
    Problem pr;
    bool empty = false;
    if (!bytes) return NA2D_ERR_NULL;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    *bytes = empty ? 0 : host_plan(p).ws;
    return NA2D_OK;
}

na2d_status na2d_forward_host(const na2d_problem *p, const void *q, const void *k, const void *v, const void *rpb,
                              void *out, void *workspace, size_t workspace_bytes, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!q || !k || !v || !out || !workspace) return NA2D_ERR_NULL;
    if (!aligned16(workspace) || !rpb_aligned(p, rpb)) return NA2D_ERR_ALIGN;
    const HostPlan h = host_plan(p);
    if (workspace_bytes < h.ws) return NA2D_ERR_SHAPE;
    const size_t n = tensor_bytes(p), nr = rpb ? rpb_bytes(p) : 0;
    if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, rpb, nr))
        return NA2D_ERR_ALIAS;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    auto slot = [&](int b, int t) { return ws + (4 * (size_t)b + (size_t)t) * h.per; };   // t: q, k, v, out
    const unsigned char *src[3] = {static_cast<const unsigned char *>(q), static_cast<const unsigned char *>(k),
                                   static_cast<const unsigned char *>(v)};
    unsigned char *dst = static_cast<unsigned char *>(out);

    // two copy streams and the events that order them with the caller's
    // stream; released at the end (the release completes with their work)
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[8] = {};   // start, in[2], comp[2], out[2], done
    cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
    for (int i = 0; i < 8 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    cudaEvent_t &e_start = ev[0], *e_in = ev + 1, *e_comp = ev + 3, *e_out = ev + 5, &e_done = ev[7];
    if (e == cudaSuccess) e = cudaEventRecord(e_start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, e_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, e_start, 0);
    if (e == cudaSuccess && rpb)
        e = cudaMemcpyAsync(ws + h.rpb_off, rpb, nr, cudaMemcpyHostToDevice, s_in);
    s = NA2D_OK;
    for (int i = 0; i < h.nchunk && e == cudaSuccess && s == NA2D_OK; ++i) {
        const int b = i % h.slots;
        const int bi = (i + 1) * h.cb <= p->B ? h.cb : p->B - i * h.cb;
        const size_t off = (size_t)i * h.cb * h.batch_bytes, bytes = (size_t)bi * h.batch_bytes;
        // the slot's inputs were read by the forward two chunks back
        if (i >= h.slots) e = cudaStreamWaitEvent(s_in, e_comp[b], 0);
        for (int t = 0; t < 3 && e == cudaSuccess; ++t)
            e = cudaMemcpyAsync(slot(b, t), src[t] + off, bytes, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess) e = cudaEventRecord(e_in[b], s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, e_in[b], 0);
        // the slot's output was copied out two chunks back
        if (e == cudaSuccess && i >= h.slots) e = cudaStreamWaitEvent(st, e_out[b], 0);
        if (e != cudaSuccess) break;
        na2d_problem pc = *p;
        pc.B = bi;
        s = na2d_forward(&pc, slot(b, 0), slot(b, 1), slot(b, 2), rpb ? ws + h.rpb_off : nullptr, slot(b, 3), st);
        if (s != NA2D_OK) break;
        e = cudaEventRecord(e_comp[b], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, e_comp[b], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(dst + off, slot(b, 3), bytes, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess) e = cudaEventRecord(e_out[b], s_out);
    }
    // the caller's stream passes the call's end only after the last copy out
    if (e == cudaSuccess && s == NA2D_OK) e = cudaEventRecord(e_done, s_out);
    if (e == cudaSuccess && s == NA2D_OK) e = cudaStreamWaitEvent(st, e_done, 0);
    for (int i = 0; i < 8; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    if (s != NA2D_OK) return s;
    return from_cuda(e);
}

na2d_status na2d_forward_ex(const na2d_problem *p, const na2d_tensor *q, const na2d_tensor *k,
                            const na2d_tensor *v, const void *rpb, const na2d_tensor *out, float *attn,
                            const na2d_dropout *drop, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    View vq, vk, vv, vo;
    if ((s = check_tensor(p, q, &vq)) != NA2D_OK || (s = check_tensor(p, k, &vk)) != NA2D_OK ||
        (s = check_tensor(p, v, &vv)) != NA2D_OK || (s = check_tensor(p, out, &vo)) != NA2D_OK)
        return s;
    if (!rpb_aligned(p, rpb) || (attn && !aligned16(attn))) return NA2D_ERR_ALIGN;
    Dropout dr{0.f, 0, 0};
    if (drop) {
        if (!(drop->p >= 0.f && drop->p < 1.f)) return NA2D_ERR_SHAPE;
        dr = Dropout{drop->p, drop->seed, drop->offset};
    }
    if (!view_disjoint(p, vo)) return NA2D_ERR_ALIAS;
    uintptr_t o0, o1, a0, a1;
    view_span(p, vo, &o0, &o1);
    const View ins[3] = {vq, vk, vv};
    for (const View &x : ins)
        if (!views_disjoint(p, vo, x)) return NA2D_ERR_ALIAS;
    if (rpb && spans_overlap(o0, o1, reinterpret_cast<uintptr_t>(rpb), reinterpret_cast<uintptr_t>(rpb) + rpb_bytes(p)))
        return NA2D_ERR_ALIAS;
    if (attn) {
        const uintptr_t t0 = reinterpret_cast<uintptr_t>(attn), t1 = t0 + attn_bytes(p);
        if (spans_overlap(o0, o1, t0, t1)) return NA2D_ERR_ALIAS;
        for (const View &x : ins) {
            view_span(p, x, &a0, &a1);
            if (spans_overlap(t0, t1, a0, a1)) return NA2D_ERR_ALIAS;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    t_last_kernel = nullptr;
    // contiguous tensors without the optional parts take na2d_forward's kernels
    if (!attn && dr.p == 0.f && vq.is_contiguous(pr) && vk.is_contiguous(pr) && vv.is_contiguous(pr) &&
        vo.is_contiguous(pr))
        return na2d_forward(p, q->data, k->data, v->data, rpb, out->data, stream);
    // strided views without the optional parts: the tensor-core kernels that
    // read rows with strides
    if (!attn && dr.p == 0.f && na2d::tc_supported(pr)) {
        bool launched = false;
        cudaError_t e = na2d::launch_forward_stream(pr, vq, vk, vv, rpb, vo, st, &launched);
        if (e != cudaSuccess || launched) return from_cuda(e);
    }
    return from_cuda(na2d::launch_forward_simt(pr, vq, vk, vv, rpb, vo, attn, dr, st));
}

na2d_status na2d_qk_rpb(const na2d_problem *p, const void *q, const void *k, const void *rpb, float *attn,
                        void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!q || !k || !attn) return NA2D_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(attn) || !rpb_aligned(p, rpb)) return NA2D_ERR_ALIGN;
    const size_t n = tensor_bytes(p), na = attn_bytes(p);
    if (overlap(attn, na, q, n) || overlap(attn, na, k, n) || overlap(attn, na, rpb, rpb_bytes(p)))
        return NA2D_ERR_ALIAS;
    return from_cuda(na2d::launch_qk_rpb(pr, q, k, rpb, attn, static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_softmax(const na2d_problem *p, float *attn, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!attn) return NA2D_ERR_NULL;
    if (!aligned16(attn)) return NA2D_ERR_ALIGN;
    return from_cuda(na2d::launch_softmax(pr, attn, static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_av(const na2d_problem *p, const float *attn, const void *v, void *out, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!attn || !v || !out) return NA2D_ERR_NULL;
    if (!aligned16(attn) || !aligned16(v) || !aligned16(out)) return NA2D_ERR_ALIGN;
    const size_t n = tensor_bytes(p);
    if (overlap(out, n, v, n) || overlap(out, n, attn, attn_bytes(p))) return NA2D_ERR_ALIAS;
    return from_cuda(na2d::launch_av(pr, attn, v, out, static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_backward_workspace_size(const na2d_problem *p, size_t *bytes) {
    Problem pr;
    bool empty = false;
    if (!bytes) return NA2D_ERR_NULL;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    *bytes = empty ? 0 : na2d::backward_workspace_bytes(pr);
    return NA2D_OK;
}

na2d_status na2d_backward(const na2d_problem *p, const void *q, const void *k, const void *v, const void *rpb,
                          const void *dout, void *dq, void *dk, void *dv, void *drpb, void *workspace,
                          size_t workspace_bytes, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !workspace) return NA2D_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(workspace) || !rpb_aligned(p, rpb) || !rpb_aligned(p, drpb))
        return NA2D_ERR_ALIGN;
    const size_t need = na2d::backward_workspace_bytes(pr);
    if (workspace_bytes < need) return NA2D_ERR_SHAPE;
    const size_t n = tensor_bytes(p), nr = rpb_bytes(p);
    const void *ins[5] = {q, k, v, dout, rpb};
    const size_t in_n[5] = {n, n, n, n, nr};
    const void *outs[5] = {dq, dk, dv, drpb, workspace};
    const size_t out_n[5] = {n, n, n, nr, need};
    for (int o = 0; o < 5; ++o) {
        for (int i = 0; i < 5; ++i)
            if (overlap(outs[o], out_n[o], ins[i], in_n[i])) return NA2D_ERR_ALIAS;
        for (int o2 = o + 1; o2 < 5; ++o2)
            if (overlap(outs[o], out_n[o], outs[o2], out_n[o2])) return NA2D_ERR_ALIAS;
    }
    t_last_kernel = nullptr;
    return from_cuda(na2d::launch_backward(pr, q, k, v, rpb, dout, dq, dk, dv, drpb, workspace,
                                           static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_backward_ex(const na2d_problem *p, const na2d_tensor *q, const na2d_tensor *k,
                             const na2d_tensor *v, const void *rpb, const na2d_tensor *dout, const na2d_tensor *dq,
                             const na2d_tensor *dk, const na2d_tensor *dv, void *drpb, const na2d_dropout *drop,
                             void *workspace, size_t workspace_bytes, void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    View vq, vk, vv, vg, vdq, vdk, vdv;
    if ((s = check_tensor(p, q, &vq)) != NA2D_OK || (s = check_tensor(p, k, &vk)) != NA2D_OK ||
        (s = check_tensor(p, v, &vv)) != NA2D_OK || (s = check_tensor(p, dout, &vg)) != NA2D_OK ||
        (s = check_tensor(p, dq, &vdq)) != NA2D_OK || (s = check_tensor(p, dk, &vdk)) != NA2D_OK ||
        (s = check_tensor(p, dv, &vdv)) != NA2D_OK)
        return s;
    if (!workspace) return NA2D_ERR_NULL;
    if (!aligned16(workspace) || !rpb_aligned(p, rpb) || !rpb_aligned(p, drpb)) return NA2D_ERR_ALIGN;
    const size_t need = na2d::backward_workspace_bytes(pr);
    if (workspace_bytes < need) return NA2D_ERR_SHAPE;
    Dropout dr{0.f, 0, 0};
    if (drop) {
        if (!(drop->p >= 0.f && drop->p < 1.f)) return NA2D_ERR_SHAPE;
        dr = Dropout{drop->p, drop->seed, drop->offset};
    }
    const View outs_v[3] = {vdq, vdk, vdv};
    const View ins_v[4] = {vq, vk, vv, vg};
    for (int o = 0; o < 3; ++o) {
        if (!view_disjoint(p, outs_v[o])) return NA2D_ERR_ALIAS;
        for (const View &x : ins_v)
            if (!views_disjoint(p, outs_v[o], x)) return NA2D_ERR_ALIAS;
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (!views_disjoint(p, outs_v[o], outs_v[o2])) return NA2D_ERR_ALIAS;
    }
    // the workspace and drpb against every tensor and each other
    uintptr_t lo[2] = {reinterpret_cast<uintptr_t>(workspace), reinterpret_cast<uintptr_t>(drpb)};
    uintptr_t hi[2] = {lo[0] + need, drpb ? lo[1] + rpb_bytes(p) : lo[1]};
    for (int o = 0; o < 2; ++o) {
        if (lo[o] == hi[o]) continue;
        for (const View &x : ins_v) {
            uintptr_t a0, a1;
            view_span(p, x, &a0, &a1);
            if (spans_overlap(lo[o], hi[o], a0, a1)) return NA2D_ERR_ALIAS;
        }
        for (const View &x : outs_v) {
            uintptr_t a0, a1;
            view_span(p, x, &a0, &a1);
            if (spans_overlap(lo[o], hi[o], a0, a1)) return NA2D_ERR_ALIAS;
        }
        if (rpb && spans_overlap(lo[o], hi[o], reinterpret_cast<uintptr_t>(rpb),
                                 reinterpret_cast<uintptr_t>(rpb) + rpb_bytes(p)))
            return NA2D_ERR_ALIAS;
    }
    if (lo[1] != hi[1] && spans_overlap(lo[0], hi[0], lo[1], hi[1])) return NA2D_ERR_ALIAS;
    t_last_kernel = nullptr;
    return from_cuda(na2d::launch_backward_views(pr, vq, vk, vv, rpb, vg, vdq, vdk, vdv, drpb, dr, workspace,
                                                 static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_backward_noalloc(const na2d_problem *p, const void *q, const void *k, const void *v,
                                  const void *rpb, const void *dout, void *dq, void *dk, void *dv, void *drpb,
                                  void *stream) {
    Problem pr;
    bool empty = false;
    na2d_status s = check_problem(p, &pr, &empty);
    if (s != NA2D_OK) return s;
    if (empty) return NA2D_OK;
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return NA2D_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !rpb_aligned(p, rpb) || !rpb_aligned(p, drpb))
        return NA2D_ERR_ALIGN;
    // the built-in scratch has a fixed size: larger problems are refused here
    if (na2d::backward_workspace_bytes(pr) > na2d::noalloc_scratch_bytes()) return NA2D_ERR_SHAPE;
    const size_t n = tensor_bytes(p), nr = rpb_bytes(p);
    const void *ins[5] = {q, k, v, dout, rpb};
    const size_t in_n[5] = {n, n, n, n, nr};
    void *outs[4] = {dq, dk, dv, drpb};
    const size_t out_n[4] = {n, n, n, nr};
    for (int o = 0; o < 4; ++o) {
        for (int i = 0; i < 5; ++i)
            if (overlap(outs[o], out_n[o], ins[i], in_n[i])) return NA2D_ERR_ALIAS;
        for (int o2 = o + 1; o2 < 4; ++o2)
            if (overlap(outs[o], out_n[o], outs[o2], out_n[o2])) return NA2D_ERR_ALIAS;
    }
    t_last_kernel = nullptr;
    return from_cuda(na2d::launch_backward_noalloc(pr, q, k, v, rpb, dout, dq, dk, dv, drpb,
                                                   static_cast<cudaStream_t>(stream)));
}

na2d_status na2d_device_faults(unsigned int *count, void *stream) {
    if (!count) return NA2D_ERR_NULL;
    unsigned int a = 0, b = 0, c = 0, g = 0;
    cudaError_t e = na2d::read_device_faults(&a, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = na2d::read_stream_faults(&b, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = na2d::read_umma_faults(&c, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = na2d::read_ugrp_faults(&g, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e);
    *count = a + b + c + g;
    return NA2D_OK;
}

const char *na2d_status_str(na2d_status s) {
    switch (s) {
    case NA2D_OK: return "ok";
    case NA2D_ERR_NULL: return "null pointer";
    case NA2D_ERR_DTYPE: return "unsupported dtype";
    case NA2D_ERR_SHAPE: return "unsupported shape";
    case NA2D_ERR_KERNEL: return "unsupported kernel size";
    case NA2D_ERR_DILATION: return "unsupported dilation";
    case NA2D_ERR_ALIGN: return "misaligned pointer";
    case NA2D_ERR_ALIAS: return "output overlaps an input";
    case NA2D_ERR_CUDA: return "CUDA error";
    case NA2D_ERR_INTERNAL: return "internal error";
    }
    return "unknown status";
}

int na2d_version(void) { return 200; }

const char *na2d_last_kernel(void) { return t_last_kernel; }

void na2d_debug_set_wait_limit(long long sm_clocks) {
    na2d::set_stream_wait_limit(sm_clocks);
    na2d::set_ugrp_wait_limit(sm_clocks);
}

}  // extern "C"
