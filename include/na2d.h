/*
 * na2d.h -- C ABI of libna2d: 2D (dilated) neighborhood attention (NA / DiNA)
 * forward for NVIDIA B200 (sm_100a).
 *
 * The operation (web pages on NAT / DiNAT):
 *   - "Neighborhood Attention Transformer" (README mirror, figure caption under
 *     the abstract): each query pixel attends to its nearest k x k
 *     neighbourhood; at the image edges the window stays inside the image;
 *     with the window as large as the image this is plain dot-product self
 *     attention.
 *   - "Dilated Neighborhood Attention Transformer" (HF docs, overview; gitcode
 *     DiNAT article, section "DiNAT 的核心思想"): DiNA takes every d-th pixel,
 *     keeping k*k keys per query; the layer is
 *         scores = natten2dqkrpb(q, k, rpb, kernel_size, dilation)
 *         probs  = softmax(scores, dim=-1)
 *         out    = natten2dav(probs, v, kernel_size, dilation)
 *     which this library exports as na2d_qk_rpb, na2d_softmax and na2d_av, and
 *     fused (no k*k tensor in memory) as na2d_forward.
 *
 * Window rule (NATTEN clamp rule), per axis, for coordinate i on an axis of
 * length L, r = k / 2:
 *     g = i mod d, i' = i / d, Lg = ceil((L - g) / d),
 *     s' = clamp(i' - r, 0, Lg - k), keys g + d * (s' + t), t = 0 .. k-1.
 * Score of key (ty, tx):
 *     q . key / sqrt(D) + rpb[h, s'_y + ty - i'_y + k - 1, s'_x + tx - i'_x + k - 1]
 * The neighbour index in the k*k axis of the split path is n = ty * k + tx.
 *
 * Layouts (all row-major, contiguous, innermost last):
 *     q, k, v, out : [B, heads, H, W, D] in the problem's dtype
 *     rpb          : [heads, 2k-1, 2k-1] in the problem's dtype, or NULL for
 *                    a zero bias
 *     attn         : [B, heads, H, W, k*k] fp32 (split path only)
 *
 * Ownership and threading: every buffer is a DEVICE pointer owned by the
 * caller (na2d_forward_host alone takes host buffers and a device
 * workspace).  The library allocates no memory and keeps no per-call state; calls
 * are asynchronous on `stream` (a cudaStream_t; NULL means the legacy default
 * stream) and never synchronise the host.  Calls from several host threads
 * are safe.  Outputs must not overlap inputs.
 *
 * Errors: every argument check runs on the host before any launch; a failing
 * check returns its status and launches nothing.  A failed launch returns
 * NA2D_ERR_CUDA (the CUDA error is cleared with cudaGetLastError).  Nothing
 * in the library aborts, traps or prints.
 *
 * Supported set: dtype f32 / f16 / bf16; D in {16, 32, 64, 128}; odd k in
 * [1, 13]; d >= 1; H, W >= 1; B, heads >= 0 (an empty problem returns NA2D_OK
 * without a launch); with Hp = max(H, k*d), Wp = max(W, k*d):
 * B*heads*Hp*Wp*max(D, k*k) < 2^62 and Hp*Wp*max(D, k*k) < 2^31; tensor
 * pointers 16-byte aligned (rpb: element aligned).  Arithmetic: fp32
 * accumulation for every dtype; f16 / bf16 outputs are rounded to nearest
 * even.
 *
 * Maps shorter than k*d: the HF DiNAT layer pads its feature map at the
 * bottom and right up to kernel_size * dilation before attention and crops
 * afterwards ("maybe_pad"; "Dilated Neighborhood Attention Transformer", HF
 * docs, DinatModel, and the gitcode DiNAT article's source walkthrough).  At
 * this boundary the padded pixels are zero vectors of q, k and v: the window
 * rule runs on the padded size Hp x Wp, a padded key scores its bias alone
 * and carries a zero value, and only the H x W real queries are computed and
 * written.  (The layer pads before its q/k/v projection, so its padded
 * pixels hold the projection biases; a caller that wants exactly that pads
 * its hidden states itself, which makes H, W >= k*d here.)
 *
 * Fast paths: f16 / bf16 with D = 32 and H, W >= k*d run on tensor-core
 * kernels; every other problem runs on the CUDA-core kernel.
 */
#ifndef NA2D_H
#define NA2D_H

#if defined(__GNUC__)
#define NA2D_API __attribute__((visibility("default")))
#else
#define NA2D_API
#endif

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NA2D_OK = 0,
    NA2D_ERR_NULL = 1,      /* a required pointer (problem, q, k, v, out, attn) is NULL */
    NA2D_ERR_DTYPE = 2,     /* dtype is not one of na2d_dtype */
    NA2D_ERR_SHAPE = 3,     /* negative B/heads, H or W < 1, D not 16/32/64/128, a
                               size limit exceeded, a workspace too small, or a
                               dropout probability outside [0, 1) */
    NA2D_ERR_KERNEL = 4,    /* k even, < 1 or > 13 */
    NA2D_ERR_DILATION = 5,  /* d < 1 */
    NA2D_ERR_ALIGN = 6,     /* a tensor not 16-byte aligned (or a stride not a multiple of 16
                               bytes), rpb not element aligned */
    NA2D_ERR_ALIAS = 7,     /* an output buffer overlaps an input buffer */
    NA2D_ERR_CUDA = 8,      /* a CUDA runtime call or kernel launch failed */
    NA2D_ERR_INTERNAL = 9   /* an internal consistency check failed */
} na2d_status;

typedef enum { NA2D_F32 = 0, NA2D_F16 = 1, NA2D_BF16 = 2 } na2d_dtype;

/* One problem.  The softmax scale is fixed at 1/sqrt(D). */
typedef struct {
    int B;            /* batch */
    int heads;        /* attention heads */
    int H, W;         /* feature map height and width */
    int D;            /* head dim: 16, 32, 64 or 128 */
    int k;            /* kernel size: odd, 1..13 */
    int d;            /* dilation: >= 1 */
    na2d_dtype dtype; /* element type of q, k, v, rpb and out */
} na2d_problem;

/* Scores (natten2dqkrpb): attn[b,h,i,j,n] = q.key_n / sqrt(D) + rpb bias, fp32.
 * q, k: [B,heads,H,W,D]; rpb: [heads,2k-1,2k-1] or NULL; attn: [B,heads,H,W,k*k]. */
NA2D_API na2d_status na2d_qk_rpb(const na2d_problem *p, const void *q, const void *k, const void *rpb,
                        float *attn, void *stream);

/* Softmax over the last (k*k) axis of attn, in place (dim=-1 softmax). */
NA2D_API na2d_status na2d_softmax(const na2d_problem *p, float *attn, void *stream);

/* Weighted sum (natten2dav): out[b,h,i,j,:] = sum_n attn[b,h,i,j,n] * v[key_n].
 * attn: [B,heads,H,W,k*k] fp32; v, out: [B,heads,H,W,D] in the problem's dtype. */
NA2D_API na2d_status na2d_av(const na2d_problem *p, const float *attn, const void *v, void *out,
                    void *stream);

/* Fused forward: out = softmax(q.key/sqrt(D) + rpb) . v over each query's k*k
 * (dilated) window, in one kernel; no k*k tensor is written to memory. */
NA2D_API na2d_status na2d_forward(const na2d_problem *p, const void *q, const void *k, const void *v,
                         const void *rpb, void *out, void *stream);

/* Bytes of device workspace na2d_forward_host needs for problem p (two chunk
 * slots of q, k, v and out, plus the bias table; see na2d_forward_host).
 * Writes 0 for an empty problem.  Host-only; launches nothing. */
NA2D_API na2d_status na2d_forward_host_workspace_size(const na2d_problem *p, size_t *bytes);

/* na2d_forward on HOST buffers: the call a program makes when its tensors
 * live in host memory.  q, k, v, out: [B,heads,H,W,D] and rpb
 * [heads,2k-1,2k-1] (or NULL) in host memory, in the problem's dtype; they
 * should be page-locked (cudaHostAlloc / pinned), or the copies run
 * synchronously.  The batch is cut into at most 8 chunks of equal size (the
 * last one shorter); chunk i is copied host -> device into workspace slot
 * i % 2, computed by na2d_forward on the caller's stream, and copied back,
 * so that the copy in of one chunk, the forward of the next and the copy
 * out of a third overlap (two copy directions and the kernels run at once).
 * workspace: a caller-owned device buffer of at least
 * na2d_forward_host_workspace_size() bytes, 16-byte aligned (256-byte
 * aligned lets the kernels use their widest stores), scratch afterwards.
 * Ordering: the call's work starts after the work already queued on
 * `stream`, and everything it does, the last copy into out included, is
 * complete when `stream` reaches the point after the call; out must not be
 * read (nor q, k, v, rpb written) by the host before then.  The call creates
 * two CUDA streams and a few events for its copies and releases them before
 * it returns (the release finishes when their work does); it allocates no
 * memory and does not synchronise the host.  Errors: the argument checks of
 * na2d_forward, with out not overlapping an input (NA2D_ERR_ALIAS), a NULL or
 * too small workspace (NA2D_ERR_NULL / NA2D_ERR_SHAPE) and a misaligned one
 * (NA2D_ERR_ALIGN), all before any copy; NA2D_ERR_CUDA if a CUDA call fails,
 * after which out is unspecified. */
NA2D_API na2d_status na2d_forward_host(const na2d_problem *p, const void *q, const void *k, const void *v,
                                       const void *rpb, void *out, void *workspace, size_t workspace_bytes,
                                       void *stream);

/* Bytes of device workspace na2d_backward needs for problem p: fp32
 * log-sum-exp and delta per query and head (8 bytes each pair) plus an fp32
 * bias-gradient table of heads * (2k-1)^2 floats.  Writes 0 for an empty
 * problem.  Host-only; launches nothing. */
NA2D_API na2d_status na2d_backward_workspace_size(const na2d_problem *p, size_t *bytes);

/* Backward of na2d_forward.  The layer is trained end to end ("Dilated
 * Neighborhood Attention Transformer", gitcode DiNAT article, section
 * "微调示例：加载预训练权重继续训练"), and its gradients are the chain rule through
 * scores -> softmax -> weighted sum: for a query with weights p_n and output
 * gradient g, dp_n = g . v_n, ds_n = p_n (dp_n - sum_m p_m dp_m),
 *     dq = sum_n ds_n key_n / sqrt(D),  dk_n += ds_n q / sqrt(D),
 *     dv_n += p_n g,  drpb[h, key' - i' + k - 1 (both axes)] += ds_n.
 * Inputs: q, k, v, dout [B,heads,H,W,D] and rpb [heads,2k-1,2k-1] (or NULL
 * for a zero bias), in the problem's dtype.  Outputs: dq, dk, dv
 * [B,heads,H,W,D] and drpb [heads,2k-1,2k-1] (or NULL if not wanted), in the
 * problem's dtype, fully overwritten.  workspace: a caller-owned device buffer
 * of at least na2d_backward_workspace_size() bytes, 16-byte aligned, used as
 * scratch (its contents are undefined afterwards).  Same supported set,
 * ownership, threading and error rules as na2d_forward; no output or the
 * workspace may overlap an input or another output (NA2D_ERR_ALIAS); a
 * workspace smaller than required returns NA2D_ERR_SHAPE.  fp32 arithmetic;
 * the bias gradient is summed in fp32 with atomics, so its last bits may vary
 * from run to run. */
NA2D_API na2d_status na2d_backward(const na2d_problem *p, const void *q, const void *k, const void *v,
                                   const void *rpb, const void *dout, void *dq, void *dk, void *dv, void *drpb,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* na2d_backward without a workspace argument, for callers that cannot
 * allocate device memory: code whose host framework owns every device
 * allocation and allows none during execution, or a loop that cannot accept
 * the device-wide synchronisation a cudaMalloc / cudaFree may cause.  The
 * papers have no counterpart to this call; it exists only for such callers.
 * It computes exactly what na2d_backward computes, but its scratch is a
 * 16 MiB array built into the library, which every GPU that loads the
 * library holds until the process exits.  Problems whose workspace
 * (na2d_backward_workspace_size: 8 bytes per query and head plus
 * 4 * heads * (2k-1)^2 bytes) exceeds 16 MiB are refused with NA2D_ERR_SHAPE
 * before any launch.  The call allocates nothing.  Its first call on a device
 * looks up the array's device address with that device current (a host-side
 * step done once per device); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents (the
 * call clears what must start at zero), so calls whose work can overlap on
 * the GPU, e.g. on two streams without ordering between them, race on it and
 * give wrong results.  Arguments, outputs and errors otherwise as for
 * na2d_backward. */
NA2D_API na2d_status na2d_backward_noalloc(const na2d_problem *p, const void *q, const void *k, const void *v,
                                           const void *rpb, const void *dout, void *dq, void *dk, void *dv,
                                           void *drpb, void *stream);

/* A [B, heads, H, W, D] tensor given by element strides, channels contiguous
 * (element (b, h, y, x, c) at data + b*stride_b + h*stride_h + y*stride_y +
 * x*stride_x + c).  It covers the channels-last layouts of the model: the
 * hidden states are (b, h, w, channels) ("Dilated Neighborhood Attention
 * Transformer", gitcode DiNAT article, "作为骨干网络（Backbone）使用"), and the
 * fused q/k/v projection output (B, H, W, 3, heads, D) is read in place as
 * three such views (strides 3*heads*D per pixel, D per head, offsets 0,
 * heads*D and 2*heads*D).  data is 16-byte aligned and every stride is
 * non-negative with stride * element size a multiple of 16 bytes
 * (NA2D_ERR_ALIGN otherwise). */
typedef struct {
    void *data;
    long long stride_b, stride_h, stride_y, stride_x;
} na2d_tensor;

/* Attention dropout between the softmax and the weighted sum, as in the
 * layer (gitcode DiNAT article, "DiNAT 的核心思想": the weights pass through
 * dropout before natten2dav).  Weight number e (its linear index in the
 * [B, heads, H, W, k*k] weight tensor) is kept when word e % 4 of
 * Philox4x32-10(counter = (e/4 low 32 bits, e/4 high, offset low, offset
 * high), key = (seed low, seed high)) is >= round(p * 2^32); a kept weight is
 * scaled by 1 / (1 - p).  p in [0, 1); 0 disables dropout.  The same seed and
 * offset in na2d_backward_ex reproduce the mask. */
typedef struct {
    float p;
    unsigned long long seed;
    unsigned long long offset;
} na2d_dropout;

/* na2d_forward on strided tensors, optionally also writing the attention
 * weights (after dropout, as the layer returns them with output_attentions)
 * to attn [B, heads, H, W, k*k] fp32 (NULL: not written) and applying
 * dropout (drop NULL or drop->p == 0: none; p outside [0, 1):
 * NA2D_ERR_SHAPE).  q, k, v, out are views (see na2d_tensor); out must not
 * overlap itself, an input or attn (NA2D_ERR_ALIAS).  Contiguous tensors
 * without weights or dropout take the same kernels as na2d_forward; other
 * calls run on the CUDA-core kernel. */
NA2D_API na2d_status na2d_forward_ex(const na2d_problem *p, const na2d_tensor *q, const na2d_tensor *k,
                                     const na2d_tensor *v, const void *rpb, const na2d_tensor *out, float *attn,
                                     const na2d_dropout *drop, void *stream);

/* na2d_backward on strided tensors with attention dropout (the mask of the
 * forward call with the same na2d_dropout).  Same workspace rule as
 * na2d_backward; runs on the CUDA cores. */
NA2D_API na2d_status na2d_backward_ex(const na2d_problem *p, const na2d_tensor *q, const na2d_tensor *k,
                                      const na2d_tensor *v, const void *rpb, const na2d_tensor *dout,
                                      const na2d_tensor *dq, const na2d_tensor *dk, const na2d_tensor *dv,
                                      void *drpb, const na2d_dropout *drop, void *workspace,
                                      size_t workspace_bytes, void *stream);

/* Diagnostic.  Kernels that wait on shared-memory barriers for their own
 * tensor copies give up after about a second of device time (a wait that long
 * means the copy will never arrive), skip their remaining work and count the
 * event.  This call writes that count for the current device into *count and
 * clears it.  Unlike the calls above it synchronises `stream`.  A non-zero
 * count means some outputs of the kernels since the last call were not
 * written; it has never been observed and indicates a library bug. */
NA2D_API na2d_status na2d_device_faults(unsigned int *count, void *stream);

/* A static, human-readable name for a status. */
NA2D_API const char *na2d_status_str(na2d_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
NA2D_API int na2d_version(void);

/* Diagnostic.  The name of the kernel that the calling host thread's most
 * recent na2d_forward call launched (a static string such as
 * "fwd_stream_kernel"), or NULL if that call launched nothing (an argument
 * error or an empty problem) or no call was made on this thread yet.  Used by
 * the tests to record which kernel each problem shape reaches. */
NA2D_API const char *na2d_last_kernel(void);

/* Test hook for the error path of the bounded waits.  The streaming kernel
 * (the k = 7 sliding-window forward) and the tcgen05 kernel for dilation
 * groups of up to 16 x 16 pixels with k >= 9 wait for their copies and
 * products with a limit; when a wait runs out the kernel counts the event
 * (see na2d_device_faults), stops issuing and computing, waits for its copies
 * and products already in flight (always with the full limit, so nothing
 * lands in released memory), and returns;
 * the outputs of that call are then unspecified.  This call shortens the
 * data waits' limit to sm_clocks for the calls that follow on any thread
 * (0 restores the default, about 2^31 clocks).  A limit of a few hundred
 * clocks makes a wait run out on purpose without any device fault; tests use
 * it to run the error path. */
NA2D_API void na2d_debug_set_wait_limit(long long sm_clocks);

#ifdef __cplusplus
}
#endif

#endif /* NA2D_H */
