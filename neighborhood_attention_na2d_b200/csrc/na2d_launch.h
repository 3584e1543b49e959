// na2d_launch.h -- host-side launchers behind the C ABI (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace na2d {

enum class DType { F32 = 0, F16 = 1, BF16 = 2 };

struct Problem {
    int B, heads, H, W, D, k, d;
    DType dtype;
    int64_t bh() const { return (int64_t)B * heads; }
    // padded map (maps shorter than k*d are padded with zero pixels at the
    // bottom / right and the output cropped)
    int Hp() const { return H > k * d ? H : k * d; }
    int Wp() const { return W > k * d ? W : k * d; }
};

// A [B, heads, H, W, D] tensor given by element strides; channels contiguous.
struct View {
    const void *p;
    int64_t sb, sh, sy, sx;
    static View contiguous(const void *ptr, const Problem &pr) {
        const int64_t sx = pr.D, sy = (int64_t)pr.W * sx, sh = (int64_t)pr.H * sy, sb = (int64_t)pr.heads * sh;
        return View{ptr, sb, sh, sy, sx};
    }
    bool is_contiguous(const Problem &pr) const {
        const View c = contiguous(p, pr);
        return sb == c.sb && sh == c.sh && sy == c.sy && sx == c.sx;
    }
};

// Attention dropout: probability p (0: none), Philox key and counter offset.
struct Dropout {
    float p;
    uint64_t seed, offset;
};

// Fused forward on the tensor cores (f16 / bf16, D = 32, k in 3..13).
cudaError_t launch_forward_tc(const Problem &p, const void *q, const void *k, const void *v,
                              const void *rpb, void *out, cudaStream_t stream);

// Fused forward on the CUDA cores: any dtype, D in {16, 32, 64, 128}, any
// odd k <= 13, strided views, padded short maps; optionally writes the
// (dropped-out) attention weights to attn and applies dropout.
cudaError_t launch_forward_simt(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                const View &out, float *attn, const Dropout &drop, cudaStream_t stream);

// Split path.
cudaError_t launch_qk_rpb(const Problem &p, const void *q, const void *k, const void *rpb, float *attn,
                          cudaStream_t stream);
cudaError_t launch_softmax(const Problem &p, float *attn, cudaStream_t stream);
cudaError_t launch_av(const Problem &p, const float *attn, const void *v, void *out, cudaStream_t stream);

// Backward (dq, dk, dv, drpb) of the fused forward; workspace holds
// backward_workspace_bytes(p) bytes of fp32 scratch.
size_t backward_workspace_bytes(const Problem &p);
cudaError_t launch_backward(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                            const void *dout, void *dq, void *dk, void *dv, void *drpb, void *workspace,
                            cudaStream_t stream);
// The same on strided views, with attention dropout.
cudaError_t launch_backward_views(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                  const View &dout, const View &dq, const View &dk, const View &dv, void *drpb,
                                  const Dropout &drop, void *workspace, cudaStream_t stream);

// The backward with the library's built-in scratch array instead of a
// caller workspace (no allocation); problems whose workspace exceeds
// noalloc_scratch_bytes() are refused by the caller of this function.
size_t noalloc_scratch_bytes();
cudaError_t launch_backward_noalloc(const Problem &p, const void *q, const void *k, const void *v, const void *rpb,
                                    const void *dout, void *dq, void *dk, void *dv, void *drpb, cudaStream_t stream);

// Records, for the calling host thread, the name of the kernel a forward call
// has just launched (a static string); read back by na2d_last_kernel.
void note_kernel(const char *name);

// Reads and clears the count of device-side bounded waits that ran out;
// synchronises the stream.
cudaError_t read_device_faults(unsigned int *count, cudaStream_t stream);

// True when launch_forward_tc handles this problem.
bool tc_supported(const Problem &p);

// 5-D TMA view (D, gx, j', gy, bh * H / d + i') of a [B*heads, H, W, 32]
// tensor with H and W multiples of d (pixel (gy + d*i', gx + d*j') of plane
// bh), 64-byte swizzled boxes of 32 x box_gx x box_cols x 1 x box_rows
// elements (box_gx adjacent groups side by side).  False when the driver
// entry point is missing or the encoding is refused.
bool encode_group_map(CUtensorMap *map, const void *base, DType dt, int64_t bh, int H, int W, int d, int box_cols,
                      int box_rows, int box_gx);

// Forward on the 5th-generation tensor cores (tcgen05) for maps whose
// dilation groups are all exactly 7 x 7 (H = W = 7d, k = 7, D = 32, f16 /
// bf16).  Sets *launched when it took the problem.
bool umma_supported(const Problem &p);
cudaError_t launch_forward_umma(const Problem &p, const void *q, const void *k, const void *v,
                                const void *rpb, void *out, cudaStream_t stream, bool *launched);
// As read_device_faults, for the tcgen05 kernel's counter.
cudaError_t read_umma_faults(unsigned int *count, cudaStream_t stream);

// Forward on the tcgen05 tensor cores for maps whose dilation groups are
// between k and 16 pixels on each side with k >= 9 (H and W multiples of d,
// D = 32, f16 / bf16).  Sets *launched when it took the problem.
bool ugrp_supported(const Problem &p);
cudaError_t launch_forward_ugrp(const Problem &p, const void *q, const void *k, const void *v,
                                const void *rpb, void *out, cudaStream_t stream, bool *launched);
// Test hook: the kernel's data waits give up after `clocks` SM clocks (0: the
// default, about a second).
void set_ugrp_wait_limit(long long clocks);
// As read_device_faults, for this kernel's counter.
cudaError_t read_ugrp_faults(unsigned int *count, cudaStream_t stream);

// Streaming tensor-core forward for k = 7 (f16 / bf16, D = 32): d = 1 maps with
// W >= 14 and H >= 8 (maps wider than 64 columns in column bands), or
// H = W = 7d (every dilation group 7 x 7).  Sets
// *launched when it took the problem; otherwise the caller uses
// launch_forward_tc.
bool stream_supported(const Problem &p);
// q, k, v are views with one shared set of strides; out any view.
cudaError_t launch_forward_stream(const Problem &p, const View &q, const View &k, const View &v, const void *rpb,
                                  const View &out, cudaStream_t stream, bool *launched);
// Test hook: the streaming kernel's data waits give up after `clocks` SM
// clocks (0: the default, about a second).
void set_stream_wait_limit(long long clocks);
// As read_device_faults, for the streaming kernel's counter.
cudaError_t read_stream_faults(unsigned int *count, cudaStream_t stream);

}  // namespace na2d
