// na2d_tcgen05.cuh -- inline PTX wrappers shared by the kernels on the
// 5th-generation tensor cores: mbarriers, programmatic dependent launch, TMA
// tensor loads, tensor-memory (TMEM) allocation and access, the sm_100
// shared-memory matrix and kind::f16 instruction descriptors, tcgen05.mma and
// its commit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

namespace na2d {

constexpr uint32_t kTmemCols = 512;   // every tcgen05 kernel here takes the whole tensor memory

// ---- mbarriers ---------------------------------------------------------------
__device__ __forceinline__ void mb_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mb_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after `limit` SM clocks (by default 2^31, about a
// second); each try may suspend for up to 20 us, so a short limit is
// overrun by at most that much.
__device__ __forceinline__ bool mb_wait(uint32_t bar, uint32_t parity, long long limit = 1LL << 31) {
    if (mb_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mb_try(bar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}
__device__ __forceinline__ void mb_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mb_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// ---- programmatic dependent launch ------------------------------------------
// The kernels are launched with programmatic stream serialisation: a grid
// may be scheduled while the previous kernel on the stream finishes, runs its
// prologue (barriers, tensor-memory allocation), and reads no global memory
// before grid_dep_wait() returns, i.e. before that kernel has completed and
// its writes are visible.  grid_dep_launch() lets the next grid be scheduled.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- TMA ---------------------------------------------------------------------
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c1, int c2,
                                            int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5, %6}], [%7];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}

// ---- TMEM --------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem),
                 "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "n"(kTmemCols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// Loads N consecutive 32-bit columns of this thread's lane (complete after
// tmem_ld_wait).
__device__ __forceinline__ void tmem_ld8(uint32_t ta, float *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "r"(ta)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t ta, float *v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(ta)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t ta, float *v) {
    tmem_ld16(ta, v);
    tmem_ld16(ta + 16, v + 16);
}
// Stores 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t ta, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
            ta),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// ---- MMA -----------------------------------------------------------------------
// Shared-memory matrix descriptor, 64-byte swizzle (the layout the TMA copies
// write: 16-byte chunk c of the 64-byte row at byte address a stored at chunk
// c ^ ((a >> 7) & 3)); byte offsets in 16-byte units; version 1.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (4ull << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator, A and B of type T,
// A K-major, B K-major (b_mn = 0) or MN-major (1), M = 128.
template <typename T> __host__ __device__ constexpr uint32_t idesc_f16(int N, int b_mn) {
    return (1u << 4) | ((std::is_same<T, __nv_bfloat16>::value ? 1u : 0u) << 7) |
           ((std::is_same<T, __nv_bfloat16>::value ? 1u : 0u) << 10) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
            d),
        "r"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrives once on the mbarrier when every earlier tcgen05.mma of this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}

template <typename T> struct Pack2;
template <> struct Pack2<__half> {
    __device__ __forceinline__ static uint32_t run(float lo, float hi) {
        uint32_t e;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(e) : "f"(hi), "f"(lo));
        return e;
    }
};
template <> struct Pack2<__nv_bfloat16> {
    __device__ __forceinline__ static uint32_t run(float lo, float hi) {
        uint32_t e;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(e) : "f"(hi), "f"(lo));
        return e;
    }
};

// One output pixel of D = 32 channels (64 bytes): o scaled by inv, packed to
// 16-bit pairs.  With st32 (the pixel is 32-byte aligned) as two 32-byte
// stores, else four 16-byte ones; a warp's pixels lie in different lines
// (they are d pixels apart), so the wider stores halve the store wavefronts.
template <typename T>
__device__ __forceinline__ void store_pixel64(unsigned char *dst, const float (&o)[32], float inv, bool st32) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = Pack2<T>::run(o[2 * i] * inv, o[2 * i + 1] * inv);
    if (st32) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"l"(dst + 32 * h),
                         "r"(pk[8 * h]), "r"(pk[8 * h + 1]), "r"(pk[8 * h + 2]), "r"(pk[8 * h + 3]), "r"(pk[8 * h + 4]),
                         "r"(pk[8 * h + 5]), "r"(pk[8 * h + 6]), "r"(pk[8 * h + 7])
                         : "memory");
    } else {
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

}  // namespace na2d
