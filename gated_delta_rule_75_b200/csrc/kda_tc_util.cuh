// Small device helpers shared by the tensor-core prefill kernels (sm_100a):
// fast exp2, bf16 packing, named barriers, and the tf32 16x16 block product
// used by the blocked inverse of (I + A).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_umma.cuh"

namespace kda {
namespace tcu {

using umma::pack_bf16;

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void unpack8(uint4 u, float* f)
{
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float* f)
{
    uint4 u;
    u.x = pack_bf16(f[0], f[1]);
    u.y = pack_bf16(f[2], f[3]);
    u.z = pack_bf16(f[4], f[5]);
    u.w = pack_bf16(f[6], f[7]);
    return u;
}

__device__ __forceinline__ void ld8f(const float* p, float* f)
{
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ uint32_t tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// Barrier `id` (1..15) over the first `count` threads that reach it (whole warps).
__device__ __forceinline__ void bar_sync_named(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier `id` over `count` threads that also ANDs `pred` across them: every thread gets the
// same answer, so a group can leave a loop together.
__device__ __forceinline__ bool bar_and_named(int id, int count, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t"
        ".reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t"
        "}\n"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// acc (16x16, m16n8 fragments for the two 8-column halves) += X * Y, where X
// and Y are 16x16 fp32 blocks in shared memory with a row pitch of P floats.
template <int P>
__device__ __forceinline__ void mma16x16x16_tf32(float (&acc)[2][4], const float* X, const float* Y,
                                                 int lane)
{
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = tf32(X[g * P + 8 * ks + q]);
        const uint32_t a1 = tf32(X[(g + 8) * P + 8 * ks + q]);
        const uint32_t a2 = tf32(X[g * P + 8 * ks + q + 4]);
        const uint32_t a3 = tf32(X[(g + 8) * P + 8 * ks + q + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const uint32_t b0 = tf32(Y[(8 * ks + q) * P + 8 * nh + g]);
            const uint32_t b1 = tf32(Y[(8 * ks + q + 4) * P + 8 * nh + g]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[nh][0]), "+f"(acc[nh][1]), "+f"(acc[nh][2]), "+f"(acc[nh][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}

// Store a 16x16 accumulator (m16n8 fragments) scaled by `s` into a block with
// a row pitch of P floats.
template <int P>
__device__ __forceinline__ void store16x16(float* Z, const float (&acc)[2][4], float s, int lane)
{
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        Z[g * P + 8 * nh + 2 * q] = s * acc[nh][0];
        Z[g * P + 8 * nh + 2 * q + 1] = s * acc[nh][1];
        Z[(g + 8) * P + 8 * nh + 2 * q] = s * acc[nh][2];
        Z[(g + 8) * P + 8 * nh + 2 * q + 1] = s * acc[nh][3];
    }
}

}  // namespace tcu
}  // namespace kda
