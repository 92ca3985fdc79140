// Shared device helpers of the KDA CUDA library (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

constexpr int kChunk = 64;       // tokens per chunk of the chunkwise prefill
constexpr int kSubChunk = 16;    // sub-chunk used for exponent references

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization (launch_pdl) may be scheduled while the kernel before it on the
// stream is still running or draining.  griddep_wait() holds the calling thread
// until every grid that this one depends on has completed and its memory writes
// are visible, so each such kernel calls it before its first global-memory access;
// griddep_launch_dependents() lets the next kernel's CTAs be scheduled as SMs free
// up (they still wait for this grid to complete).  Both do nothing in a kernel
// launched without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// I/O element access: fp32 or bf16 storage, fp32 arithmetic.
template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float load(const float* p, int64_t i) { return p[i]; }
    static __device__ __forceinline__ void store(float* p, int64_t i, float x) { p[i] = x; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p, int64_t i) {
        return __bfloat162float(p[i]);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, int64_t i, float x) {
        p[i] = __float2bfloat16_rn(x);
    }
};

// Sequence n's token range [bos, eos) clamped into [0, T]: malformed offsets
// never produce an out-of-bounds index.
__device__ __forceinline__ void seq_range(const int32_t* cu, int64_t n, int64_t T_seq,
                                          int64_t T_total, int64_t& bos, int64_t& eos) {
    if (cu == nullptr) {
        bos = n * T_seq;
        eos = bos + T_seq;
        return;
    }
    int64_t a = cu[n], b = cu[n + 1];
    a = a < 0 ? 0 : (a > T_total ? T_total : a);
    b = b < a ? a : (b > T_total ? T_total : b);
    bos = a;
    eos = b;
}

}  // namespace kda
