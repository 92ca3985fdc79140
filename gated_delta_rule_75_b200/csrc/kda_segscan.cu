// Composition of segment maps: the sequential step of the segment-parallel
// state walk, and of context parallelism across GPUs.
//
// The delta-rule recurrence is linear in the state, so a run of chunks maps
// its entry state affinely, S -> M S + B (M: dk x dk, B: dk x dv; with the
// notation of the chunk equations, one chunk has
// M = Diag(e^{G_last}) - (K e^{G_last - G})^T W and
// B = (K e^{G_last - G})^T T' V).  Given the maps of consecutive segments, the
// entry state of segment s is X_s with X_0 = h0 and X_{s+1} = M_s X_s + B_s.
//
// Kernel layout: one CTA per (chain, 16-column block of the state); the 16
// columns of X stay in shared memory across the segments (columns of the
// state never mix).  Each M_s is staged in shared memory by asynchronous
// 16-byte copies (all threads, coalesced), double-buffered so that M_{s+1}
// arrives while X_{s+1} = M_s X_s + B_s is computed.  The contraction over the
// dk rows of X is split four ways: four groups of 128 threads (four warps per
// scheduler, so the shared-memory loads of one warp hide behind the FMAs of
// the others) each take a quarter of the rows, and group 0 adds the other
// three partial products from shared memory.  In every group a thread owns a
// 4 x 4 register tile of the product (rows r, r+32, r+64, r+96; 4 columns), so
// every 16-byte shared-memory load feeds 16 FMAs; rows of the staged M are
// padded to 132 floats so that the 8 consecutive rows a warp reads fall in
// distinct banks.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kPrefixGroups = 4;                               // split of the contraction
constexpr int kPrefixThreads = 128 * kPrefixGroups;
constexpr int kPrefixCols = 16;
constexpr int kMPitch = 132;                                   // floats per staged row
constexpr int kMapFloats = 2 * 128 * kMPitch;                  // the double-buffered M_s
constexpr int kPartFloats = (kPrefixGroups - 1) * 128 * kPrefixCols;
constexpr int kPrefixSmem = (kMapFloats + kPartFloats) * (int)sizeof(float);

__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kPrefixThreads, 1)   // one CTA per SM
affine_prefix_kernel(PrefixArgs p)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ __align__(16) float msm[];               // 2 x [128][kMPitch], partials
    float* part = msm + kMapFloats;                            // [groups - 1][128][kPrefixCols]
    __shared__ __align__(16) float X[128][kPrefixCols];
    const int64_t chain = blockIdx.x;
    const int64_t n = chain / p.hg;
    const int64_t hl = chain - n * p.hg;
    const int64_t h = p.h_base + hl;
    const int64_t head = p.abs_head ? h : hl;
    const int tid = threadIdx.x;
    // this thread: rows rg + 32 i (i < dk / 32) and columns j0 + 4 cg .. +3 of the product,
    // summed over rows kg dk / 4 .. (kg + 1) dk / 4 - 1 of X; group 0 holds X_s
    const int kg = tid >> 7, gt = tid & 127;
    const int cg = gt & 3, rg = gt >> 2;
    const int j = blockIdx.y * kPrefixCols + 4 * cg;
    const int nr = p.dk >> 5;
    const int64_t dkdk = (int64_t)p.dk * p.dk, dkdv = (int64_t)p.dk * p.dv;

    int64_t base, count;
    if (p.seg_off) {
        base = p.seg_off[n];
        count = p.seg_off[n + 1] - base;
    } else {
        base = n * p.nseg;
        count = p.nseg;
    }
    int64_t sidx = n * p.H + h;
    if (p.slots) {
        const int64_t sl = p.slots[n];
        sidx = (sl >= 0 && sl < p.P) ? sl * p.H + h : -1;
        if (sl >= p.P && tid == 0 && blockIdx.y == 0 && p.err) atomicOr(p.err, 1);
    }
    // step s multiplies by M_s unless it is the last one and only entry states are wanted
    const int64_t steps = p.out ? count : count - 1;
    auto stage_map = [&](int64_t s) {                          // all threads
        const float* src = p.maps + ((base + s) * p.hstride + head) * dkdk;
        float* dst = msm + (s & 1) * 128 * kMPitch;
        const int quads = p.dk >> 2;
        for (int i = tid; i < p.dk * quads; i += kPrefixThreads) {
            const int rr = i / quads, c = i - rr * quads;
            cp_async16(dst + rr * kMPitch + 4 * c, src + (int64_t)rr * p.dk + 4 * c);
        }
        cp_async_commit();
    };
    if (steps > 0) stage_map(0);

    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kg == 0 && i < nr) {
            const int r = rg + 32 * i;
            if (p.h0 && sidx >= 0)
                x[i] = *reinterpret_cast<const float4*>(p.h0 + sidx * dkdv + (int64_t)r * p.dv + j);
            *reinterpret_cast<float4*>(&X[r][4 * cg]) = x[i];
        }
    }

    for (int64_t s = 0; s < count; ++s) {
        const int64_t idx = (base + s) * p.hstride + head;
        if (p.starts && kg == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < nr)
                    *reinterpret_cast<float4*>(p.starts + idx * dkdv + (int64_t)(rg + 32 * i) * p.dv + j) = x[i];
        }
        if (s >= steps) break;
        float4 acc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {                          // B_s: in flight during the wait
            acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kg == 0 && i < nr)
                acc[i] = *reinterpret_cast<const float4*>(p.offs + idx * dkdv +
                                                          (int64_t)(rg + 32 * i) * p.dv + j);
        }
        if (s + 1 < steps) {
            stage_map(s + 1);                                  // its buffer was freed at the end of s-1
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                                       // M_s staged, X_s written
        const float* mb = msm + (s & 1) * 128 * kMPitch + rg * kMPitch;
        auto fma4 = [](float4& a, float m, const float4& xv) {
            a.x = fmaf(m, xv.x, a.x);
            a.y = fmaf(m, xv.y, a.y);
            a.z = fmaf(m, xv.z, a.z);
            a.w = fmaf(m, xv.w, a.w);
        };
        if (nr == 4) {
#pragma unroll 2
            for (int k = 32 * kg; k < 32 * kg + 32; k += 4) {
                float4 m[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) m[i] = *reinterpret_cast<const float4*>(mb + 32 * i * kMPitch + k);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 xv = *reinterpret_cast<const float4*>(&X[k + u][4 * cg]);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        fma4(acc[i], u == 0 ? m[i].x : u == 1 ? m[i].y : u == 2 ? m[i].z : m[i].w, xv);
                }
            }
        } else {
#pragma unroll 2
            for (int k = 16 * kg; k < 16 * kg + 16; k += 4) {
                float4 m[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) m[i] = *reinterpret_cast<const float4*>(mb + 32 * i * kMPitch + k);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 xv = *reinterpret_cast<const float4*>(&X[k + u][4 * cg]);
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        fma4(acc[i], u == 0 ? m[i].x : u == 1 ? m[i].y : u == 2 ? m[i].z : m[i].w, xv);
                }
            }
        }
        if (kg > 0) {
            float* pp = part + (kg - 1) * 128 * kPrefixCols;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < nr) *reinterpret_cast<float4*>(pp + (rg + 32 * i) * kPrefixCols + 4 * cg) = acc[i];
        }
        __syncthreads();                                       // partials written; X_s, M_s read
        if (kg == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i < nr) {
                    const int r = rg + 32 * i;
#pragma unroll
                    for (int g = 0; g < kPrefixGroups - 1; ++g) {
                        const float4 v = *reinterpret_cast<const float4*>(part + (g * 128 + r) * kPrefixCols + 4 * cg);
                        acc[i].x += v.x; acc[i].y += v.y; acc[i].z += v.z; acc[i].w += v.w;
                    }
                    x[i] = acc[i];
                    *reinterpret_cast<float4*>(&X[r][4 * cg]) = acc[i];
                }
            }
        }
        // the next step's first barrier orders X_{s+1} before its reads, and this step's
        // partial reads before the next partial writes
    }
    if (p.out && sidx >= 0 && kg == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < nr)
                *reinterpret_cast<float4*>(p.out + sidx * dkdv + (int64_t)(rg + 32 * i) * p.dv + j) = x[i];
    }
}

cudaError_t launch_affine_prefix(const PrefixArgs& p, cudaStream_t st)
{
    if ((p.dk != 64 && p.dk != 128) || p.dv % kPrefixCols != 0) return cudaErrorInvalidValue;
    if (p.N * p.hg == 0) return cudaSuccess;
    static std::atomic<uint64_t> attr_done{0};
    cudaError_t e = once_per_device(attr_done, [] {
        return cudaFuncSetAttribute(affine_prefix_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefixSmem);
    });
    if (e) return e;
    dim3 grid((unsigned)(p.N * p.hg), (unsigned)(p.dv / kPrefixCols));
    LaunchScope scope(st, K_AFFINE_PREFIX);
    return launch_pdl(affine_prefix_kernel, grid, dim3(kPrefixThreads), kPrefixSmem, st, p);
}

__global__ void fill_identity_kernel(float* __restrict__ dst, int64_t total, int d)
{
    const int64_t dd = (int64_t)d * d;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = i % dd;
        dst[i] = (e / d == e % d) ? 1.f : 0.f;
    }
}

cudaError_t launch_fill_identity(float* dst, int64_t count, int d, cudaStream_t st)
{
    const int64_t total = count * d * d;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    LaunchScope scope(st, K_FILL);
    fill_identity_kernel<<<(unsigned)blocks, 256, 0, st>>>(dst, total, d);
    return cudaGetLastError();
}

}  // namespace kda
