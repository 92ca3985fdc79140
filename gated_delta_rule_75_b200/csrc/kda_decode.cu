// Decode step of the KDA recurrence: one token per sequence, state updated in
// place.  Follows the per-token step of "Kimi Delta Attention: la atencion
// lineal detras de Kimi K2 y Qwen3" (section "Como funciona Kimi Delta
// Attention paso a paso"): decay per key channel, predict, beta-scaled error,
// write, read.
//
// The step is bound by HBM: each (sequence, head) state of dk*dv fp32 is read
// once and written once; everything else is a few hundred bytes.  One CTA of
// 256 threads owns one (sequence, head).  Thread (row-group rg, column quad c4)
// keeps DK/RG state rows of 4 columns in registers, loaded with 128-bit
// streaming loads (whole 512 B rows per warp for dv = 128), so the state never
// touches shared memory; only the two dk-reductions (vhat and the read) go
// through shared memory, across row groups.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ log_alpha, const float* __restrict__ beta,
                   float* __restrict__ state, T* __restrict__ out, float scale,
                   const int32_t* __restrict__ slots, int64_t H, int64_t P, int* __restrict__ err,
                   int gate_scalar)
{
    constexpr int TPR = DV / 4;        // threads per state row (float4 each)
    constexpr int RG = 256 / TPR;      // row groups
    constexpr int RPT = DK / RG;       // rows per thread
    static_assert(RPT * RG == DK && TPR * RG == 256, "shape");

    __shared__ float sk[DK], sq[DK], sa[DK], sv[DV], se[DV];
    __shared__ float4 red[RG][TPR];

    const int64_t p = blockIdx.x;                 // (sequence, head) pair
    const int tid = threadIdx.x;
    const int c4 = tid % TPR;
    const int rg = tid / TPR;

    // pooled states: sequence n owns state slot slots[n]; a negative slot means
    // "no state" (output zeros); a slot past the pool is reported and skipped
    int64_t sp = p;
    if (slots) {
        const int64_t n = p / H, h = p - n * H;
        const int64_t sl = slots[n];
        if (sl < 0 || sl >= P) {
            if (sl >= P && tid == 0 && err) atomicOr(err, 1);
            for (int j = tid; j < DV; j += 256) IO<T>::store(out, p * DV + j, 0.f);
            return;
        }
        sp = sl * H + h;
    }
    float4* S4 = reinterpret_cast<float4*>(state + sp * (int64_t)DK * DV);
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)                 // issue every state load first
        s[r] = __ldcs(&S4[(rg * RPT + r) * TPR + c4]);

    for (int i = tid; i < DK; i += 256) {
        sk[i] = IO<T>::load(k, p * DK + i);
        sq[i] = scale * IO<T>::load(q, p * DK + i);
        sa[i] = expf(gate_scalar ? log_alpha[p] : log_alpha[p * DK + i]);
    }
    for (int j = tid; j < DV; j += 256) sv[j] = IO<T>::load(v, p * DV + j);
    const float b = beta[p];
    __syncthreads();

    // decay, then the partial prediction vhat = S~^T k over this thread's rows
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float a = sa[i], kk = sk[i];
        s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
        acc.x += kk * s[r].x; acc.y += kk * s[r].y; acc.z += kk * s[r].z; acc.w += kk * s[r].w;
    }
    red[rg][c4] = acc;
    __syncthreads();
    for (int j = tid; j < DV; j += 256) {
        float vh = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) vh += reinterpret_cast<const float*>(&red[g][0])[j];
        se[j] = b * (sv[j] - vh);                 // beta-scaled error
    }
    __syncthreads();

    // write the error along k, then the partial read o = scale * S^T q
    const float4 e = reinterpret_cast<const float4*>(se)[c4];
    acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float kk = sk[i], qq = sq[i];
        s[r].x += kk * e.x; s[r].y += kk * e.y; s[r].z += kk * e.z; s[r].w += kk * e.w;
        __stcs(&S4[i * TPR + c4], s[r]);
        acc.x += qq * s[r].x; acc.y += qq * s[r].y; acc.z += qq * s[r].z; acc.w += qq * s[r].w;
    }
    red[rg][c4] = acc;
    __syncthreads();
    for (int j = tid; j < DV; j += 256) {
        float o = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) o += reinterpret_cast<const float*>(&red[g][0])[j];
        IO<T>::store(out, p * DV + j, o);
    }
}

template <typename T, int DK, int DV>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream)
{
    LaunchScope scope(stream, K_DECODE);
    decode_step_kernel<T, DK, DV><<<(unsigned)(a.N * a.H), 256, 0, stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, a.log_alpha, a.beta, a.state, (T*)a.out,
        a.scale, a.slots, a.H, a.P, a.err, a.gate_scalar ? 1 : 0);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t st)
{
    if (a.dk == 128 && a.dv == 128) return launch_decode_t<T, 128, 128>(a, st);
    if (a.dk == 128 && a.dv == 64) return launch_decode_t<T, 128, 64>(a, st);
    if (a.dk == 64 && a.dv == 128) return launch_decode_t<T, 64, 128>(a, st);
    return launch_decode_t<T, 64, 64>(a, st);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st)
{
    // one CTA per (sequence, head); grid.x is limited to 2^31-1
    if (a.N * a.H > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (a.io == KDA_IO_F32) return launch_decode_d<float>(a, st);
    return launch_decode_d<__nv_bfloat16>(a, st);
}

}  // namespace kda
