// Chunkwise KDA prefill, fp32 SIMT kernels.
//
// The chunk form is derived by unrolling the per-token step of "Kimi Delta
// Attention: la atencion lineal detras de Kimi K2 y Qwen3" (section "Como
// funciona Kimi Delta Attention paso a paso") over a block of C = 64 tokens;
// "Kimi Linear acaba de superar a la atencion completa en sus propios
// terminos" says a chunkwise algorithm over the diagonal-plus-low-rank
// transition exists but prints no equations.  Per chunk (padded with g = 0,
// beta = 0, k = q = v = 0), G_i = sum_{j<=i} g_j restarting at the chunk:
//
//   A_ij   = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}        (i > j)
//   Aqk_ij = scale  sum_c q_ic k_jc e^{G_ic - G_jc}        (i >= j)
//   T = (I + A)^{-1},  W = T diag(beta)(K e^G),  Ut = T diag(beta) V
//   U = Ut - W S,  O = scale (Q e^G) S + Aqk U,
//   S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T U
//
// Two kernels: `prep` (steps a and b: cumulative decay and the intra-chunk
// WY/UT transform, parallel over (chunk, head)) writes W, Ut, Aqk, Q e^G,
// K e^{G_last-G} and e^{G_last} to an fp32 workspace; `state` (steps c and d)
// walks the chunks of one (sequence, head, 32-column dv tile) in order with the
// state tile in registers and writes the output.  Every exponential is either a
// factor <= 1 or, inside a 16-token diagonal block, bounded by 64 nats of decay;
// blocks that decay faster are taken pairwise (e^{G_i - G_j}), so this path has
// no limit on the decay rate.  It is the reference-quality GPU path: fp32 I/O
// and the bisection baseline of the tensor-core kernels.
#include "kda_chunk_simt.cuh"

namespace kda {

int64_t simt_ws_floats_per_chunk(int dk, int dv)
{
    return (int64_t)kChunk * (3 * dk + dv + kChunk) + dk;
}

template <typename T, int DK, int DV>
static cudaError_t run_simt_t(const PrefillArgs& a, float* ws, int64_t Hg, cudaStream_t st)
{
    const size_t smem_prep = simt_prep_smem<DK, DV>();
    const size_t smem_state = simt_state_smem<DK, DV>();
    static std::atomic<uint64_t> attrs_done{0};
    cudaError_t e = once_per_device(attrs_done, [&] {
        cudaError_t r = cudaFuncSetAttribute(chunk_prep_simt_kernel<T, DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_prep);
        if (r) return r;
        return cudaFuncSetAttribute(chunk_state_simt_kernel<T, DK, DV>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_state);
    });
    if (e) return e;
    for (int64_t hb = 0; hb < a.H; hb += Hg) {
        const int64_t hg = (a.H - hb) < Hg ? (a.H - hb) : Hg;
        if (a.si.chunks_upper > 0) {
            dim3 gp((unsigned)a.si.chunks_upper, (unsigned)hg);
            LaunchScope scope(st, K_PREP_SIMT);
            e = launch_pdl(chunk_prep_simt_kernel<T, DK, DV>, gp, dim3(kSimtPrepThreads), smem_prep, st,
                           (const T*)a.q, (const T*)a.k, (const T*)a.v, a.log_alpha, a.beta, a.si, a.H, hb,
                           Hg, a.scale, ws, a.gate_scalar ? 1 : 0);
            if (e) return e;
        }
        dim3 gs((unsigned)(a.si.N * hg * (DV / 32)));
        {
            LaunchScope scope(st, K_STATE_SIMT);
            e = launch_pdl(chunk_state_simt_kernel<T, DK, DV>, gs, dim3(256), smem_state, st, ws, a, hb, Hg);
        }
        if (e) return e;
    }
    return cudaSuccess;
}

template <typename T>
static cudaError_t run_simt_d(const PrefillArgs& a, float* ws, int64_t Hg, cudaStream_t st)
{
    if (a.dk == 128 && a.dv == 128) return run_simt_t<T, 128, 128>(a, ws, Hg, st);
    if (a.dk == 128 && a.dv == 64) return run_simt_t<T, 128, 64>(a, ws, Hg, st);
    if (a.dk == 64 && a.dv == 128) return run_simt_t<T, 64, 128>(a, ws, Hg, st);
    return run_simt_t<T, 64, 64>(a, ws, Hg, st);
}

cudaError_t run_prefill_simt(const PrefillArgs& a, float* ws, int64_t Hg, cudaStream_t st)
{
    if (a.io == KDA_IO_F32) return run_simt_d<float>(a, ws, Hg, st);
    return run_simt_d<__nv_bfloat16>(a, ws, Hg, st);
}

}  // namespace kda
