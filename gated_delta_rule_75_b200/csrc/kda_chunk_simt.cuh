// fp32 SIMT chunk kernels shared by the prefill (kda_chunk_simt.cu) and the
// backward pass (kda_chunk_bwd.cu); the chunk equations are listed at the top
// of kda_chunk_simt.cu.  The backward variants (kBwd) use a larger block per
// (chunk, head) (BwdWs) and also save what the gradient kernels need.
#pragma once
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kTW = 32;           // dv columns per state-walk tile
constexpr int kSP = 36;           // row pitch of a [DK][32] state tile in shared memory:
                                  // 16-byte accesses by 8 consecutive rows hit distinct banks

// acc[r] += sum_k A[(row0 + RS r) * lda + k] * B[k * LDB + lane], r < NR (A rows read as
// 16-byte broadcasts, B columns one per lane), K a multiple of 4.
template <int NR, int RS, int LDB>
__device__ __forceinline__ void rows_mac(float (&acc)[NR], const float* A, int lda, int row0,
                                         const float* B, int K, int lane)
{
    for (int k = 0; k < K; k += 4) {
        const float b0 = B[k * LDB + lane], b1 = B[(k + 1) * LDB + lane];
        const float b2 = B[(k + 2) * LDB + lane], b3 = B[(k + 3) * LDB + lane];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const float4 a = *reinterpret_cast<const float4*>(A + (row0 + RS * r) * lda + k);
            acc[r] += a.x * b0 + a.y * b1 + a.z * b2 + a.w * b3;
        }
    }
}

// The eight-warp form: rows row0 + 8 r, r < 8.
template <int LDB = kTW>
__device__ __forceinline__ void rows8_mac(float (&acc)[8], const float* A, int lda, int row0,
                                          const float* B, int K, int lane)
{
    rows_mac<8, 8, LDB>(acc, A, lda, row0, B, K, lane);
}

// Workspace block of one (chunk, head), in floats.
template <int DK, int DV>
struct SimtWs {
    static constexpr int64_t W = 0;
    static constexpr int64_t Ut = W + kChunk * DK;
    static constexpr int64_t Aqk = Ut + kChunk * DV;
    static constexpr int64_t QG = Aqk + kChunk * kChunk;
    static constexpr int64_t KG = QG + kChunk * DK;
    static constexpr int64_t Gam = KG + kChunk * DK;
    static constexpr int64_t size = Gam + DK;
};

// Backward block of one (chunk, head): the prefill block, then what the
// backward kernels pass to one another (all fp32):
//   Tm = (I + A)^{-1}, Ap = A' (A before the beta row scaling), KGm = K e^G  (prep)
//   Sx = the chunk's entry state, dSx = gradient of its exit state           (walks)
//   E = U, R = V - (K e^G) S, dE, dR                                         (dense pass 1)
//   dKG, dQG, dKh: gradients of K e^G, scale Q e^G, K e^{G_last - G};
//   dTp, dAqk: gradients of T diag(beta) and Aqk; dGlS = sum_v S * dS_exit  (dense pass 2)
template <int DK, int DV>
struct BwdWs {
    static constexpr int C = kChunk;
    static constexpr int64_t Tm = SimtWs<DK, DV>::size;
    static constexpr int64_t Ap = Tm + C * C;
    static constexpr int64_t KGm = Ap + C * C;
    static constexpr int64_t Sx = KGm + C * DK;
    static constexpr int64_t dSx = Sx + DK * DV;
    static constexpr int64_t E = dSx + DK * DV;
    static constexpr int64_t R = E + C * DV;
    static constexpr int64_t dE = R + C * DV;
    static constexpr int64_t dR = dE + C * DV;
    static constexpr int64_t dKG = dR + C * DV;
    static constexpr int64_t dQG = dKG + C * DK;
    static constexpr int64_t dKh = dQG + C * DK;
    static constexpr int64_t dTp = dKh + C * DK;
    static constexpr int64_t dAqk = dTp + C * C;
    static constexpr int64_t dGlS = dAqk + C * C;
    static constexpr int64_t size = dGlS + DK;
};

template <int DK, int DV>
constexpr size_t simt_prep_smem()
{
    return sizeof(float) * (size_t)(kChunk * (3 * DK + DV) + 2 * kChunk * kChunk + kChunk + 32 * DK + 48 * (DK + 4));
}
template <int DK, int DV, bool kBwd = false>
constexpr size_t simt_state_smem()
{
    return sizeof(float) * (size_t)((kBwd ? 2 : 3) * kChunk * DK + (kBwd ? 0 : kChunk * kChunk) +
                                    kChunk * kTW + DK * kSP + DK);
}


// ---------------------------------------------------------------------------
// step a + b: cumulative log-decay and intra-chunk transform
// ---------------------------------------------------------------------------
constexpr int kSimtPrepThreads = 256;   // 16 rows x 16 column lanes in the A / Aqk phase

template <typename T, int DK, int DV, bool kBwd = false>
__global__ void __launch_bounds__(kSimtPrepThreads, 1)
chunk_prep_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ log_alpha, const float* __restrict__ beta,
                       SeqInfo si, int64_t H, int64_t h_base, int64_t Hg, float scale,
                       float* __restrict__ ws, int gate_scalar)
{
    constexpr int C = kChunk;
    extern __shared__ float smem[];
    float* sK = smem;                 // [C][DK]
    float* sQ = sK + C * DK;          // [C][DK], later beta K e^G
    float* sV = sQ + C * DK;          // [C][DV], later beta V
    float* sG = sV + C * DV;          // [C][DK]
    float* sA = sG + C * DK;          // [C][C]
    float* sT = sA + C * C;           // [C][C]
    float* sB = sT + C * C;           // [C]
    float* sKin = sB + C;             // [16][DK]  rows of one sub-chunk, referenced to its first row
    float* sQin = sKin + 16 * DK;     // [16][DK]
    constexpr int KVP = DK + 4;       // padded row pitch of sKvar (16 rows -> distinct banks)
    float* sKvar = sQin + 16 * DK;    // [48][KVP] earlier rows, referenced forward to it

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int64_t h = h_base + hl;
    int64_t n, t0, len;
    if (!si.locate(gc, n, t0, len)) return;
    const int tid = threadIdx.x;

    for (int e = tid; e < C * DK; e += blockDim.x) {
        const int t = e / DK, c = e % DK;
        const bool ok = t < len;
        const int64_t src = ((t0 + t) * H + h) * DK + c;
        sK[e] = ok ? IO<T>::load(k, src) : 0.f;
        sQ[e] = ok ? IO<T>::load(q, src) : 0.f;
        sG[e] = ok ? log_alpha[gate_scalar ? (t0 + t) * H + h : src] : 0.f;
    }
    for (int e = tid; e < C * DV; e += blockDim.x) {
        const int t = e / DV, c = e % DV;
        sV[e] = t < len ? IO<T>::load(v, ((t0 + t) * H + h) * DV + c) : 0.f;
    }
    for (int t = tid; t < C; t += blockDim.x) sB[t] = t < len ? beta[(t0 + t) * H + h] : 0.f;
    __syncthreads();

    // (a) inclusive cumulative sum of log-decay per channel within the chunk
    if (tid < DK) {
        float run = 0.f;
        for (int t = 0; t < C; ++t) { run += sG[t * DK + tid]; sG[t * DK + tid] = run; }
    }
    __syncthreads();

    float* blk = ws + (gc * Hg + hl) * (kBwd ? BwdWs<DK, DV>::size : SimtWs<DK, DV>::size);
    // (b1) A (strictly lower, beta-weighted) and Aqk (lower incl. diagonal), one 16-row
    // sub-chunk of rows i at a time.  For columns j before the sub-chunk (first row f) the
    // exponential splits into two factors <= 1, e^{G_i - G_f} e^{G_f - G_j}, so the sums are
    // dot products of precomputed rows; inside the diagonal block it is taken pairwise.
    for (int e = tid; e < C * C; e += blockDim.x) {
        sA[e] = 0.f;
        sT[e] = 0.f;
        if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + e] = 0.f;
    }
    for (int p = 0; p < C / 16; ++p) {
        const int f = 16 * p;
        __syncthreads();                          // zeros written, scratch rows free
        for (int e = tid; e < 16 * DK; e += blockDim.x) {
            const int i = f + e / DK, c = e % DK;
            const float x = expf(sG[i * DK + c] - sG[f * DK + c]);
            sKin[e] = sK[i * DK + c] * x;
            sQin[e] = sQ[i * DK + c] * x;
        }
        for (int e = tid; e < f * DK; e += blockDim.x) {
            const int j = e / DK, c = e % DK;
            sKvar[j * KVP + c] = sK[e] * expf(sG[f * DK + c] - sG[e]);
        }
        __syncthreads();
        {   // rows f .. f+15 (r = tid / 16), columns jg + 16 u < f; lanes run along the
            // columns (padded Kvar rows), the row is a broadcast
            const int r = tid >> 4, jg = tid & 15, i = f + r;
            float kk[3] = {0.f, 0.f, 0.f}, qk[3] = {0.f, 0.f, 0.f};
            for (int c = 0; c < DK; c += 4) {
                const float4 a = *reinterpret_cast<const float4*>(sKin + r * DK + c);
                const float4 q4 = *reinterpret_cast<const float4*>(sQin + r * DK + c);
#pragma unroll
                for (int u = 0; u < 3; ++u) {
                    if (u < p) {
                        const float4 kv = *reinterpret_cast<const float4*>(sKvar + (jg + 16 * u) * KVP + c);
                        kk[u] += a.x * kv.x + a.y * kv.y + a.z * kv.z + a.w * kv.w;
                        qk[u] += q4.x * kv.x + q4.y * kv.y + q4.z * kv.z + q4.w * kv.w;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 3; ++u) {
                if (u < p) {
                    const int j = jg + 16 * u;
                    sA[i * C + j] = sB[i] * kk[u];
                    sT[i * C + j] = scale * qk[u];   // Aqk parked in sT for now
                    if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + i * C + j] = kk[u];
                }
            }
            // diagonal block: pair (i, j = f + jg) when j <= i; lanes differ in j, so the
            // rotated channel index spreads them over the banks
            const int j = f + jg;
            if (j <= i) {
                float dk_ = 0.f, dq_ = 0.f;
                for (int cc = 0; cc < DK; ++cc) {
                    const int c = (cc + j) % DK;    // rotate to spread banks
                    const float e = expf(sG[i * DK + c] - sG[j * DK + c]);
                    const float kj = sK[j * DK + c] * e;
                    dk_ += sK[i * DK + c] * kj;
                    dq_ += sQ[i * DK + c] * kj;
                }
                if (j < i) {
                    sA[i * C + j] = sB[i] * dk_;
                    if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + i * C + j] = dk_;
                }
                sT[i * C + j] = scale * dq_;
            }
        }
    }
    __syncthreads();

    for (int e = tid; e < C * C; e += blockDim.x) blk[SimtWs<DK, DV>::Aqk + e] = sT[e];
    // Q e^G (scaled), K e^{G_last - G}, e^{G_last}
    for (int e = tid; e < C * DK; e += blockDim.x) {
        const int c = e % DK;
        const float G = sG[e], Gl = sG[(C - 1) * DK + c];
        blk[SimtWs<DK, DV>::QG + e] = scale * sQ[e] * expf(G);
        blk[SimtWs<DK, DV>::KG + e] = sK[e] * expf(Gl - G);
    }
    for (int c = tid; c < DK; c += blockDim.x) blk[SimtWs<DK, DV>::Gam + c] = expf(sG[(C - 1) * DK + c]);
    __syncthreads();

    // (b2) T = (I + A)^{-1}: column c by forward substitution
    if (tid < C) {
        const int c = tid;
        for (int i = 0; i < C; ++i) sT[i * C + c] = (i == c) ? 1.f : 0.f;
        for (int i = c + 1; i < C; ++i) {
            float acc = 0.f;
            for (int j = c; j < i; ++j) acc += sA[i * C + j] * sT[j * C + c];
            sT[i * C + c] = -acc;
        }
    }
    // beta K e^G into sQ, beta V in place
    for (int e = tid; e < C * DK; e += blockDim.x) sQ[e] = sB[e / DK] * sK[e] * expf(sG[e]);
    for (int e = tid; e < C * DV; e += blockDim.x) sV[e] *= sB[e / DV];
    __syncthreads();

    if constexpr (kBwd) {                       // T and K e^G for the backward
        for (int e = tid; e < C * C; e += blockDim.x) blk[BwdWs<DK, DV>::Tm + e] = sT[e];
        for (int e = tid; e < C * DK; e += blockDim.x)
            blk[BwdWs<DK, DV>::KGm + e] = sK[e] * expf(sG[e]);
    }

    // (b3) W = T (beta K e^G), Ut = T (beta V)
    for (int e = tid; e < C * DK; e += blockDim.x) {
        const int i = e / DK, c = e % DK;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc += sT[i * C + j] * sQ[j * DK + c];
        blk[SimtWs<DK, DV>::W + e] = acc;
    }
    for (int e = tid; e < C * DV; e += blockDim.x) {
        const int i = e / DV, c = e % DV;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc += sT[i * C + j] * sV[j * DV + c];
        blk[SimtWs<DK, DV>::Ut + e] = acc;
    }
}

// ---------------------------------------------------------------------------
// steps c + d: sequential state propagation and output, per 32-column dv tile
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV, bool kBwd = false>
__global__ void __launch_bounds__(256, kBwd ? 2 : 1)   // occupancy set by shared memory
chunk_state_simt_kernel(float* __restrict__ ws, PrefillArgs a, int64_t h_base, int64_t Hg)
{
    // kBwd: backward blocks; every chunk's entry state is saved (Sx) and
    // no output is written
    constexpr int64_t kStride = kBwd ? BwdWs<DK, DV>::size : SimtWs<DK, DV>::size;
    const SeqInfo& si = a.si;
    const int64_t H = a.H;
    T* __restrict__ out = (T*)a.out;
    constexpr int C = kChunk, TW = kTW;
    extern __shared__ __align__(16) float smem[];
    // (the backward walk writes no output: no Q e^G, no Aqk, and half the shared memory)
    float* sW = smem;                                  // [C][DK]
    float* sKG = sW + C * DK;                          // [C][DK]
    float* sU = sKG + C * DK;                          // [C][TW]
    float* sS = sU + C * TW;                           // [DK][kSP]  copy of the entry state
    float* sGam = sS + DK * kSP;                       // [DK]
    float* sQG = sGam + DK;                            // [C][DK]    (forward only)
    float* sAqk = sQG + C * DK;                        // [C][C]     (forward only)

    // blocks run (tile, head)-innermost over sequences ranked longest first
    const int64_t hg = (H - h_base) < Hg ? (H - h_base) : Hg;
    const int64_t tiles = DV / TW;
    const int64_t bid = blockIdx.x;
    const int64_t n = si.seq_of(bid / (hg * tiles));
    const int hl = (int)((bid / tiles) % hg);
    const int64_t h = h_base + hl;
    const int j0 = (int)(bid % tiles) * TW;
    const int tid = threadIdx.x, lane = tid & 31, wrp = tid >> 5;
    int64_t bos, eos;
    seq_range(si.cu, n, si.T_seq, si.T_total, bos, eos);
    const int64_t nchunks = si.chunk_count(n, eos - bos);
    const int64_t gc0 = si.chunk_start(n);

    const int64_t sidx = a.state_index(n, h);
    const float* h0p = (a.h0 && sidx >= 0) ? a.h0 + sidx * DK * DV : nullptr;
    float* hTp = (a.hT && sidx >= 0) ? a.hT + sidx * DK * DV : nullptr;
    // the state tile lives in registers: thread (warp w, lane) owns row c = 32 (w mod DK/32)
    // + lane and NJ consecutive columns (NJ = 16 for DK = 128, 8 for DK = 64)
    constexpr int RG = DK / 32, NJ = TW / (8 / RG);
    const int c = 32 * (wrp % RG) + lane, jb = NJ * (wrp / RG);
    float st[NJ];
#pragma unroll
    for (int x = 0; x < NJ; ++x) st[x] = h0p ? h0p[(int64_t)c * DV + j0 + jb + x] : 0.f;

    for (int64_t ch = 0; ch < nchunks; ++ch) {
        float* blk = ws + ((gc0 + ch) * Hg + hl) * kStride;
        const int64_t t0 = bos + ch * C;
        const int len = (int)((eos - t0) < C ? (eos - t0) : C);
        __syncthreads();                          // the previous chunk's reads are done
        for (int e = tid; e < C * DK / 4; e += blockDim.x) {
            reinterpret_cast<float4*>(sW)[e] = reinterpret_cast<const float4*>(blk + SimtWs<DK, DV>::W)[e];
            reinterpret_cast<float4*>(sKG)[e] = reinterpret_cast<const float4*>(blk + SimtWs<DK, DV>::KG)[e];
            if constexpr (!kBwd)
                reinterpret_cast<float4*>(sQG)[e] = reinterpret_cast<const float4*>(blk + SimtWs<DK, DV>::QG)[e];
        }
        if constexpr (!kBwd)
            for (int e = tid; e < C * C / 4; e += blockDim.x)
                reinterpret_cast<float4*>(sAqk)[e] = reinterpret_cast<const float4*>(blk + SimtWs<DK, DV>::Aqk)[e];
        for (int e = tid; e < C * TW; e += blockDim.x)
            sU[e] = blk[SimtWs<DK, DV>::Ut + (e / TW) * DV + j0 + (e % TW)];
        for (int cc = tid; cc < DK; cc += blockDim.x) sGam[cc] = blk[SimtWs<DK, DV>::Gam + cc];
#pragma unroll
        for (int x = 0; x < NJ; x += 4) {
            const float4 v4 = make_float4(st[x], st[x + 1], st[x + 2], st[x + 3]);
            *reinterpret_cast<float4*>(sS + c * kSP + jb + x) = v4;
            if constexpr (kBwd)
                *reinterpret_cast<float4*>(blk + BwdWs<DK, DV>::Sx + (int64_t)c * DV + j0 + jb + x) = v4;
        }
        __syncthreads();
        // U = Ut - W S: rows t = w + 8 r, column lane
        {
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = 0.f;
            rows8_mac<kSP>(acc, sW, DK, wrp, sS, DK, lane);
#pragma unroll
            for (int r = 0; r < 8; ++r) sU[(wrp + 8 * r) * TW + lane] -= acc[r];
        }
        __syncthreads();
        // O = scale (Q e^G) S + Aqk U   (the entry state; Aqk is zero above the diagonal)
        if constexpr (!kBwd) {
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = 0.f;
            rows8_mac<kSP>(acc, sQG, DK, wrp, sS, DK, lane);
            rows8_mac<TW>(acc, sAqk, C, wrp, sU, C, lane);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int t = wrp + 8 * r;
                if (t < len) IO<T>::store(out, ((t0 + t) * H + h) * DV + j0 + lane, acc[r]);
            }
        }
        // S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T U, in registers
        {
            const float gmc = sGam[c];
#pragma unroll
            for (int x = 0; x < NJ; ++x) st[x] *= gmc;
            for (int t = 0; t < C; ++t) {
                const float kg = sKG[t * DK + c];
#pragma unroll
                for (int x = 0; x < NJ; x += 4) {
                    const float4 u4 = *reinterpret_cast<const float4*>(sU + t * TW + jb + x);
                    st[x] += kg * u4.x;
                    st[x + 1] += kg * u4.y;
                    st[x + 2] += kg * u4.z;
                    st[x + 3] += kg * u4.w;
                }
            }
        }
    }
    if (hTp)
#pragma unroll
        for (int x = 0; x < NJ; ++x) hTp[(int64_t)c * DV + j0 + jb + x] = st[x];
}

}  // namespace kda
