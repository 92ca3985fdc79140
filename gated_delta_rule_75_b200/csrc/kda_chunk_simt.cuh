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

// 16-byte global -> shared copies that complete asynchronously (cp.async, L2 only),
// grouped by commit and waited for per thread: every thread's own copies are done
// after async_wait<N>() with at most N newer groups pending; a barrier after it makes
// them visible to the block.
__device__ __forceinline__ void async16(float* dst, const float* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// acc[i][x] += sum_k A[(row0 + i) * LDA + k] * B[k * LDB + 2 cp + x], i < 4, x < 2, K a
// multiple of 4: four rows by two columns per thread.  With the lanes of a warp split
// into two row groups (row0 four rows apart) and 16 column pairs, each 16-byte row load
// serves 16 lanes and each 8-byte column load two, so a k step costs two shared-memory
// wavefronts for eight FMAs when LDA keeps the two row groups on different banks.
template <int LDA, int LDB>
__device__ __forceinline__ void tile42_mac(float (&acc)[4][2], const float* A, int row0,
                                           const float* B, int K, int cp)
{
    for (int k = 0; k < K; k += 4) {
        float2 b[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) b[kk] = *reinterpret_cast<const float2*>(B + (k + kk) * LDB + 2 * cp);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 a = *reinterpret_cast<const float4*>(A + (row0 + i) * LDA + k);
            acc[i][0] += a.x * b[0].x + a.y * b[1].x + a.z * b[2].x + a.w * b[3].x;
            acc[i][1] += a.x * b[0].y + a.y * b[1].y + a.z * b[2].y + a.w * b[3].y;
        }
    }
}

// The same with A read transposed: acc[i][x] += sum_k A[k * LDA + row0 + i] * B[k * LDB + 2 cp + x]
// (the four rows of a thread are one 16-byte load per k).
template <int LDA, int LDB>
__device__ __forceinline__ void tile42t_mac(float (&acc)[4][2], const float* A, int row0,
                                            const float* B, int K, int cp)
{
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        const float2 bv = *reinterpret_cast<const float2*>(B + k * LDB + 2 * cp);
        const float4 a = *reinterpret_cast<const float4*>(A + k * LDA + row0);
        acc[0][0] += a.x * bv.x; acc[0][1] += a.x * bv.y;
        acc[1][0] += a.y * bv.x; acc[1][1] += a.y * bv.y;
        acc[2][0] += a.z * bv.x; acc[2][1] += a.z * bv.y;
        acc[3][0] += a.w * bv.x; acc[3][1] += a.w * bv.y;
    }
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
    return sizeof(float) * (size_t)(kChunk * (3 * DK + DV) + 2 * kChunk * kChunk + kChunk + 32 * DK + 64 * (DK + 4));
}
template <int DK, int DV, bool kBwd = false>
constexpr size_t simt_state_smem()
{
    return sizeof(float) * (size_t)((kBwd ? 1 : 2) * kChunk * (DK + 4) + kChunk * DK +
                                    (kBwd ? 0 : kChunk * (kChunk + 4)) + 2 * kChunk * kTW + DK * kSP + DK);
}


// ---------------------------------------------------------------------------
// step a + b: cumulative log-decay and intra-chunk transform
// ---------------------------------------------------------------------------
constexpr int kSimtPrepThreads = 512;   // 16 warps: one CTA per SM (shared memory), so more warps hide latency

// One 16-byte global load of I/O elements, widened to fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    using Raw = float4;
    static __device__ __forceinline__ void widen(const float4& r, float (&o)[4]) {
        o[0] = r.x; o[1] = r.y; o[2] = r.z; o[3] = r.w;
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    using Raw = uint4;
    static __device__ __forceinline__ void widen(const uint4& r, float (&o)[8]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {          // a bf16 is the high half of its fp32 value
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// Rows [C][D] of one (chunk, head) into shared memory as fp32: every 16-byte
// load of the thread is issued before the first one is used.
template <typename T, int D, int NT>
__device__ __forceinline__ void load_rows(float* dst, const T* __restrict__ src, int64_t t0,
                                          int len, int64_t H, int64_t h, int tid)
{
    using V = Vec16<T>;
    constexpr int PER_ROW = D / V::N, NV = kChunk * PER_ROW / NT;
    static_assert(kChunk * PER_ROW % NT == 0, "rows split evenly over the block");
    typename V::Raw r[NV];
#pragma unroll
    for (int x = 0; x < NV; ++x) {
        const int e = tid + x * NT, t = e / PER_ROW, c = (e % PER_ROW) * V::N;
        if (t < len) r[x] = *reinterpret_cast<const typename V::Raw*>(src + ((t0 + t) * H + h) * D + c);
        else r[x] = typename V::Raw{};
    }
#pragma unroll
    for (int x = 0; x < NV; ++x) {
        const int e = tid + x * NT, t = e / PER_ROW, c = (e % PER_ROW) * V::N;
        float o[V::N];
        V::widen(r[x], o);
#pragma unroll
        for (int i = 0; i < V::N; i += 4)
            *reinterpret_cast<float4*>(dst + t * D + c + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
    }
}

template <typename T, int DK, int DV, bool kBwd = false>
__global__ void __launch_bounds__(kSimtPrepThreads, 1)
chunk_prep_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ log_alpha, const float* __restrict__ beta,
                       SeqInfo si, int64_t H, int64_t h_base, int64_t Hg, float scale,
                       float* __restrict__ ws, int gate_scalar)
{
    griddep_wait();
    griddep_launch_dependents();
    constexpr int C = kChunk, NT = kSimtPrepThreads;
    extern __shared__ __align__(16) float smem[];
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
    float* sKvar = sQin + 16 * DK;    // [64][KVP] earlier rows (and the sub-chunk's own), referenced to it

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int64_t h = h_base + hl;
    int64_t n, t0, len64;
    if (!si.locate(gc, n, t0, len64)) return;
    const int len = (int)len64;
    const int tid = threadIdx.x, lane = tid & 31;

    load_rows<T, DK, NT>(sK, k, t0, len, H, h, tid);
    load_rows<T, DK, NT>(sQ, q, t0, len, H, h, tid);
    load_rows<T, DV, NT>(sV, v, t0, len, H, h, tid);
    if (gate_scalar) {
        for (int e = tid; e < C * DK; e += NT) {
            const int t = e / DK;
            sG[e] = t < len ? log_alpha[(t0 + t) * H + h] : 0.f;
        }
    } else {
        load_rows<float, DK, NT>(sG, log_alpha, t0, len, H, h, tid);
    }
    for (int t = tid; t < C; t += NT) sB[t] = t < len ? beta[(t0 + t) * H + h] : 0.f;
    __syncthreads();

    // (a) inclusive cumulative sum of log-decay per channel within the chunk
    if (tid < DK) {
        float run = 0.f;
        for (int t = 0; t < C; ++t) { run += sG[t * DK + tid]; sG[t * DK + tid] = run; }
    }
    __syncthreads();

    float* blk = ws + (gc * Hg + hl) * (kBwd ? BwdWs<DK, DV>::size : SimtWs<DK, DV>::size);
    // (b1) A (strictly lower, beta-weighted) and Aqk (lower incl. diagonal), one 16-row
    // sub-chunk of rows i at a time.  The exponential splits at the sub-chunk's first row f,
    // e^{G_i - G_f} e^{G_f - G_j}, so the sums are dot products of precomputed rows.  For
    // columns j before the sub-chunk both factors are <= 1.  Inside the diagonal block the
    // second factor is >= 1, bounded by the block's decay; where some channel decays by more
    // than 64 nats across the block (e^64 ~ 6e27, its inverse still a normal fp32 number)
    // that block is taken pairwise, e^{G_i - G_j} per channel, so any decay rate is exact.
    for (int e = tid; e < C * C; e += NT) {
        sA[e] = 0.f;
        sT[e] = 0.f;
        if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + e] = 0.f;
    }
    // pairwise diagonal blocks: threads 0..239 take the 120 pairs i > j of a 16-row block,
    // two threads per pair (one channel half each, partner = lane ^ 1); threads 240..255
    // take the 16 diagonal entries of Aqk, where the decay factor is 1; the rest idle
    constexpr int kPairThreads = 240, HALF = DK / 2;
    int pi = 0, pj = 0;
    if (tid < kPairThreads) {
        int m = tid >> 1;
        pi = 1;
        while (m >= pi) { m -= pi; ++pi; }
        pj = m;
    } else if (tid < 256) {
        pi = pj = tid - kPairThreads;
    }
    constexpr float kMaxBlockDecay = 64.f;
    for (int p = 0; p < C / 16; ++p) {
        const int f = 16 * p;
        // (this barrier also: zeros written, scratch rows free)
        const int pairwise = __syncthreads_or(
            tid < DK && fabsf(sG[f * DK + tid] - sG[(f + 15) * DK + tid]) > kMaxBlockDecay);
        for (int e = tid; e < 16 * DK; e += NT) {
            const int i = f + e / DK, c = e % DK;
            const float d = sG[i * DK + c] - sG[f * DK + c];
            const float x = expf(d);
            sKin[e] = sK[i * DK + c] * x;
            sQin[e] = sQ[i * DK + c] * x;
            if (!pairwise) sKvar[i * KVP + c] = sK[i * DK + c] * expf(-d);
        }
        for (int e = tid; e < f * DK; e += NT) {
            const int j = e / DK, c = e % DK;
            sKvar[j * KVP + c] = sK[e] * expf(sG[f * DK + c] - sG[e]);
        }
        __syncthreads();
        const int nu = pairwise ? p : p + 1;      // column blocks taken as dot products
        if (nu > 0) {  // row f + w of warp w, columns jg + 16 u (lane = 16 half + jg); lanes run
                       // along the columns (padded Kvar rows), the row is a broadcast; the two
                       // half-warps take one channel half each and meet by a shuffle
            const int r = tid >> 5, jg = lane & 15, i = f + r, c0 = (lane >> 4) * (DK / 2);
            float kk[4] = {0.f, 0.f, 0.f, 0.f}, qk[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c = c0; c < c0 + DK / 2; c += 4) {
                const float4 a = *reinterpret_cast<const float4*>(sKin + r * DK + c);
                const float4 q4 = *reinterpret_cast<const float4*>(sQin + r * DK + c);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (u < nu) {
                        const float4 kv = *reinterpret_cast<const float4*>(sKvar + (jg + 16 * u) * KVP + c);
                        kk[u] += a.x * kv.x + a.y * kv.y + a.z * kv.z + a.w * kv.w;
                        qk[u] += q4.x * kv.x + q4.y * kv.y + q4.z * kv.z + q4.w * kv.w;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                kk[u] += __shfl_xor_sync(0xffffffffu, kk[u], 16);
                qk[u] += __shfl_xor_sync(0xffffffffu, qk[u], 16);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = jg + 16 * u;
                if (lane < 16 && u < nu && j <= i) {   // (the diagonal block: its lower half only)
                    if (j < i) {
                        sA[i * C + j] = sB[i] * kk[u];
                        if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + i * C + j] = kk[u];
                    }
                    sT[i * C + j] = scale * qk[u];   // Aqk parked in sT for now
                }
            }
        }
        if (pairwise && tid < 256) {   // diagonal block, pairwise; the channel order is rotated
                                       // by the lane so that the 32 lanes of a warp hit 32 banks
            const int i = f + pi, j = f + pj;
            float dk_ = 0.f, dq_ = 0.f;
            if (tid < kPairThreads) {
                const int c0 = (tid & 1) * HALF;
                for (int cc = 0; cc < HALF; ++cc) {
                    const int c = c0 + (cc + lane) % HALF;
                    const float kj = sK[j * DK + c] * expf(sG[i * DK + c] - sG[j * DK + c]);
                    dk_ += sK[i * DK + c] * kj;
                    dq_ += sQ[i * DK + c] * kj;
                }
            } else {
                for (int cc = 0; cc < DK; ++cc) {
                    const int c = (cc + lane) % DK;
                    dq_ += sQ[i * DK + c] * sK[i * DK + c];
                }
            }
            const float ok = __shfl_xor_sync(0xffffffffu, dk_, 1);
            const float oq = __shfl_xor_sync(0xffffffffu, dq_, 1);
            if (tid < kPairThreads) {
                if ((tid & 1) == 0) {
                    dk_ += ok;
                    dq_ += oq;
                    sA[i * C + j] = sB[i] * dk_;
                    sT[i * C + j] = scale * dq_;
                    if constexpr (kBwd) blk[BwdWs<DK, DV>::Ap + i * C + j] = dk_;
                }
            } else {
                sT[i * C + i] = scale * dq_;
            }
        }
    }
    __syncthreads();

    for (int e = tid; e < C * C; e += NT) blk[SimtWs<DK, DV>::Aqk + e] = sT[e];
    // Q e^G (scaled), K e^{G_last - G}, e^{G_last}
    for (int e4 = tid; e4 < C * DK / 4; e4 += NT) {
        const int e = 4 * e4, c = e % DK;
        const float4 G = *reinterpret_cast<const float4*>(sG + e);
        const float4 Gl = *reinterpret_cast<const float4*>(sG + (C - 1) * DK + c);
        const float4 q4 = *reinterpret_cast<const float4*>(sQ + e);
        const float4 k4 = *reinterpret_cast<const float4*>(sK + e);
        *reinterpret_cast<float4*>(blk + SimtWs<DK, DV>::QG + e) =
            make_float4(scale * q4.x * expf(G.x), scale * q4.y * expf(G.y),
                        scale * q4.z * expf(G.z), scale * q4.w * expf(G.w));
        *reinterpret_cast<float4*>(blk + SimtWs<DK, DV>::KG + e) =
            make_float4(k4.x * expf(Gl.x - G.x), k4.y * expf(Gl.y - G.y),
                        k4.z * expf(Gl.z - G.z), k4.w * expf(Gl.w - G.w));
    }
    for (int c = tid; c < DK; c += NT) blk[SimtWs<DK, DV>::Gam + c] = expf(sG[(C - 1) * DK + c]);
    __syncthreads();

    // (b2) T = (I + A)^{-1} by 16 x 16 blocks.  Diagonal blocks: one column per thread
    // (threads 0..63), forward substitution in registers; the other threads clear the
    // blocks above the diagonal and scale K e^G and V by beta.
    if (tid < 64) {
        const int f = 16 * (tid >> 4), c = tid & 15;
        float col[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc += sA[(f + i) * C + f + j] * col[j];
            col[i] = (i == c) ? 1.f : -acc;       // zero above the diagonal (acc = 0 there)
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sT[(f + i) * C + f + c] = col[i];
    } else {
        for (int e = tid - 64; e < C * C; e += NT - 64) {
            const int i = e / C, j = e % C;
            if ((j >> 4) > (i >> 4)) sT[e] = 0.f;
        }
        // beta K e^G into sQ, beta V in place
        for (int e = tid - 64; e < C * DK; e += NT - 64) sQ[e] = sB[e / DK] * sK[e] * expf(sG[e]);
        for (int e = tid - 64; e < C * DV; e += NT - 64) sV[e] *= sB[e / DV];
    }
    // Off-diagonal blocks by distance d = p - r: T_pr = -T_pp sum_{m=r}^{p-1} A_pm T_mr,
    // whose factors all lie at distances below d.  Thread (a, b) < 256 owns entry (a, b) of
    // each block of the level; the partial sums go through sKin.
    {
        const int a = (tid >> 4) & 15, b = tid & 15;
        const bool act = tid < 256;
        float* sX = sKin;                         // [3][16][16]
        for (int d = 1; d < 4; ++d) {
            __syncthreads();                      // level d - 1 (or the diagonal) written
            for (int r = 0; act && r + d < 4; ++r) {
                const int p = r + d;
                float x = 0.f;
                for (int m = r; m < p; ++m) {
#pragma unroll
                    for (int l = 0; l < 16; l += 4) {
                        const float4 av = *reinterpret_cast<const float4*>(sA + (16 * p + a) * C + 16 * m + l);
                        x += av.x * sT[(16 * m + l) * C + 16 * r + b] + av.y * sT[(16 * m + l + 1) * C + 16 * r + b] +
                             av.z * sT[(16 * m + l + 2) * C + 16 * r + b] + av.w * sT[(16 * m + l + 3) * C + 16 * r + b];
                    }
                }
                sX[r * 256 + a * 16 + b] = x;
            }
            __syncthreads();
            for (int r = 0; act && r + d < 4; ++r) {
                const int p = r + d;
                float y = 0.f;
#pragma unroll
                for (int l = 0; l < 16; l += 4) {
                    const float4 tv = *reinterpret_cast<const float4*>(sT + (16 * p + a) * C + 16 * p + l);
                    y += tv.x * sX[r * 256 + l * 16 + b] + tv.y * sX[r * 256 + (l + 1) * 16 + b] +
                         tv.z * sX[r * 256 + (l + 2) * 16 + b] + tv.w * sX[r * 256 + (l + 3) * 16 + b];
                }
                sT[(16 * p + a) * C + 16 * r + b] = -y;
            }
        }
    }
    __syncthreads();

    if constexpr (kBwd) {                       // T and K e^G for the backward
        for (int e = tid; e < C * C; e += NT) blk[BwdWs<DK, DV>::Tm + e] = sT[e];
        for (int e = tid; e < C * DK; e += NT)
            blk[BwdWs<DK, DV>::KGm + e] = sK[e] * expf(sG[e]);
    }

    // (b3) [W | Ut] = T [beta K e^G | beta V], register-tiled: thread (g, cg) owns rows
    // g (which needs columns j <= g of T) and 63 - g (j <= 63 - g), so all threads do the
    // same number of products, and 16-byte column groups 4 cg + 64 u.
    {
        constexpr int NU = (DK + DV) / 64;
        const int g = tid >> 4, cg = tid & 15;
        const int row[2] = {g, 63 - g};
        const int jl = (g + 1 + 3) & ~3;
        const int jh = (64 - g + 3) & ~3;
        float4 acc[2][NU];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int u = 0; u < NU; ++u) acc[rr][u] = make_float4(0.f, 0.f, 0.f, 0.f);
        auto bcol = [&](int u, int j) -> float4 {
            return 64 * u < DK ? *reinterpret_cast<const float4*>(sQ + j * DK + 64 * u + 4 * cg)
                               : *reinterpret_cast<const float4*>(sV + j * DV + 64 * u - DK + 4 * cg);
        };
        auto step = [&](int j, const float (&tj)[2][4], int r0) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int u = 0; u < NU; ++u) {
                    const float4 bv = bcol(u, j + jj);
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        if (rr < r0) continue;
                        const float t = tj[rr][jj];
                        acc[rr][u].x += t * bv.x;
                        acc[rr][u].y += t * bv.y;
                        acc[rr][u].z += t * bv.z;
                        acc[rr][u].w += t * bv.w;
                    }
                }
        };
        for (int j = 0; j < jl; j += 4) {
            float tj[2][4];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const float4 t4 = *reinterpret_cast<const float4*>(sT + row[rr] * C + j);
                tj[rr][0] = t4.x; tj[rr][1] = t4.y; tj[rr][2] = t4.z; tj[rr][3] = t4.w;
            }
            step(j, tj, 0);
        }
        for (int j = jl; j < jh; j += 4) {
            float tj[2][4] = {};
            const float4 t4 = *reinterpret_cast<const float4*>(sT + row[1] * C + j);
            tj[1][0] = t4.x; tj[1][1] = t4.y; tj[1][2] = t4.z; tj[1][3] = t4.w;
            step(j, tj, 1);
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                float* dst = 64 * u < DK ? blk + SimtWs<DK, DV>::W + row[rr] * DK + 64 * u + 4 * cg
                                         : blk + SimtWs<DK, DV>::Ut + row[rr] * DV + 64 * u - DK + 4 * cg;
                *reinterpret_cast<float4*>(dst) = acc[rr][u];
            }
    }
}

// ---------------------------------------------------------------------------
// steps c + d: sequential state propagation and output, per 32-column dv tile
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV, bool kBwd = false>
__global__ void __launch_bounds__(256, kBwd ? 2 : 1)   // occupancy set by shared memory
chunk_state_simt_kernel(float* __restrict__ ws, PrefillArgs a, int64_t h_base, int64_t Hg)
{
    griddep_wait();
    griddep_launch_dependents();
    // kBwd: backward blocks; every chunk's entry state is saved (Sx) and
    // no output is written
    constexpr int64_t kStride = kBwd ? BwdWs<DK, DV>::size : SimtWs<DK, DV>::size;
    const SeqInfo& si = a.si;
    const int64_t H = a.H;
    T* __restrict__ out = (T*)a.out;
    constexpr int C = kChunk, TW = kTW, NT = 256;
    extern __shared__ __align__(16) float smem[];
    // (the backward walk writes no output: no Q e^G, no Aqk, and less shared memory)
    // row pitches DK + 4 and C + 4: the two row groups of a warp in tile42_mac (four rows
    // apart) land on different banks
    constexpr int WP = DK + 4, AP = C + 4;
    float* sW = smem;                                  // [C][WP]
    float* sKG = sW + C * WP;                          // [C][DK]
    float* sUb = sKG + C * DK;                         // 2 x [C][TW]  (chunk ch in buffer ch & 1)
    float* sS = sUb + 2 * C * TW;                      // [DK][kSP]  copy of the entry state
    float* sGam = sS + DK * kSP;                       // [DK]
    float* sQG = sGam + DK;                            // [C][WP]    (forward only)
    float* sAqk = sQG + C * WP;                        // [C][AP]    (forward only)

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
    auto block_of = [&](int64_t ch) { return ws + ((gc0 + ch) * Hg + hl) * kStride; };

    // Each buffer is refilled by cp.async as soon as its last reader of the previous
    // chunk is past a barrier, so the loads of chunk ch + 1 run under chunk ch's work:
    //   group U:  K e^{G_last-G}, e^{G_last} of ch and the Ut tile of ch + 1   (top of ch)
    //   group W:  W of ch + 1                                           (after U = Ut - W S)
    //   group QA: Q e^G and Aqk of ch + 1                               (after the output)
    // Every wait is "all but the newest group", and each is followed by a barrier.
    auto load_ut = [&](int64_t ch) {
        const float* src = block_of(ch) + SimtWs<DK, DV>::Ut + j0;
        float* dst = sUb + (ch & 1) * C * TW;
        for (int e = tid; e < C * TW / 4; e += NT)
            async16(dst + 4 * e, src + (e / (TW / 4)) * DV + 4 * (e % (TW / 4)));
    };
    auto load_kg = [&](int64_t ch) {
        const float* b = block_of(ch);
        for (int e = tid; e < C * DK / 4; e += NT) async16(sKG + 4 * e, b + SimtWs<DK, DV>::KG + 4 * e);
        for (int e = tid; e < DK / 4; e += NT) async16(sGam + 4 * e, b + SimtWs<DK, DV>::Gam + 4 * e);
    };
    auto load_w = [&](int64_t ch) {
        const float* b = block_of(ch) + SimtWs<DK, DV>::W;
        for (int e = tid; e < C * DK / 4; e += NT)
            async16(sW + (e / (DK / 4)) * WP + 4 * (e % (DK / 4)), b + 4 * e);
    };
    auto load_qa = [&](int64_t ch) {
        if constexpr (!kBwd) {
            const float* b = block_of(ch);
            for (int e = tid; e < C * DK / 4; e += NT)
                async16(sQG + (e / (DK / 4)) * WP + 4 * (e % (DK / 4)), b + SimtWs<DK, DV>::QG + 4 * e);
            for (int e = tid; e < C * C / 4; e += NT)
                async16(sAqk + (e / (C / 4)) * AP + 4 * (e % (C / 4)), b + SimtWs<DK, DV>::Aqk + 4 * e);
        }
    };

    const int64_t sidx = a.state_index(n, h);
    const float* h0p = (a.h0 && sidx >= 0) ? a.h0 + sidx * DK * DV : nullptr;
    float* hTp = (a.hT && sidx >= 0) ? a.hT + sidx * DK * DV : nullptr;
    // the state tile lives in registers: thread (warp w, lane) owns rows c_r = 64 (w mod DK/64)
    // + lane + 32 r, r < 2, and NJ consecutive columns (NJ = 8 for DK = 128, 4 for DK = 64):
    // per token of the update two key loads and NJ / 4 broadcast loads of U feed 2 NJ FMAs
    constexpr int RG = DK / 64, NJ = TW / (8 / RG);
    const int cb = 64 * (wrp % RG) + lane, jb = NJ * (wrp / RG);
    const int crow[2] = {cb, cb + 32};
    float st[2][NJ];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int x = 0; x < NJ; ++x) st[r][x] = h0p ? h0p[(int64_t)crow[r] * DV + j0 + jb + x] : 0.f;

    if (nchunks > 0) {
        load_ut(0);
        load_w(0);
    }
    async_commit();
    if (nchunks > 0) load_qa(0);
    async_commit();

    for (int64_t ch = 0; ch < nchunks; ++ch) {
        float* blk = block_of(ch);
        float* sU = sUb + (ch & 1) * C * TW;
        const int64_t t0 = bos + ch * C;
        const int len = (int)((eos - t0) < C ? (eos - t0) : C);
        async_wait<1>();                          // Ut and W of this chunk
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int x = 0; x < NJ; x += 4) {
                const float4 v4 = make_float4(st[r][x], st[r][x + 1], st[r][x + 2], st[r][x + 3]);
                *reinterpret_cast<float4*>(sS + crow[r] * kSP + jb + x) = v4;
                if constexpr (kBwd)
                    *reinterpret_cast<float4*>(blk + BwdWs<DK, DV>::Sx + (int64_t)crow[r] * DV + j0 + jb + x) = v4;
            }
        __syncthreads();                          // also: the previous chunk's state update is done
        load_kg(ch);
        if (ch + 1 < nchunks) load_ut(ch + 1);
        async_commit();
        // U = Ut - W S: thread (warp w, lane) takes rows 8 w + 4 (lane / 16) + i, i < 4,
        // and columns 2 (lane mod 16) + x, x < 2
        const int row0 = 8 * wrp + 4 * (lane >> 4), cp = lane & 15;
        {
            float acc[4][2] = {};
            tile42_mac<WP, kSP>(acc, sW, row0, sS, DK, cp);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float2* u2 = reinterpret_cast<float2*>(sU + (row0 + i) * TW + 2 * cp);
                const float2 u = *u2;
                *u2 = make_float2(u.x - acc[i][0], u.y - acc[i][1]);
            }
        }
        async_wait<1>();                          // Q e^G and Aqk of this chunk
        __syncthreads();
        if (ch + 1 < nchunks) load_w(ch + 1);
        async_commit();
        // O = scale (Q e^G) S + Aqk U   (the entry state; Aqk is zero above the diagonal)
        if constexpr (!kBwd) {
            float acc[4][2] = {};
            tile42_mac<WP, kSP>(acc, sQG, row0, sS, DK, cp);
            tile42_mac<AP, TW>(acc, sAqk, row0, sU, C, cp);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = row0 + i;
                if (t < len) {
                    const int64_t o = ((t0 + t) * H + h) * DV + j0 + 2 * cp;
                    IO<T>::store(out, o, acc[i][0]);
                    IO<T>::store(out, o + 1, acc[i][1]);
                }
            }
        }
        async_wait<1>();                          // K e^{G_last - G} and e^{G_last} of this chunk
        __syncthreads();
        if (ch + 1 < nchunks) load_qa(ch + 1);
        async_commit();
        // S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T U, in registers
        {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float gmc = sGam[crow[r]];
#pragma unroll
                for (int x = 0; x < NJ; ++x) st[r][x] *= gmc;
            }
            for (int t = 0; t < C; ++t) {
                const float kg0 = sKG[t * DK + crow[0]], kg1 = sKG[t * DK + crow[1]];
#pragma unroll
                for (int x = 0; x < NJ; x += 4) {
                    const float4 u4 = *reinterpret_cast<const float4*>(sU + t * TW + jb + x);
                    st[0][x] += kg0 * u4.x;
                    st[0][x + 1] += kg0 * u4.y;
                    st[0][x + 2] += kg0 * u4.z;
                    st[0][x + 3] += kg0 * u4.w;
                    st[1][x] += kg1 * u4.x;
                    st[1][x + 1] += kg1 * u4.y;
                    st[1][x + 2] += kg1 * u4.z;
                    st[1][x + 3] += kg1 * u4.w;
                }
            }
        }
        // the next chunk's barrier (after its Ut / W wait) orders these reads before any refill
    }
    async_wait<0>();
    if (hTp)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int x = 0; x < NJ; ++x) hTp[(int64_t)crow[r] * DV + j0 + jb + x] = st[r][x];
}

}  // namespace kda
