// Chunkwise backward pass of KDA, fp32 SIMT kernels.
//
// "Kimi Linear acaba de superar a la atencion completa en sus propios
// terminos" (section on the chunk training algorithm over the
// diagonal-plus-low-rank transition) says the chunk form exists for training;
// the pages print no gradient.  The gradients below differentiate the chunk
// equations (listed at the top of kda_chunk_simt.cu) in reverse; they are
// checked in fp64 against the oracle's token-by-token reverse mode.  Per chunk,
// with entry state S, exit-state gradient dS' and output gradient dO:
//
//   E  = U = T'(V - K_G S)          R  = V - K_G S      (T' = T diag(beta), K_G = K e^G)
//   dE = Aqk^T dO + Khat dS'        dR = T'^T dE        (Khat = K e^{G_last - G})
//   dS = Q_G^T dO + Diag(e^{G_last}) dS' - W^T dE       (Q_G = scale Q e^G, W = T' K_G)
//   dV = dR,  dK_G = -dR S^T,  dQ_G = dO S^T,  dKhat = E dS'^T
//   dT' = dE R^T,  dAqk = dO E^T (lower),  dbeta += colsum(T o dT'),
//   dA = -T^T (dT' diag(beta)) T^T (strictly lower),  dbeta += rowsum(dA o A'),
//   dA' = diag(beta) dA, then the pairwise products
//   A'_ij = sum_c k_ic k_jc e^{G_ic - G_jc} and Aqk_ij = scale sum_c q_ic k_jc e^{G_ic - G_jc}
//   give dk, dq and dG; G = cumsum(g) turns dG into dlog_alpha by a reverse cumsum.
//
// Kernels (all fp32, one (chunk, head) block of BwdWs floats each):
//   prep (kBwd)      the prefill prep, also saving T, A' and K e^G
//   walk (kBwd)      forward walk per (sequence, head, 32 columns), saving every entry state
//   bwd_state        reverse walk per (sequence, head, 32 columns): dE, dS across chunks,
//                    saving every exit-state gradient; dh0 at the start
//   bwd_dense1       per (chunk, head): E, R, dE, dR (dv written), sum_v S dS'
//   bwd_dense2       per (chunk, head, product): dK_G, dQ_G, dKhat, dT', dAqk
//   bwd_param        per (chunk, head): dbeta, dA, the pairwise terms, dq, dk, dlog_alpha
#include <cstring>

#include "kda_chunk_simt.cuh"

namespace kda {

constexpr int kBT = 256;          // threads of the backward kernels
constexpr int kPT = 512;          // threads of the parameter kernel (one CTA per SM: more warps)
constexpr int kD1T = 512;         // threads of dense pass 1 (likewise)

// ---------------------------------------------------------------------------
// reverse walk: per (sequence, head, 32-column tile)
// ---------------------------------------------------------------------------
constexpr int kAP = 68;           // row pitch of the transposed Aqk

// dS stays in registers across chunks: thread (warp w, lane) owns row c = 32 (w mod DK/32)
// + lane and NJ consecutive columns of the 32-column tile (NJ = 16 for DK = 128, 8 for 64);
// it is copied to shared memory once per chunk as the operand of Khat dS'.  Each operand
// has its own buffer, refilled by cp.async while the other phase of the chunk runs:
//   group A (Khat, Aqk of chunk ch - 1): issued after dE of chunk ch, used by dE of ch - 1
//   group B (W, Q_G, e^{G_last} of ch):  issued when chunk ch starts, used by its dS update
// and the dO tile of the next chunk is fetched into registers one chunk ahead.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kBT, 1)
chunk_bwd_state_kernel(float* __restrict__ ws, BackwardArgs b, int64_t h_base, int64_t Hg)
{
    using BW = BwdWs<DK, DV>;
    using SW = SimtWs<DK, DV>;
    using V = Vec16<T>;
    constexpr int C = kChunk, TW = kTW;
    constexpr int RG = DK / 32;       // groups of 32 rows
    constexpr int KP = DK + 4;        // row pitch of Khat (two row groups of tile42_mac on distinct banks)
    const SeqInfo& si = b.si;
    const int64_t H = b.H;
    extern __shared__ __align__(16) float smem[];
    float* sKh = smem;                // [C][KP]   K e^{G_last - G}
    float* sAqk = sKh + C * KP;       // [C][C]    Aqk (row r, column t), read as Aqk^T
    float* sW = sAqk + C * C;         // [C][DK]
    float* sQG = sW + C * DK;         // [C][DK]
    float* sGam = sQG + C * DK;       // [DK]
    float* sdO = sGam + DK;           // [C][TW]
    float* sdE = sdO + C * TW;        // [C][TW]
    float* sdS = sdE + C * TW;        // [DK][kSP]

    const int64_t hg = (H - h_base) < Hg ? (H - h_base) : Hg;
    const int64_t tiles = DV / TW;
    const int64_t bid = blockIdx.x;
    const int64_t n = bid / (hg * tiles);
    const int hl = (int)((bid / tiles) % hg);
    const int64_t h = h_base + hl;
    const int j0 = (int)(bid % tiles) * TW;
    const int tid = threadIdx.x, lane = tid & 31, wrp = tid >> 5;
    int64_t bos, eos;
    seq_range(si.cu, n, si.T_seq, si.T_total, bos, eos);
    const int64_t nchunks = si.chunk_count(n, eos - bos);
    const int64_t gc0 = si.chunk_start(n);
    const int64_t sidx = n * H + h;
    const T* __restrict__ dout = (const T*)b.dout;
    auto block_of = [&](int64_t ch) { return ws + ((gc0 + ch) * Hg + hl) * BW::size; };

    auto load_a = [&](int64_t ch) {
        const float* blk = block_of(ch);
        for (int e = tid; e < C * DK / 4; e += kBT)
            async16(sKh + (e / (DK / 4)) * KP + 4 * (e % (DK / 4)), blk + SW::KG + 4 * e);
        for (int e = tid; e < C * C / 4; e += kBT) async16(sAqk + 4 * e, blk + SW::Aqk + 4 * e);
    };
    auto load_b = [&](int64_t ch) {
        const float* blk = block_of(ch);
        for (int e = tid; e < C * DK / 4; e += kBT) {
            async16(sW + 4 * e, blk + SW::W + 4 * e);
            async16(sQG + 4 * e, blk + SW::QG + 4 * e);
        }
        for (int e = tid; e < DK / 4; e += kBT) async16(sGam + 4 * e, blk + SW::Gam + 4 * e);
    };
    // the dO tile [C][TW] of one chunk: NV 16-byte loads per thread, rows past the end as zeros
    constexpr int PER_ROW = TW / V::N, NV = C * PER_ROW / kBT;
    static_assert(C * PER_ROW % kBT == 0, "the dO tile splits evenly over the block");
    typename V::Raw rdo[NV];
    auto fetch_do = [&](int64_t ch) {
        const int64_t t0 = bos + ch * C;
        const int len = (int)((eos - t0) < C ? (eos - t0) : C);
#pragma unroll
        for (int x = 0; x < NV; ++x) {
            const int e = tid + x * kBT, t = e / PER_ROW, j = (e % PER_ROW) * V::N;
            if (t < len)
                rdo[x] = *reinterpret_cast<const typename V::Raw*>(dout + ((t0 + t) * H + h) * DV + j0 + j);
            else
                rdo[x] = typename V::Raw{};
        }
    };

    constexpr int NCW = 8 / RG;                       // warps sharing one row group
    constexpr int NJ = TW / NCW;                      // columns per thread
    const int c = 32 * (wrp % RG) + lane;
    const int jb = NJ * (wrp / RG);
    float ds[NJ];
#pragma unroll
    for (int x = 0; x < NJ; ++x)
        ds[x] = b.dhT ? b.dhT[sidx * DK * DV + (int64_t)c * DV + j0 + jb + x] : 0.f;

    if (nchunks > 0) {
        load_a(nchunks - 1);
        fetch_do(nchunks - 1);
    }
    async_commit();
    const int row0 = 8 * wrp + 4 * (lane >> 4), cp = lane & 15;   // tile42 rows and column pair
    for (int64_t ch = nchunks - 1; ch >= 0; --ch) {
        float* blk = block_of(ch);
        async_wait<0>();                              // Khat and Aqk of this chunk
        // this chunk's dO tile and exit-state gradient into shared memory (dS' also to the
        // workspace)
#pragma unroll
        for (int x = 0; x < NV; ++x) {
            const int e = tid + x * kBT, t = e / PER_ROW, j = (e % PER_ROW) * V::N;
            float o[V::N];
            V::widen(rdo[x], o);
#pragma unroll
            for (int i = 0; i < V::N; i += 4)
                *reinterpret_cast<float4*>(sdO + t * TW + j + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        }
#pragma unroll
        for (int x = 0; x < NJ; x += 4) {
            const float4 v4 = make_float4(ds[x], ds[x + 1], ds[x + 2], ds[x + 3]);
            *reinterpret_cast<float4*>(sdS + c * kSP + jb + x) = v4;
            *reinterpret_cast<float4*>(blk + BW::dSx + (int64_t)c * DV + j0 + jb + x) = v4;
        }
        __syncthreads();                              // also: the previous chunk's dS update is done
        load_b(ch);
        async_commit();
        if (ch > 0) fetch_do(ch - 1);
        // dE = Aqk^T dO + Khat dS': 4 x 2 register tiles
        {
            float acc[4][2] = {};
            tile42t_mac<C, TW>(acc, sAqk, row0, sdO, C, cp);
            tile42_mac<KP, kSP>(acc, sKh, row0, sdS, DK, cp);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float2*>(sdE + (row0 + i) * TW + 2 * cp) = make_float2(acc[i][0], acc[i][1]);
        }
        async_wait<0>();                              // W, Q_G, e^{G_last} of this chunk
        __syncthreads();
        if (ch > 0) load_a(ch - 1);
        async_commit();
        // dS = Diag(e^{G_last}) dS' + Q_G^T dO - W^T dE  (row c, columns jb .. jb + NJ - 1)
        {
            const float gmc = sGam[c];
#pragma unroll
            for (int x = 0; x < NJ; ++x) ds[x] *= gmc;
            for (int t = 0; t < C; ++t) {
                const float qg = sQG[t * DK + c], wv = sW[t * DK + c];
#pragma unroll
                for (int x = 0; x < NJ; x += 4) {
                    const float4 o4 = *reinterpret_cast<const float4*>(sdO + t * TW + jb + x);
                    const float4 e4 = *reinterpret_cast<const float4*>(sdE + t * TW + jb + x);
                    ds[x] += qg * o4.x - wv * e4.x;
                    ds[x + 1] += qg * o4.y - wv * e4.y;
                    ds[x + 2] += qg * o4.z - wv * e4.z;
                    ds[x + 3] += qg * o4.w - wv * e4.w;
                }
            }
        }
        __syncthreads();                              // dO and dE reads done before the next chunk's writes
    }
    async_wait<0>();
    if (b.dh0)
#pragma unroll
        for (int x = 0; x < NJ; ++x) b.dh0[sidx * DK * DV + (int64_t)c * DV + j0 + jb + x] = ds[x];
}

// ---------------------------------------------------------------------------
// dense pass 1: per (chunk, head)
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kD1T, 1)
chunk_bwd_dense1_kernel(float* __restrict__ ws, BackwardArgs b, int64_t h_base, int64_t Hg)
{
    using BW = BwdWs<DK, DV>;
    using SW = SimtWs<DK, DV>;
    constexpr int C = kChunk;
    const SeqInfo& si = b.si;
    const int64_t H = b.H;
    extern __shared__ __align__(16) float smem[];
    float* sW = smem;                 // [C][DK]
    float* sKG = sW + C * DK;         // [C][DK]   K e^G
    float* sKh = sKG + C * DK;        // [C][DK]   K e^{G_last - G}
    float* sAqkT = sKh + C * DK;      // [C][kAP]  Aqk transposed
    float* sTT = sAqkT + C * kAP;     // [C][kAP]  diag(beta) T^T
    float* sS = sTT + C * kAP;        // [DK][32]
    float* sdSn = sS + DK * kTW;      // [DK][32]
    float* sdO = sdSn + DK * kTW;     // [C][32]
    float* sdE = sdO + C * kTW;       // [C][32]
    float* sUt = sdE + C * kTW;       // [C][32]
    float* sV = sUt + C * kTW;        // [C][32]
    float* sB = sV + C * kTW;         // [C]

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int64_t h = h_base + hl;
    int64_t n, t0, len64;
    if (!si.locate(gc, n, t0, len64)) return;
    const int len = (int)len64;
    const int tid = threadIdx.x, lane = tid & 31, wrp = tid >> 5;
    float* blk = ws + (gc * Hg + hl) * BW::size;
    const T* __restrict__ dout = (const T*)b.dout;
    const T* __restrict__ v = (const T*)b.v;
    T* __restrict__ dv = (T*)b.dv;

    // the per-tile operands (S, dS', dO, V, Ut columns j0 .. j0 + 31) go through registers
    // one tile ahead, so their loads run under the previous tile's products
    constexpr int NS = DK * kTW / kD1T, NO = C * kTW / kD1T;
    float rS[NS], rdS[NS], rdO[NO], rV[NO], rU[NO];
    auto fetch = [&](int j0) {
#pragma unroll
        for (int x = 0; x < NS; ++x) {
            const int e = tid + x * kD1T, c = e / kTW, j = e % kTW;
            rS[x] = blk[BW::Sx + c * DV + j0 + j];
            rdS[x] = blk[BW::dSx + c * DV + j0 + j];
        }
#pragma unroll
        for (int x = 0; x < NO; ++x) {
            const int e = tid + x * kD1T, t = e / kTW, j = e % kTW;
            const bool ok = t < len;
            rdO[x] = ok ? IO<T>::load(dout, ((t0 + t) * H + h) * DV + j0 + j) : 0.f;
            rV[x] = ok ? IO<T>::load(v, ((t0 + t) * H + h) * DV + j0 + j) : 0.f;
            rU[x] = blk[SW::Ut + t * DV + j0 + j];
        }
    };
    fetch(0);
    for (int e = tid; e < C * DK / 4; e += kD1T) {
        reinterpret_cast<float4*>(sW)[e] = reinterpret_cast<const float4*>(blk + SW::W)[e];
        reinterpret_cast<float4*>(sKG)[e] = reinterpret_cast<const float4*>(blk + BW::KGm)[e];
        reinterpret_cast<float4*>(sKh)[e] = reinterpret_cast<const float4*>(blk + SW::KG)[e];
    }
    for (int t = tid; t < C; t += kD1T) sB[t] = t < len ? b.beta[(t0 + t) * H + h] : 0.f;
    __syncthreads();
    for (int e = tid; e < C * C; e += kD1T) {
        const int r = e / C, t = e % C;               // Aqk[r][t] -> AqkT[t][r]; T likewise,
        sAqkT[t * kAP + r] = blk[SW::Aqk + e];        // with row t of T^T scaled by beta_t
        sTT[t * kAP + r] = blk[BW::Tm + e] * sB[t];
    }
    float glS = 0.f;                                  // thread c < DK: sum_v S[c][v] dS'[c][v]

#pragma unroll 1
    for (int j0 = 0; j0 < DV; j0 += kTW) {
        __syncthreads();
#pragma unroll
        for (int x = 0; x < NS; ++x) {
            sS[tid + x * kD1T] = rS[x];
            sdSn[tid + x * kD1T] = rdS[x];
        }
#pragma unroll
        for (int x = 0; x < NO; ++x) {
            sdO[tid + x * kD1T] = rdO[x];
            sV[tid + x * kD1T] = rV[x];
            sUt[tid + x * kD1T] = rU[x];
        }
        __syncthreads();
        if (j0 + kTW < DV) fetch(j0 + kTW);
        if (tid < DK)                                 // (column order rotated by the row: no bank conflicts)
            for (int jj = 0; jj < kTW; ++jj) {
                const int j = (jj + tid) % kTW;
                glS += sS[tid * kTW + j] * sdSn[tid * kTW + j];
            }
        // rows w, w + NW, ... of this warp (NW warps); column j0 + lane
        constexpr int NW = kD1T / 32, NR = C / NW;
        float e8[NR], r8[NR], de8[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) { e8[r] = 0.f; r8[r] = 0.f; de8[r] = 0.f; }
        rows_mac<NR, NW, kTW>(e8, sW, DK, wrp, sS, DK, lane);        // W S
        rows_mac<NR, NW, kTW>(r8, sKG, DK, wrp, sS, DK, lane);       // K_G S
        rows_mac<NR, NW, kTW>(de8, sKh, DK, wrp, sdSn, DK, lane);    // Khat dS'
        rows_mac<NR, NW, kTW>(de8, sAqkT, kAP, wrp, sdO, C, lane);   // + Aqk^T dO
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const int t = wrp + NW * r;
            e8[r] = sUt[t * kTW + lane] - e8[r];
            r8[r] = sV[t * kTW + lane] - r8[r];
            sdE[t * kTW + lane] = de8[r];
            blk[BW::E + t * DV + j0 + lane] = e8[r];
            blk[BW::R + t * DV + j0 + lane] = r8[r];
            blk[BW::dE + t * DV + j0 + lane] = de8[r];
        }
        __syncthreads();
        // dR = diag(beta) T^T dE
        float dr8[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) dr8[r] = 0.f;
        rows_mac<NR, NW, kTW>(dr8, sTT, kAP, wrp, sdE, C, lane);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const int t = wrp + NW * r;
            blk[BW::dR + t * DV + j0 + lane] = dr8[r];
            if (t < len) IO<T>::store(dv, ((t0 + t) * H + h) * DV + j0 + lane, dr8[r]);
        }
    }
    if (tid < DK) blk[BW::dGlS + tid] = glS;
}

// ---------------------------------------------------------------------------
// dense pass 2: out[i][m] = sign * sum_v A[i][v] B[m][v], per (chunk, head, product)
//   0: dK_G = -dR S^T   1: dQ_G = dO S^T   2: dKhat = E dS'^T   (m < DK)
//   3: dT'  =  dE R^T   4: dAqk = dO E^T (kept for m <= i)       (m < C)
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kBT, 4)   // four CTAs per SM hide the tile loads (64 registers)
chunk_bwd_dense2_kernel(float* __restrict__ ws, BackwardArgs b, int64_t h_base, int64_t Hg)
{
    using BW = BwdWs<DK, DV>;
    constexpr int C = kChunk;
    constexpr int P = kTW + 1;        // padded pitch: 16 consecutive rows hit distinct banks
    const SeqInfo& si = b.si;
    const int64_t H = b.H;
    __shared__ float sA[C * P];
    __shared__ float sBm[DK * P];

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int job = blockIdx.z;
    const int64_t h = h_base + hl;
    int64_t n, t0, len64;
    if (!si.locate(gc, n, t0, len64)) return;
    const int len = (int)len64;
    const int tid = threadIdx.x;
    float* blk = ws + (gc * Hg + hl) * BW::size;
    const T* __restrict__ dout = (const T*)b.dout;

    const bool a_is_dO = job == 1 || job == 4;
    const float* Ag = job == 0 ? blk + BW::dR : job == 2 ? blk + BW::E : job == 3 ? blk + BW::dE : nullptr;
    const float* Bg = (job == 0 || job == 1) ? blk + BW::Sx : job == 2 ? blk + BW::dSx
                    : job == 3 ? blk + BW::R : blk + BW::E;
    const int M = job < 3 ? DK : C;                   // rows of B
    const float sign = job == 0 ? -1.f : 1.f;
    float* out = blk + (job == 0 ? BW::dKG : job == 1 ? BW::dQG : job == 2 ? BW::dKh
                        : job == 3 ? BW::dTp : BW::dAqk);

    // thread tile: rows ti + 16 r (r < 4), columns tm + 16 q (q < M / 16)
    const int ti = tid >> 4, tm = tid & 15;
    float acc[4][DK / 16];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < DK / 16; ++q) acc[r][q] = 0.f;
    const int nq = M / 16;

    for (int v0 = 0; v0 < DV; v0 += kTW) {
        __syncthreads();
        // 16-byte loads (four columns), scattered into the padded rows
        for (int e4 = tid; e4 < C * kTW / 4; e4 += kBT) {
            const int i = e4 / (kTW / 4), j = 4 * (e4 % (kTW / 4));
            float4 x;
            if (a_is_dO) {
                const bool ok = i < len;
                const int64_t o = ((t0 + i) * H + h) * DV + v0 + j;
                x = ok ? make_float4(IO<T>::load(dout, o), IO<T>::load(dout, o + 1),
                                     IO<T>::load(dout, o + 2), IO<T>::load(dout, o + 3))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                x = *reinterpret_cast<const float4*>(Ag + i * DV + v0 + j);
            }
            float* d = sA + i * P + j;
            d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
        }
        for (int e4 = tid; e4 < M * kTW / 4; e4 += kBT) {
            const int m = e4 / (kTW / 4), j = 4 * (e4 % (kTW / 4));
            const float4 x = *reinterpret_cast<const float4*>(Bg + m * DV + v0 + j);
            float* d = sBm + m * P + j;
            d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
        }
        __syncthreads();
        for (int j = 0; j < kTW; ++j) {
            float a[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = sA[(ti + 16 * r) * P + j];
#pragma unroll
            for (int q = 0; q < DK / 16; ++q) {
                if (q < nq) {
                    const float bb = sBm[(tm + 16 * q) * P + j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[r][q] += a[r] * bb;
                }
            }
        }
    }
    const int ld = job < 3 ? DK : C;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < DK / 16; ++q)
            if (q < nq) {
                const int i = ti + 16 * r, m = tm + 16 * q;
                float x = sign * acc[r][q];
                if (job == 4 && m > i) x = 0.f;
                out[i * ld + m] = x;
            }
}

// ---------------------------------------------------------------------------
// parameter gradients: per (chunk, head)
// ---------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kPT, 1)
chunk_bwd_param_kernel(float* __restrict__ ws, BackwardArgs b, int64_t h_base, int64_t Hg)
{
    using BW = BwdWs<DK, DV>;
    using SW = SimtWs<DK, DV>;
    constexpr int C = kChunk;
    const SeqInfo& si = b.si;
    const int64_t H = b.H;
    extern __shared__ __align__(16) float smem[];
    float* sK = smem;                 // [C][DK]
    float* sQ = sK + C * DK;          // [C][DK]
    float* sG = sQ + C * DK;          // [C][DK]  cumulative log-decay
    float* sdG = sG + C * DK;         // [C][DK]
    float* sAp = sdG + C * DK;        // [C][C]   A', then dA' = diag(beta) dA
    float* sdAqk = sAp + C * C;       // [C][C]   dAqk, then scale dAqk
    constexpr int TP = C + 1;         // row pitch of T: column walks over rows hit distinct banks
    float* sT = sdAqk + C * C;        // [C][TP]  T          } free after dA: scratch of the
    float* sdT = sT + C * TP;         // [C][C]   dT', dT    } pairwise terms, 2 x [48][DK]
    float* sX = sdT + C * C;          // [C][C]   dT T^T, dA }
    float* sB = sX + C * C;           // [C]
    float* sdB = sB + C;              // [C]

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int64_t h = h_base + hl;
    int64_t n, t0, len64;
    if (!si.locate(gc, n, t0, len64)) return;
    const int len = (int)len64;
    const int tid = threadIdx.x;
    float* blk = ws + (gc * Hg + hl) * BW::size;
    const T* __restrict__ q = (const T*)b.q;
    const T* __restrict__ k = (const T*)b.k;
    const float scale = b.scale;

    // inputs by 16-byte loads, all of a thread's issued before the first is used
    load_rows<T, DK, kPT>(sK, k, t0, len, H, h, tid);
    load_rows<T, DK, kPT>(sQ, q, t0, len, H, h, tid);
    if (b.gate_scalar) {
        for (int e = tid; e < C * DK; e += kPT) {
            const int t = e / DK;
            sG[e] = t < len ? b.log_alpha[(t0 + t) * H + h] : 0.f;
        }
    } else {
        load_rows<float, DK, kPT>(sG, b.log_alpha, t0, len, H, h, tid);
    }
    {
        constexpr int N4 = C * C / 4 / kPT;
        float4 rt[N4], ra[N4], rd[N4], rq[N4];
#pragma unroll
        for (int x = 0; x < N4; ++x) {
            const int e4 = tid + x * kPT;
            rt[x] = reinterpret_cast<const float4*>(blk + BW::Tm)[e4];
            ra[x] = reinterpret_cast<const float4*>(blk + BW::Ap)[e4];
            rd[x] = reinterpret_cast<const float4*>(blk + BW::dTp)[e4];
            rq[x] = reinterpret_cast<const float4*>(blk + BW::dAqk)[e4];
        }
#pragma unroll
        for (int x = 0; x < N4; ++x) {
            const int e = 4 * (tid + x * kPT), r = e / C, c = e % C;
            sT[r * TP + c] = rt[x].x; sT[r * TP + c + 1] = rt[x].y;
            sT[r * TP + c + 2] = rt[x].z; sT[r * TP + c + 3] = rt[x].w;
            reinterpret_cast<float4*>(sAp)[e / 4] = ra[x];
            reinterpret_cast<float4*>(sdT)[e / 4] = rd[x];
            reinterpret_cast<float4*>(sdAqk)[e / 4] = rq[x];
        }
    }
    for (int t = tid; t < C; t += kPT) sB[t] = t < len ? b.beta[(t0 + t) * H + h] : 0.f;
    __syncthreads();
    if (tid < DK) {                                   // G = cumsum(g) per channel
        float run = 0.f;
        for (int t = 0; t < C; ++t) { run += sG[t * DK + tid]; sG[t * DK + tid] = run; }
    }
    // dbeta_i = sum_r T[r][i] dT'[r][i]
    if (tid < C) {
        float acc = 0.f;
        for (int r = tid; r < C; ++r) acc += sT[r * TP + tid] * sdT[r * C + tid];
        sdB[tid] = acc;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kPT) sdT[e] *= sB[e % C];   // dT = dT' diag(beta)
    __syncthreads();
    // X = dT T^T:  X[r][j] = sum_m dT[r][m] T[j][m]  (T[j][m] = 0 for m > j)
    for (int e = tid; e < C * C; e += kPT) {
        const int r = e / C, j = e % C;
        float acc = 0.f;
        for (int m = 0; m <= j; ++m) acc += sdT[r * C + m] * sT[j * TP + m];
        sX[e] = acc;
    }
    __syncthreads();
    // dA[i][j] = -sum_r T[r][i] X[r][j]  (i > j; T[r][i] = 0 for r < i)
    constexpr int NU = C * C / kPT;
    float dA[NU];
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        const int e = tid + kPT * u, i = e / C, j = e % C;
        float acc = 0.f;
        if (j < i)
            for (int r = i; r < C; ++r) acc += sT[r * TP + i] * sX[r * C + j];
        dA[u] = -acc;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < NU; ++u) sX[tid + kPT * u] = dA[u];
    __syncthreads();
    // dbeta_i += sum_{j<i} dA[i][j] A'[i][j];  dA' = diag(beta) dA
    if (tid < C) {
        float acc = 0.f;
        for (int j = 0; j < tid; ++j) acc += sX[tid * C + j] * sAp[tid * C + j];
        sdB[tid] += acc;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kPT) sAp[e] = sB[e / C] * sX[e];
    __syncthreads();

    // Pairwise terms, sub-chunk by sub-chunk (16 rows).  For the rows i of sub-chunk p,
    // with L = scale dAqk:
    //   X1 = sum_{j<i}  dA'_ij k_j e^{G_i - G_j}     X3 = sum_{j<=i} L_ij k_j e^{G_i - G_j}
    //   X2 = sum_{j>i}  dA'_ji k_j e^{G_j - G_i}     X4 = sum_{j>=i} L_ji q_j e^{G_j - G_i}
    // then dk = X1 + X2 + X4, dq = X3, dG = k (X1 - X2 - X4) + q X3.  Off the diagonal
    // block the exponential splits at the sub-chunk boundary into two factors <= 1,
    // e^{G_i - G_f} e^{G_f - G_j} (f = first row, j before it) and e^{G_j - G_e} e^{G_e - G_i}
    // (e = last row, j after it), so those sums are products with Z = k e^{G_f - G},
    // k e^{G - G_e}, q e^{G - G_e}; inside the diagonal block they are taken pairwise.
    const float* dKG = blk + BW::dKG;
    const float* dQG = blk + BW::dQG;
    const float* dKh = blk + BW::dKh;
    const float* gam = blk + SW::Gam;
    for (int e = tid; e < C * C; e += kPT) sdAqk[e] *= scale;
    constexpr int NG = kPT / 16;                      // channel groups (lanes along channels)
    constexpr int NM = DK / NG;                       // channels per thread
    const int ti = tid / NG, tc = tid % NG;           // row within the sub-chunk, channel group
    float* Z1 = sT;                                   // [48][DK]
    float* Z2 = sT + 48 * DK;                         // [48][DK]
    for (int p = 0; p < 4; ++p) {
        const int f = 16 * p, el = f + 15, nu = C - 1 - el;
        const int i = f + ti;
        float x1[NM], x2[NM], x3[NM], x4[NM];
        __syncthreads();                              // scratch free, dA', L final
        for (int e = tid; e < f * DK; e += kPT) {
            const int c = e % DK;
            Z1[e] = sK[e] * expf(sG[f * DK + c] - sG[e]);
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < NM; ++m) { x1[m] = 0.f; x3[m] = 0.f; }
        for (int j = 0; j < f; ++j) {
            const float a1 = sAp[i * C + j], a3 = sdAqk[i * C + j];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const float z = Z1[j * DK + tc + NG * m];
                x1[m] += a1 * z;
                x3[m] += a3 * z;
            }
        }
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const int c = tc + NG * m;
            const float fac = expf(sG[i * DK + c] - sG[f * DK + c]);
            x1[m] *= fac;
            x3[m] *= fac;
        }
        for (int j = f; j <= i; ++j) {                // diagonal block, j <= i
            const float a1 = (j < i) ? sAp[i * C + j] : 0.f, a3 = sdAqk[i * C + j];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const int c = tc + NG * m;
                const float kz = sK[j * DK + c] * expf(sG[i * DK + c] - sG[j * DK + c]);
                x1[m] += a1 * kz;
                x3[m] += a3 * kz;
            }
        }
        __syncthreads();                              // Z1 is refilled below
        for (int e = tid; e < nu * DK; e += kPT) {
            const int j = el + 1 + e / DK, c = e % DK;
            const float ex = expf(sG[j * DK + c] - sG[el * DK + c]);
            Z1[e] = sK[j * DK + c] * ex;
            Z2[e] = sQ[j * DK + c] * ex;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < NM; ++m) { x2[m] = 0.f; x4[m] = 0.f; }
        for (int jj = 0; jj < nu; ++jj) {
            const int j = el + 1 + jj;
            const float a2 = sAp[j * C + i], a4 = sdAqk[j * C + i];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                x2[m] += a2 * Z1[jj * DK + tc + NG * m];
                x4[m] += a4 * Z2[jj * DK + tc + NG * m];
            }
        }
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const int c = tc + NG * m;
            const float fac = expf(sG[el * DK + c] - sG[i * DK + c]);
            x2[m] *= fac;
            x4[m] *= fac;
        }
        for (int j = i; j <= el; ++j) {               // diagonal block, j >= i
            const float a2 = (j > i) ? sAp[j * C + i] : 0.f, a4 = sdAqk[j * C + i];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const int c = tc + NG * m;
                const float ex = expf(sG[j * DK + c] - sG[i * DK + c]);
                x2[m] += a2 * sK[j * DK + c] * ex;
                x4[m] += a4 * sQ[j * DK + c] * ex;
            }
        }
        // gradients of element (i, c): the pairwise part and the elementwise terms
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const int c = tc + NG * m, e = i * DK + c;
            const float gi = sG[e], ki = sK[e], qi = sQ[e];
            const float eg = expf(gi), egl = expf(sG[(C - 1) * DK + c] - gi);
            const float dqg = dQG[e], dkg = dKG[e], dkh = dKh[e];
            const float dk = x1[m] + x2[m] + x4[m] + egl * dkh + eg * dkg;
            const float dq = x3[m] + scale * eg * dqg;
            sdG[e] = ki * (x1[m] - x2[m] - x4[m]) + qi * x3[m] + scale * qi * eg * dqg +
                     ki * eg * dkg - ki * egl * dkh;
            if (i < len) {
                const int64_t dst = ((t0 + i) * H + h) * DK + c;
                IO<T>::store((T*)b.dq, dst, dq);
                IO<T>::store((T*)b.dk, dst, dk);
            }
        }
    }
    __syncthreads();
    // dG_last = sum_i dKhat o Khat + e^{G_last} sum_v S dS'; dlog_alpha = reverse cumsum of dG
    if (tid < DK) {
        const int c = tid;
        const float gl = sG[(C - 1) * DK + c];
        float acc = gam[c] * blk[BW::dGlS + c];
        for (int i = 0; i < C; ++i) acc += dKh[i * DK + c] * sK[i * DK + c] * expf(gl - sG[i * DK + c]);
        float run = acc;
        for (int i = C - 1; i >= 0; --i) {
            run += sdG[i * DK + c];
            if (b.gate_scalar) sdG[i * DK + c] = run;
            else if (i < len) b.dlog_alpha[((t0 + i) * H + h) * DK + c] = run;
        }
    }
    if (b.gate_scalar) {                              // one gate per (token, head): channel sum
        __syncthreads();
        if (tid < len) {
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc += sdG[tid * DK + (c + tid) % DK];
            b.dlog_alpha[(t0 + tid) * H + h] = acc;
        }
    }
    if (tid < len) b.dbeta[(t0 + tid) * H + h] = sdB[tid];
}

template <int DK, int DV>
constexpr size_t bwd_state_smem() { return sizeof(float) * (size_t)(kChunk * (DK + 4) + kChunk * kChunk + 2 * kChunk * DK + DK + 2 * kChunk * kTW + DK * kSP); }
template <int DK, int DV>
constexpr size_t bwd_dense1_smem() { return sizeof(float) * (size_t)(3 * kChunk * DK + 2 * kChunk * kAP + 2 * DK * kTW + 4 * kChunk * kTW + kChunk); }
template <int DK, int DV>
constexpr size_t bwd_param_smem() { return sizeof(float) * (size_t)(4 * kChunk * DK + 5 * kChunk * kChunk + 3 * kChunk); }

template <typename T, int DK, int DV>
static cudaError_t run_bwd_t(const BackwardArgs& b, float* ws, int64_t Hg, cudaStream_t st)
{
    static std::atomic<uint64_t> attrs_done{0};
    cudaError_t e = once_per_device(attrs_done, [] {
        const int mx = cudaFuncAttributeMaxDynamicSharedMemorySize;
        cudaError_t r;
        if ((r = cudaFuncSetAttribute(chunk_prep_simt_kernel<T, DK, DV, true>, (cudaFuncAttribute)mx,
                                      (int)simt_prep_smem<DK, DV>())))
            return r;
        if ((r = cudaFuncSetAttribute(chunk_state_simt_kernel<T, DK, DV, true>, (cudaFuncAttribute)mx,
                                      (int)simt_state_smem<DK, DV, true>())))
            return r;
        if ((r = cudaFuncSetAttribute(chunk_bwd_state_kernel<T, DK, DV>, (cudaFuncAttribute)mx,
                                      (int)bwd_state_smem<DK, DV>())))
            return r;
        if ((r = cudaFuncSetAttribute(chunk_bwd_dense1_kernel<T, DK, DV>, (cudaFuncAttribute)mx,
                                      (int)bwd_dense1_smem<DK, DV>())))
            return r;
        return cudaFuncSetAttribute(chunk_bwd_param_kernel<T, DK, DV>, (cudaFuncAttribute)mx,
                                    (int)bwd_param_smem<DK, DV>());
    });
    if (e) return e;
    const SeqInfo& si = b.si;
    // the forward pieces see the same inputs through a PrefillArgs view
    PrefillArgs a;
    memset(&a, 0, sizeof(a));
    a.q = b.q; a.k = b.k; a.v = b.v; a.log_alpha = b.log_alpha; a.beta = b.beta; a.h0 = b.h0;
    a.out = nullptr; a.hT = nullptr; a.si = si; a.H = b.H; a.dk = DK; a.dv = DV;
    a.scale = b.scale; a.io = b.io; a.slots = nullptr; a.P = 0; a.err = nullptr;
    a.gate_scalar = false;
    for (int64_t hb = 0; hb < b.H; hb += Hg) {
        const int64_t hg = (b.H - hb) < Hg ? (b.H - hb) : Hg;
        const dim3 gchunk((unsigned)si.chunks_upper, (unsigned)hg);
        if (si.chunks_upper > 0) {
            LaunchScope scope(st, K_PREP_SIMT);
            chunk_prep_simt_kernel<T, DK, DV, true><<<gchunk, kSimtPrepThreads, simt_prep_smem<DK, DV>(), st>>>(
                (const T*)b.q, (const T*)b.k, (const T*)b.v, b.log_alpha, b.beta, si, b.H, hb, Hg,
                b.scale, ws, b.gate_scalar ? 1 : 0);
            if ((e = cudaGetLastError())) return e;
        }
        const dim3 gwalk((unsigned)(si.N * hg * (DV / kTW)));
        {
            LaunchScope scope(st, K_STATE_SIMT);
            chunk_state_simt_kernel<T, DK, DV, true><<<gwalk, 256, simt_state_smem<DK, DV, true>(), st>>>(
                ws, a, hb, Hg);
            if ((e = cudaGetLastError())) return e;
        }
        {
            LaunchScope scope(st, K_BWD_STATE);
            chunk_bwd_state_kernel<T, DK, DV><<<gwalk, kBT, bwd_state_smem<DK, DV>(), st>>>(ws, b, hb, Hg);
            if ((e = cudaGetLastError())) return e;
        }
        if (si.chunks_upper > 0) {
            {
                LaunchScope scope(st, K_BWD_DENSE1);
                chunk_bwd_dense1_kernel<T, DK, DV><<<gchunk, kD1T, bwd_dense1_smem<DK, DV>(), st>>>(
                    ws, b, hb, Hg);
                if ((e = cudaGetLastError())) return e;
            }
            {
                LaunchScope scope(st, K_BWD_DENSE2);
                const dim3 g5((unsigned)si.chunks_upper, (unsigned)hg, 5);
                chunk_bwd_dense2_kernel<T, DK, DV><<<g5, kBT, 0, st>>>(ws, b, hb, Hg);
                if ((e = cudaGetLastError())) return e;
            }
            {
                LaunchScope scope(st, K_BWD_PARAM);
                chunk_bwd_param_kernel<T, DK, DV><<<gchunk, kPT, bwd_param_smem<DK, DV>(), st>>>(
                    ws, b, hb, Hg);
                if ((e = cudaGetLastError())) return e;
            }
        }
    }
    return cudaSuccess;
}

template <typename T>
static cudaError_t run_bwd_d(const BackwardArgs& b, float* ws, int64_t Hg, cudaStream_t st)
{
    if (b.dk_ == 128 && b.dv_ == 128) return run_bwd_t<T, 128, 128>(b, ws, Hg, st);
    if (b.dk_ == 128 && b.dv_ == 64) return run_bwd_t<T, 128, 64>(b, ws, Hg, st);
    if (b.dk_ == 64 && b.dv_ == 128) return run_bwd_t<T, 64, 128>(b, ws, Hg, st);
    return run_bwd_t<T, 64, 64>(b, ws, Hg, st);
}

int64_t bwd_ws_floats_per_chunk(int dk, int dv)
{
    if (dk == 128 && dv == 128) return BwdWs<128, 128>::size;
    if (dk == 128 && dv == 64) return BwdWs<128, 64>::size;
    if (dk == 64 && dv == 128) return BwdWs<64, 128>::size;
    return BwdWs<64, 64>::size;
}

cudaError_t run_backward_simt(const BackwardArgs& b, float* ws, int64_t Hg, cudaStream_t st)
{
    if (b.io == KDA_IO_F32) return run_bwd_d<float>(b, ws, Hg, st);
    return run_bwd_d<__nv_bfloat16>(b, ws, Hg, st);
}

}  // namespace kda
