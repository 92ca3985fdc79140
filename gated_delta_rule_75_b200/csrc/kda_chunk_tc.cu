// Chunkwise KDA prefill on the sm_100a tensor cores (bf16 I/O, dk = dv = 128).
//
// Same chunk equations as the SIMT path (derived by unrolling the per-token
// step of "Kimi Delta Attention: la atencion lineal detras de Kimi K2 y
// Qwen3", section "Como funciona Kimi Delta Attention paso a paso"; the
// chunkwise DPLR form is the one "Kimi Linear acaba de superar a la atencion
// completa en sus propios terminos" says the method trains with), with
// T' = (I + A)^{-1} diag(beta):
//
//   A_ij   = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}   (i > j)
//   Aqk_ij = sum_c q_ic k_jc e^{G_ic - G_jc}          (i >= j)
//   W = T' (K e^G),  U = T' V - W S,  O = scale ((Q e^G) S + Aqk U),
//   S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T U
//
// Kernel `chunk_prep_tc` (one CTA per (chunk, head), steps a and b): TMA loads
//   k and q (128B-swizzled) and log_alpha; cumulative decay in the log2 domain;
//   the products behind A and Aqk as tcgen05 MMAs whose exponential factors are
//   referenced to 16-token sub-chunk starts (every factor <= 1 except
//   e^{G_f - G_j} inside a sub-chunk, bounded by 16 tokens of decay); the
//   diagonal 16x16 blocks of (I + A)^{-1} by fp32 forward substitution and the
//   off-diagonal blocks by tf32 mma.sync block products; W = T' (K e^G) as a
//   tcgen05 MMA.  It writes one operand image per (chunk, head), already in the
//   128B-swizzled shared-memory layout the state kernel's MMAs read.
// Kernel `chunk_prep_gdn_tc` (Gated DeltaNet, one gate per (token, head)): the same
//   image from two plain MMAs (k k^T, k q^T) and per-token scalings, since a scalar
//   decay factors out of the key products; three CTAs per SM.
// Kernel `chunk_state_tc` (one CTA per (sequence, head), steps c and d): walks
//   the chunks in order with S^T (dv x dk, fp32) resident in tensor memory and
//   a bf16 copy in shared memory as the MMA operand; each chunk's image (bulk
//   copy) and its v tile (TMA) are double-buffered.  Per chunk:
//     U^T = V^T T'^T + S^T (-W)^T             (fp32 in TMEM)
//     O^T = S^T (Q e^G)^T
//     S^T += U^T (K e^{G_last - G}),  O^T += U^T Aqk^T
//   then S^T is copied to bf16 for the next chunk and scaled by the next
//   chunk's e^{G_last} in TMEM, and O leaves through a shared-memory tile (one
//   tensor store per whole chunk).  Eight worker warps do the TMEM and SIMT work;
//   one thread of a ninth warp issues every MMA and copy, and the two sides meet
//   only on mbarriers, so the issuer's waits on the tensor pipe hold back no worker.
// Every mbarrier wait is bounded; on a timeout the CTA records it in the
// workspace error word, drains its own copies and frees its TMEM.
#include <cstring>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tma.cuh"
#include "kda_umma.cuh"
#include "kda_tc_util.cuh"

namespace kda {

using namespace umma;
using namespace tcu;

namespace tc {

constexpr int C = 64;
constexpr int D = 128;     // dk = dv = 128
constexpr float kLog2e = 1.4426950408889634f;
// Decay range of the 16-token references (log2 units): a factor e^{G_f - G_j} with j in
// the 16-token block that starts at f stays below 2^116 when no channel decays by more
// than e^-80 over the block's 15 steps (the prep reports a block past this).
constexpr float kRangeLog2 = 80.f * kLog2e;

// Operand image of one (chunk, head), byte offsets (all 1024-aligned).
constexpr uint32_t IMG_W = 0;          // -W^T        MN-major B: 128 channel rows x 64 tokens
constexpr uint32_t IMG_QG = 16384;     // Q e^G       K-major B: 64 token rows x 128 ch (2 K-blocks)
constexpr uint32_t IMG_B2 = 32768;     // MN-major B, K = 64 token rows: [Aqk^T | K e^{Gl-G}] (3 x 64)
constexpr uint32_t IMG_T = 57344;      // T' = T diag(beta), K-major: 64 rows x 64
constexpr uint32_t IMG_GAM = 65536;    // e^{G_last}, fp32 [128]
constexpr uint32_t IMG_BYTES = 66560;

// Kvar rows: variant p holds key rows 0 .. 16p+15 referenced to token 16p.
__device__ __constant__ int kVoff[4] = {0, 16, 48, 96};

// ---------------------------------------------------------------------------
// prep kernel shared memory (bytes from a 1024-aligned base)
// ---------------------------------------------------------------------------
constexpr int PT = 256;                // threads
constexpr int AP = 68;                 // row pitch (floats) of the fp32 A and T matrices
constexpr uint32_t P_K = 0;            // k, MN-major [t][c] image (TMA, swizzled); later K e^G   16 KB
constexpr uint32_t P_Q = 16384;        // q, same layout (TMA); later the T' bf16 image           16 KB
constexpr uint32_t P_G = 32768;        // fp32 log_alpha -> G: 4 swizzled slabs of 32 channels   32 KB
constexpr uint32_t P_KQ = 65536;       // K-major B: [Kin_p; Qin_p] x 4, one K-block             16 KB
constexpr uint32_t P_KV = 81920;       // K-major A: Kvar rows (160), one K-block                20 KB
constexpr uint32_t P_A = 65536;        // fp32 A [64][68] (aliases KQ/KV after the strips)       17 KB
constexpr uint32_t P_T = P_A + 64 * AP * 4;   // fp32 T [64][68]                                 17 KB
constexpr uint32_t P_VEC = 102400;     // per-channel vectors: egf[4], eglf[4], dvec[6]          8 KB
constexpr int VP = 144;                // floats per vector: 4 pad floats after every 32 channels
constexpr uint32_t P_BETA = P_VEC + 14 * VP * 4;   // beta [64], then the scalar gates [64]
constexpr uint32_t P_BYTES = P_BETA + 512;
constexpr uint32_t P_SMEM = P_BYTES + 1024 + 64;
static_assert(P_T + 64 * AP * 4 <= P_VEC, "A/T overlap the vectors");

// Index of channel c in a padded per-channel vector: the 8-channel groups that a
// quarter-warp reads (32 channels apart) fall in distinct banks.
__device__ __forceinline__ int vidx(int c) { return c + 4 * (c >> 5); }

// Byte offset of G[t][c] in the four 128B-swizzled slabs of 32 fp32 channels.
__device__ __forceinline__ uint32_t g_off(int t, int c)
{
    return (uint32_t)(c >> 5) * 8192u + (uint32_t)t * 128u +
           ((uint32_t)(((c & 31) >> 2) ^ (t & 7)) << 4) + (uint32_t)(c & 3) * 4u;
}

struct PrepMaps {
    CUtensorMap k, q, g;
};

// Shared tail of the prep kernels, after A (fp32, strictly lower, beta-scaled rows, pitch
// AP) is in sA and K e^G (bf16, MN-major image rows) in P_K (sT: room for T, pitch AP): T = (I + A)^{-1}, T' = T diag(beta) as a
// bf16 K-major image (in P_Q and in the workspace), and W = -T' (K e^G) by one MMA whose
// completion is phase `parity` of `bar`; W goes to the workspace image.  `after_mma()` runs in
// every thread once that MMA has completed (its operands in P_Q and P_K are no longer read).
// The inverse runs on warps 0-3; warps 4-7 run `side()` meanwhile (work that touches none of
// A, T, beta or the operands here), whose result every thread gets in `side_ok`.
// Returns false when the bounded wait gave up.
template <bool kSplit, typename AfterMma, typename Side>
__device__ __forceinline__ bool prep_tail(unsigned char* sm, unsigned char* img, float* sA, float* sT,
                                          const float* sB, uint32_t tmem, uint64_t* bar,
                                          uint32_t parity, int* err, AfterMma after_mma, Side side,
                                          bool& side_ok)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int sp = w & 3;                          // TMEM lane quarter of this warp
    // barrier of the warps that take part in the inverse: 0-3 with kSplit, else all
    auto inv_sync = [] {
        if constexpr (kSplit) bar_sync_named(1, 128);
        else __syncthreads();
    };
    bool mine = true;
    if (kSplit && w >= 4) {
        mine = side();
    } else {
        // ---- (b2) T = (I + A)^{-1}: diagonal 16x16 blocks by forward substitution,
        // one column per thread, held in registers
        if (tid < C) {
            const int b = tid >> 4, cc = tid & 15, o = 16 * b;
            float tcol[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc0 = 0.f, acc1 = 0.f;            // two chains: half the dependent adds
#pragma unroll
                for (int m = 0; m < r; ++m) {
                    if (m & 1) acc1 += sA[(o + r) * AP + o + m] * tcol[m];
                    else acc0 += sA[(o + r) * AP + o + m] * tcol[m];
                }
                tcol[r] = (r == cc) ? 1.f : ((r < cc) ? 0.f : -(acc0 + acc1));
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sT[(o + r) * AP + o + cc] = tcol[r];
        }
        inv_sync();
        // off-diagonal blocks, 32 x 32 recursion (X blocks are parked in the unused
        // upper blocks of A):
        //   level 1 (warps 0, 1): T_10 = -T_11 A_10 T_00,  T_32 = -T_33 A_32 T_22
        //   level 2 (warps 0-3): X = A_21 T_1 (rows 2..3, cols 0..1), then T_21 = -T_2 X
        auto Ab = [&](int r, int c) { return sA + (16 * r) * AP + 16 * c; };
        auto Tb = [&](int r, int c) { return sT + (16 * r) * AP + 16 * c; };
        if (w < 2) {
            const int p = 2 * w + 1, r = 2 * w;
            float acc[2][4] = {};
            mma16x16x16_tf32<AP>(acc, Ab(p, r), Tb(r, r), l);
            store16x16<AP>(Ab(r, p), acc, 1.f, l);
            __syncwarp();
            float acc2[2][4] = {};
            mma16x16x16_tf32<AP>(acc2, Tb(p, p), Ab(r, p), l);
            store16x16<AP>(Tb(p, r), acc2, -1.f, l);
        }
        inv_sync();
        if (w < 4) {
            const int p = 2 + (w >> 1), r = w & 1;       // X_pr = sum_{m=r..1} A_pm T_mr
            float acc[2][4] = {};
            for (int m = r; m < 2; ++m) mma16x16x16_tf32<AP>(acc, Ab(p, m), Tb(m, r), l);
            store16x16<AP>(Ab(r, p), acc, 1.f, l);
        }
        inv_sync();
        if (w < 4) {
            const int p = 2 + (w >> 1), r = w & 1;       // T_pr = -sum_{m=2..p} T_pm X_mr
            float acc[2][4] = {};
            for (int m = 2; m <= p; ++m) mma16x16x16_tf32<AP>(acc, Tb(p, m), Ab(r, m), l);
            store16x16<AP>(Tb(p, r), acc, -1.f, l);
        }
    }
    if constexpr (kSplit) {
        side_ok = __syncthreads_and(mine ? 1 : 0) != 0;
    } else {
        __syncthreads();
        side_ok = true;
    }
    // T' = T diag(beta) in bf16: K-major image (rows i, K = j), in smem and in the workspace.
    // Blocks above the diagonal are zero (never written in sT); the diagonal blocks already
    // hold zeros above their diagonal, and the blocks below are complete.
    for (int e = tid; e < C * 8; e += PT) {
        const int i = e >> 3, cb = e & 7;
        uint4 u = make_uint4(0, 0, 0, 0);
        if ((cb >> 1) <= (i >> 4)) {
            float f[8], bt[8];
            ld8f(sT + i * AP + 8 * cb, f);
            ld8f(sB + 8 * cb, bt);
#pragma unroll
            for (int x = 0; x < 8; ++x) f[x] *= bt[x];
            u = pack8(f);
        }
        *reinterpret_cast<uint4*>(sm + P_Q + sw128_offset(i, 8 * cb)) = u;
        *reinterpret_cast<uint4*>(img + IMG_T + sw128_offset(i, 8 * cb)) = u;
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();

    // ---- (b3) -W^T = -(K e^G)^T T'^T: M = 128 channels (every TMEM lane holds a row),
    // N = 64 tokens, K = 64 tokens; stored as the MN-major [channel][token] tile the state
    // kernel reads as its B operand
    if (tid == 0) {
        fence_after_sync();
        const uint32_t idesc = make_idesc_bf16(128, 64, true, false, true);   // -(K e^G)^T T'^T
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = make_desc(smem_u32(sm + P_K + ks * 2048), 8192, 1024);   // MN-major
            const uint64_t bd = make_desc(smem_u32(sm + P_Q + ks * 32), 16, 1024);      // K-major
            mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        commit(bar);
    }
    const bool ok = block_wait(bar, parity, err, 3);
    fence_after_sync();
    if (ok) {
        after_mma();                               // P_Q and P_K are free from here on
        // warp w: channel 32 (w % 4) + lane, tokens 32 (w / 4) .. +31
        const int c = 32 * sp + l, half = w >> 2;
        float f[2][16];
        tmem_ld16(tmem + ((uint32_t)(32 * sp) << 16) + 32 * half, f[0]);
        tmem_ld16(tmem + ((uint32_t)(32 * sp) << 16) + 32 * half + 16, f[1]);
        tmem_wait_ld();
        unsigned char* dst = img + IMG_W;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            *reinterpret_cast<uint4*>(dst + sw128_offset(c, 32 * half + 16 * x)) = pack8(f[x]);
            *reinterpret_cast<uint4*>(dst + sw128_offset(c, 32 * half + 16 * x + 8)) = pack8(f[x] + 8);
        }
    }
    return ok;
}

__global__ void __launch_bounds__(PT, 2)
chunk_prep_tc_kernel(const __grid_constant__ PrepMaps maps, const float* __restrict__ beta,
                     SeqInfo si, int64_t H, int64_t h_base, int64_t Hg, int64_t hg,
                     unsigned char* __restrict__ ws, int* __restrict__ err, int* __restrict__ range_flag)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_g, bar_kq, bar;
    __shared__ uint32_t tmem_base;
    __shared__ int32_t s_next[2][3];              // an item, its first token and length
    __shared__ int s_gates_ok;                    // the next item's gates arrived (warps 4-7)

    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int sp = w & 3;                          // TMEM lane quarter of this warp
    unsigned char* sGb = sm + P_G;
    float* egf = reinterpret_cast<float*>(sm + P_VEC);           // [4][VP]  e^{G_f}
    float* eglf = egf + 4 * VP;                                   // [4][VP]  e^{G_last - G_f}
    float* dvec = eglf + 4 * VP;                                  // [6][VP]  e^{G_fp - G_fr}
    float* sB = reinterpret_cast<float*>(sm + P_BETA);
    auto G = [&](int t, int c) -> float& { return *reinterpret_cast<float*>(sGb + g_off(t, c)); };

    // Work items are (chunk, head) pairs, item = chunk * hg + head; this CTA takes
    // blockIdx.x, blockIdx.x + gridDim.x, ...  The next item's gates are fetched as soon
    // as the current one's are last read (after the operand build), its k and q once the
    // W MMA has consumed P_K and P_Q, and its beta at the start of the current item, so the
    // loads overlap the rest of the current item.  One thread finds the next item (items
    // and token rows fit in 32 bits: the launch checks both).
    const int32_t items = (int32_t)(si.chunks_upper * hg), hg32 = (int32_t)hg;
    auto next_item = [&](int32_t from, int32_t& t0_, int32_t& len_) -> int32_t {
        for (int32_t it = from; it < items; it += (int32_t)gridDim.x) {
            int64_t n_, t, ln;
            if (si.locate(it / hg32, n_, t, ln)) {
                t0_ = (int32_t)t;
                len_ = (int32_t)ln;
                return it;
            }
        }
        return -1;
    };
    auto issue_g = [&](int32_t item, int32_t t0_) {               // one thread
        const int32_t y = t0_, x = (int32_t)((h_base + item % hg32) * D);
        tma::expect_tx(&bar_g, 32768);
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) tma::load_2d(sGb + s4 * 8192, &maps.g, x + 32 * s4, y, &bar_g);
    };
    auto issue_kq = [&](int32_t item, int32_t t0_) {              // one thread
        const int32_t y = t0_, x = (int32_t)((h_base + item % hg32) * D);
        tma::expect_tx(&bar_kq, 32768);
        tma::load_2d(sm + P_K, &maps.k, x, y, &bar_kq);
        tma::load_2d(sm + P_K + 8192, &maps.k, x + 64, y, &bar_kq);
        tma::load_2d(sm + P_Q, &maps.q, x, y, &bar_kq);
        tma::load_2d(sm + P_Q + 8192, &maps.q, x + 64, y, &bar_kq);
    };

    auto load_beta = [&](int32_t item, int32_t t0_, int32_t len_) -> float {
        return (item >= 0 && tid < len_) ? beta[((int64_t)t0_ + tid) * H + h_base + item % hg32] : 0.f;
    };

    if (tid == 0) {
        int32_t t_ = 0, l_ = 0;
        const int32_t it = next_item((int32_t)blockIdx.x, t_, l_);
        s_next[0][0] = it;
        s_next[0][1] = t_;
        s_next[0][2] = l_;
        mbar_init(&bar_g, 1);
        mbar_init(&bar_kq, 1);
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (it >= 0) {
            issue_g(it, t_);
            issue_kq(it, t_);
        }
    }
    if (w == 0) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    int32_t cur = s_next[0][0], t0 = s_next[0][1], len = s_next[0][2];
    float bnext = load_beta(cur, t0, len);
    const uint32_t tmem = tmem_base;
    // loads issued and waited for per barrier (at most one in flight each), and
    // completions of the MMA barrier waited for; identical in every thread
    uint32_t g_issued = cur >= 0 ? 1 : 0, kq_issued = g_issued, g_seen = 0, kq_seen = 0, mph = 0;
    uint32_t started = 0;                          // items begun
    bool ok = true, scanned = false;               // scanned: this item's step (a) is done
    float* sA = reinterpret_cast<float*>(sm + P_A);
    float* sT = reinterpret_cast<float*>(sm + P_T);

    // Step (a) for one channel c over all tokens, by one thread (the 128-thread form that
    // warps 4-7 run for the next item while warps 0-3 invert (I + A) of the current one):
    // G in place, the per-channel vectors and e^{G_last} into `img_`.
    auto scan_channel = [&](int c, int len_, unsigned char* img_) {
        unsigned char* slab = sGb + (c >> 5) * 8192 + (c & 3) * 4;
        const int q0 = (c & 31) >> 2;
        float run = 0.f, Gf[4];
#pragma unroll
        for (int pq = 0; pq < 4; ++pq) {
            float v[16];
#pragma unroll
            for (int x = 0; x < 16; ++x)
                v[x] = *reinterpret_cast<const float*>(slab + (16 * pq + x) * 128 + ((q0 ^ (x & 7)) << 4));
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                run += (len_ == C || 16 * pq + x < len_) ? kLog2e * v[x] : 0.f;
                v[x] = run;
            }
            Gf[pq] = v[0];
            if (range_flag && v[0] - v[15] > kRangeLog2) atomicOr(range_flag, 1);
#pragma unroll
            for (int x = 0; x < 16; ++x)
                *reinterpret_cast<float*>(slab + (16 * pq + x) * 128 + ((q0 ^ (x & 7)) << 4)) = v[x];
        }
        const float Gl = run;
#pragma unroll
        for (int pq = 0; pq < 4; ++pq) {
            egf[pq * VP + vidx(c)] = ex2(Gf[pq]);
            eglf[pq * VP + vidx(c)] = ex2(Gl - Gf[pq]);
        }
        int idx = 0;
#pragma unroll
        for (int pq = 1; pq < 4; ++pq)
#pragma unroll
            for (int r = 0; r < pq; ++r) dvec[(idx++) * VP + vidx(c)] = ex2(Gf[pq] - Gf[r]);
        reinterpret_cast<float*>(img_ + IMG_GAM)[c] = ex2(Gl);
    };

    while (cur >= 0 && ok) {
        const int32_t gc = cur / hg32, hl = cur - gc * hg32;
        unsigned char* img = ws + ((int64_t)gc * Hg + hl) * (int64_t)IMG_BYTES;
        // item i + 1 goes to s_next[(i + 1) & 1]: the last reads of that entry came before
        // the previous item's barriers
        int32_t* sn = s_next[(started + 1) & 1];
        if (tid == 0) {
            int32_t t_ = 0, l_ = 0;
            sn[0] = next_item(cur + (int32_t)gridDim.x, t_, l_);
            sn[1] = t_;
            sn[2] = l_;
        }
        if (tid < C) sB[tid] = bnext;
        if (!scanned) {
            fence_before_sync();
            ok = block_wait(&bar_g, g_seen & 1, err, 1);
            fence_after_sync();
            if (!ok) break;
            ++g_seen;
            // ---- (a) cumulative log-decay per channel in log2 units; rows >= len add nothing.
            // Threads c and c + 128 scan tokens 0..31 and 32..63 in registers; the second
            // half then adds the first half's total and derives the per-channel vectors.
            {
                const int c = tid & 127, part = tid >> 7, tb = 32 * part;
                const unsigned char* slab = sGb + (c >> 5) * 8192 + (c & 3) * 4;
                const int q0 = (c & 31) >> 2;
                float v[32];
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    v[x] = *reinterpret_cast<const float*>(slab + (tb + x) * 128 + ((q0 ^ (x & 7)) << 4));
                float run = 0.f;
                if (len == C) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        run += kLog2e * v[x];
                        v[x] = run;
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        run += (tb + x < len) ? kLog2e * v[x] : 0.f;
                        v[x] = run;
                    }
                }
                if (range_flag && (v[0] - v[15] > kRangeLog2 || v[16] - v[31] > kRangeLog2))
                    atomicOr(range_flag, 1);
                if (part == 0) {
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        *reinterpret_cast<float*>(const_cast<unsigned char*>(slab) + x * 128 + ((q0 ^ (x & 7)) << 4)) = v[x];
                }
                __syncthreads();
                if (part == 1) {
                    const float base = G(31, c);
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        v[x] += base;
                        *reinterpret_cast<float*>(const_cast<unsigned char*>(slab) + (32 + x) * 128 + ((q0 ^ (x & 7)) << 4)) = v[x];
                    }
                    const float Gl = v[31];
                    const float Gf[4] = {G(0, c), G(16, c), v[0], v[16]};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        egf[p * VP + vidx(c)] = ex2(Gf[p]);
                        eglf[p * VP + vidx(c)] = ex2(Gl - Gf[p]);
                    }
                    int idx = 0;
#pragma unroll
                    for (int p = 1; p < 4; ++p)
#pragma unroll
                        for (int r = 0; r < p; ++r) dvec[(idx++) * VP + vidx(c)] = ex2(Gf[p] - Gf[r]);
                    reinterpret_cast<float*>(img + IMG_GAM)[c] = ex2(Gl);
                }
            }
        }
        ok = block_wait(&bar_kq, kq_seen & 1, err, 1);   // end of (a); barrier for sB and s_next
        fence_after_sync();
        if (!ok) break;
        ++kq_seen;
        const int32_t nxt = sn[0], t02 = sn[1], len2 = sn[2];
        bnext = load_beta(nxt, t02, len2);
        {
            if (len < C) {
                // a partial chunk: tokens past its end (next sequence or zero fill) read as zero
                for (int e = tid; e < (C - (int)len) * 16; e += PT) {
                    const int t = (int)len + (e >> 4), ch = e & 15;
                    const uint32_t off = (ch >> 3) * 8192 + sw128_offset(t, (8 * ch) & 63);
                    *reinterpret_cast<uint4*>(sm + P_K + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sm + P_Q + off) = make_uint4(0, 0, 0, 0);
                }
                __syncthreads();
            }

            // ---- (b1) A / Aqk strips: operands built per channel half, MMAs accumulate.
            // Thread (ch8, tr, p) handles channels c0 .. c0 + 7 of row 16p + tr (sub-chunk
            // p) and of row 16(3 - p) + tr + 8 (sub-chunk 3 - p): every thread then writes
            // the same number of later-sub-chunk key variants (three).
            const int ch8 = tid & 7, tr = (tid >> 3) & 7, p = tid >> 6;
            for (int hh = 0; hh < 2 && ok; ++hh) {
                const int c0 = 64 * hh + 8 * ch8;
                const int vc = vidx(c0);
                const unsigned char* slab = sGb + (c0 >> 5) * 8192;
                const int q0 = (c0 & 31) >> 2;
                float kin[2][8], qin[2][8], kd[2][8];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int ps = rr == 0 ? p : 3 - p;            // sub-chunk of this row
                    const int t = 16 * ps + tr + 8 * rr;
                    float Gf8[8], G8[8], kk[8], qq[8];
                    {
                        const int tf = 16 * ps;
                        const float4 fa = *reinterpret_cast<const float4*>(slab + tf * 128 + (q0 << 4));
                        const float4 fb = *reinterpret_cast<const float4*>(slab + tf * 128 + ((q0 + 1) << 4));
                        Gf8[0] = fa.x; Gf8[1] = fa.y; Gf8[2] = fa.z; Gf8[3] = fa.w;
                        Gf8[4] = fb.x; Gf8[5] = fb.y; Gf8[6] = fb.z; Gf8[7] = fb.w;
                        const float4 a = *reinterpret_cast<const float4*>(slab + t * 128 + ((q0 ^ (t & 7)) << 4));
                        const float4 b = *reinterpret_cast<const float4*>(slab + t * 128 + (((q0 + 1) ^ (t & 7)) << 4));
                        G8[0] = a.x; G8[1] = a.y; G8[2] = a.z; G8[3] = a.w;
                        G8[4] = b.x; G8[5] = b.y; G8[6] = b.z; G8[7] = b.w;
                    }
                    const uint32_t off = hh * 8192 + sw128_offset(t, 8 * ch8);
                    unpack8(*reinterpret_cast<const uint4*>(sm + P_K + off), kk);
                    unpack8(*reinterpret_cast<const uint4*>(sm + P_Q + off), qq);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float x = G8[j] - Gf8[j];
                        const float e1 = ex2(x);          // <= 1
                        const float r1 = ex2(-x);         // >= 1, at most 15 tokens of decay
                        kin[rr][j] = kk[j] * e1;
                        qin[rr][j] = qq[j] * e1;
                        kd[rr][j] = kk[j] * r1;
                    }
                    // operands of the strip MMAs first
                    const int ts = tr + 8 * rr;          // row within the sub-chunk
                    float tmp[8];
                    *reinterpret_cast<uint4*>(sm + P_KQ + sw128_offset(32 * ps + ts, 8 * ch8)) = pack8(kin[rr]);
                    *reinterpret_cast<uint4*>(sm + P_KQ + sw128_offset(32 * ps + 16 + ts, 8 * ch8)) = pack8(qin[rr]);
                    *reinterpret_cast<uint4*>(sm + P_KV + sw128_offset(kVoff[ps] + t, 8 * ch8)) = pack8(kd[rr]);
#pragma unroll
                    for (int pv = 1; pv < 4; ++pv) {
                        if (pv > ps) {
                            float dv8[8];
                            ld8f(dvec + ((pv * (pv - 1)) / 2 + ps) * VP + vc, dv8);
#pragma unroll
                            for (int j = 0; j < 8; ++j) tmp[j] = kd[rr][j] * dv8[j];
                            *reinterpret_cast<uint4*>(sm + P_KV + sw128_offset(kVoff[pv] + t, 8 * ch8)) = pack8(tmp);
                        }
                    }
                }
                fence_smem_to_async();
                fence_before_sync();
                __syncthreads();
                if (tid == 0) {
                    fence_after_sync();
                    const uint32_t idesc = make_idesc_bf16(64, 32, false, false);
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad = make_desc(smem_u32(sm + P_KV + kVoff[pp] * 128 + ks * 32), 16, 1024);
                            const uint64_t bd = make_desc(smem_u32(sm + P_KQ + 32 * pp * 128 + ks * 32), 16, 1024);
                            mma_bf16(tmem + 32 * pp, ad, bd, idesc, (hh > 0 || ks > 0) ? 1u : 0u);
                        }
                    commit(&bar);
                    if (hh == 1 && nxt >= 0) issue_g(nxt, t02);   // G is not read again
                }
                if (hh == 1 && nxt >= 0) ++g_issued;
                // while the MMAs run: the image's Q e^G and K e^{G_last - G}, and K e^G (in place)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int ps = rr == 0 ? p : 3 - p;
                    const int t = 16 * ps + tr + 8 * rr;
                    const uint32_t off = hh * 8192 + sw128_offset(t, 8 * ch8);
                    float eg[8], egl[8], tmp[8];
                    ld8f(egf + ps * VP + vc, eg);
                    ld8f(eglf + ps * VP + vc, egl);
#pragma unroll
                    for (int j = 0; j < 8; ++j) tmp[j] = qin[rr][j] * eg[j];
                    *reinterpret_cast<uint4*>(img + IMG_QG + hh * 8192 + sw128_offset(t, 8 * ch8)) = pack8(tmp);
#pragma unroll
                    for (int j = 0; j < 8; ++j) tmp[j] = kd[rr][j] * egl[j];
                    *reinterpret_cast<uint4*>(img + IMG_B2 + (1 + hh) * 8192 + sw128_offset(t, 8 * ch8)) = pack8(tmp);
#pragma unroll
                    for (int j = 0; j < 8; ++j) tmp[j] = kin[rr][j] * eg[j];
                    *reinterpret_cast<uint4*>(sm + P_K + off) = pack8(tmp);
                }
                ok = block_wait(&bar, mph & 1, err, 2) && ok;
                fence_after_sync();
                ++mph;
            }
        }

        if (ok) {
            // ---- extract A (fp32, for the inverse) and Aqk^T (bf16 image rows);
            // warps w and w + 4 share a TMEM lane quarter and take two strips each
            const int j = 16 * sp + l;
            float kp[2][16], qp[2][16];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int p = 2 * (w >> 2) + x;
                tmem_ld16(tmem + ((uint32_t)(32 * sp) << 16) + 32 * p, kp[x]);
                tmem_ld16(tmem + ((uint32_t)(32 * sp) << 16) + 32 * p + 16, qp[x]);
            }
            tmem_wait_ld();
            // Rows i of strip p against columns j of block sp (warp-uniform): blocks above
            // the diagonal are zero in Aqk and never read in A (the inverse reads the strictly
            // lower part of A and parks scratch blocks above it), so A needs no mask at all.
            if (l < 16) {
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int p = 2 * (w >> 2) + x, rel = sp - p;
                    float aq[16];
                    if (rel <= 0) {
                        float bt[16];
                        ld8f(sB + 16 * p, bt);
                        ld8f(sB + 16 * p + 8, bt + 8);
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc) sA[(16 * p + cc) * AP + j] = bt[cc] * kp[x][cc];
                    }
                    if (rel < 0) {
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc) aq[cc] = qp[x][cc];
                    } else if (rel == 0) {
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc) aq[cc] = (l <= cc) ? qp[x][cc] : 0.f;
                    } else {
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc) aq[cc] = 0.f;
                    }
                    *reinterpret_cast<uint4*>(img + IMG_B2 + sw128_offset(j, 16 * p)) = pack8(aq);
                    *reinterpret_cast<uint4*>(img + IMG_B2 + sw128_offset(j, 16 * p + 8)) = pack8(aq + 8);
                }
            }
            fence_before_sync();
            __syncthreads();

            // warps 4-7: step (a) of the next item while warps 0-3 invert
            bool side_ok = true;
            ok = prep_tail<true>(sm, img, sA, sT, sB, tmem, &bar, mph & 1, err, [&] {
                if (tid == 0 && nxt >= 0) issue_kq(nxt, t02);
                if (nxt >= 0) ++kq_issued;
            }, [&]() -> bool {
                if (nxt < 0) return true;
                if (tid == 128) s_gates_ok = mbar_wait(&bar_g, g_seen & 1, err, 1) ? 1 : 0;
                bar_sync_named(2, 128);
                if (!s_gates_ok) return false;
                const int32_t gcn = nxt / hg32;
                scan_channel(tid - 128, len2,
                             ws + ((int64_t)gcn * Hg + (nxt - gcn * hg32)) * (int64_t)IMG_BYTES);
                return true;
            }, side_ok);
            ++mph;
            scanned = nxt >= 0 && side_ok;
            if (scanned) ++g_seen;
            ok = ok && side_ok;
        }
        fence_before_sync();
        __syncthreads();                               // TMEM, sA, sT and sB reads of this item are done
        cur = nxt;
        t0 = t02;
        len = len2;
        ++started;
    }
    // after an error: let the loads in flight land before the CTA leaves
    if (tid == 0) {
        if (g_seen < g_issued) mbar_wait(&bar_g, g_seen & 1, nullptr, 0, 200);
        if (kq_seen < kq_issued) mbar_wait(&bar_kq, kq_seen & 1, nullptr, 0, 200);
    }
    fence_before_sync();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// Gated DeltaNet prep: one gate per (token, head)
// ---------------------------------------------------------------------------
// With a scalar decay per token the pairwise factor e^{G_i - G_j} is the same for every
// channel, so ("Kimi Delta Attention: la atencion lineal detras de Kimi K2 y Qwen3",
// comparison of DeltaNet, Gated DeltaNet and KDA; the gate is per head there)
//   A_ij = beta_i e^{G_i - G_j} (k_i . k_j),   Aqk_ij = e^{G_i - G_j} (q_i . k_j)
// come from two plain MMAs on the loaded k and q tiles, with one exponential per (i, j) at
// extraction and every factor <= 1; the image rows are k and q scaled per token.  No
// per-channel operands are built, so the kernel needs 68 KB of shared memory and few
// registers: three CTAs per SM.
constexpr uint32_t GP_K = 0;                        // k (TMA, swizzled), later K e^G   16 KB
constexpr uint32_t GP_Q = 16384;                    // q (TMA), later the T' image      16 KB
constexpr uint32_t GP_A = 32768;                    // fp32 A [64][AP]                  17 KB
constexpr uint32_t GP_T = GP_A + 64 * AP * 4;       // fp32 T [64][AP]                  17 KB
constexpr uint32_t GP_BETA = GP_T + 64 * AP * 4;    // beta [64], cumulative gate [64]
constexpr uint32_t GP_BYTES = GP_BETA + 512;
constexpr uint32_t GP_SMEM = GP_BYTES + 1024;

__global__ void __launch_bounds__(PT, 3)
chunk_prep_gdn_tc_kernel(const __grid_constant__ PrepMaps maps, const float* __restrict__ beta,
                         const float* __restrict__ log_a, SeqInfo si, int64_t H, int64_t h_base,
                         int64_t Hg, unsigned char* __restrict__ ws, int* __restrict__ err)
{
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_in, bar;
    __shared__ uint32_t tmem_base;

    const int64_t gc = blockIdx.x;
    const int hl = blockIdx.y;
    const int64_t h = h_base + hl;
    int64_t n, t0, len;
    if (!si.locate(gc, n, t0, len)) return;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int sp = w & 3;                          // TMEM lane quarter of this warp
    unsigned char* img = ws + (gc * Hg + hl) * (int64_t)IMG_BYTES;
    float* sB = reinterpret_cast<float*>(sm + GP_BETA);
    float* sG = sB + C;                            // [64] cumulative gate, log2 units

    if (tid == 0) {                                // the input loads go out first
        mbar_init(&bar_in, 1);
        mbar_init(&bar, 1);
        fence_mbar_init();
        tma::expect_tx(&bar_in, 32768);
        const int32_t y = (int32_t)t0, x = (int32_t)(h * D);
        tma::load_2d(sm + GP_K, &maps.k, x, y, &bar_in);
        tma::load_2d(sm + GP_K + 8192, &maps.k, x + 64, y, &bar_in);
        tma::load_2d(sm + GP_Q, &maps.q, x, y, &bar_in);
        tma::load_2d(sm + GP_Q + 8192, &maps.q, x + 64, y, &bar_in);
    }
    const float bval = (tid < len) ? beta[(t0 + (tid < C ? tid : 0)) * H + h] : 0.f;
    const float gval = (tid < len) ? log_a[(t0 + (tid < C ? tid : 0)) * H + h] : 0.f;
    if (w == 0) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }
    if (tid < C) {
        sB[tid] = bval;
        sG[tid] = kLog2e * gval;
    }
    fence_before_sync();
    bool ok = block_wait(&bar_in, 0, err, 1);      // also the barrier for sB, sG and TMEM
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    if (ok && len < C) {
        // a partial chunk: tokens past its end (next sequence or zero fill) read as zero
        for (int e = tid; e < (C - (int)len) * 16; e += PT) {
            const int t = (int)len + (e >> 4), ch = e & 15;
            const uint32_t off = (ch >> 3) * 8192 + sw128_offset(t, (8 * ch) & 63);
            *reinterpret_cast<uint4*>(sm + GP_K + off) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(sm + GP_Q + off) = make_uint4(0, 0, 0, 0);
        }
    }
    if (ok && w == 0) {                            // cumulative gate: lanes hold tokens l, l + 32
        float a = sG[l], b = sG[l + 32];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float ua = __shfl_up_sync(0xffffffffu, a, o), ub = __shfl_up_sync(0xffffffffu, b, o);
            if (l >= o) { a += ua; b += ub; }
        }
        b += __shfl_sync(0xffffffffu, a, 31);
        sG[l] = a;
        sG[l + 32] = b;
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    if (ok && tid == 0) {                          // D1[j][i] = k_j . k_i, D2[j][i] = k_j . q_i
        fence_after_sync();
        const uint32_t idesc = make_idesc_bf16(64, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
            const uint64_t kd = make_desc(smem_u32(sm + GP_K + o), 16, 1024);
            const uint64_t qd = make_desc(smem_u32(sm + GP_Q + o), 16, 1024);
            mma_bf16(tmem, kd, kd, idesc, ks > 0 ? 1u : 0u);
            mma_bf16(tmem + 64, kd, qd, idesc, ks > 0 ? 1u : 0u);
        }
        commit(&bar);
    }
    // while the MMAs run: Q e^G and K e^{G_last - G} into the image, e^{G_last}
    if (ok) {
        const float gl = sG[C - 1];
        for (int e = tid; e < C * 16; e += PT) {
            const int t = e >> 4, cg = e & 15;
            const uint32_t off = (cg >> 3) * 8192 + sw128_offset(t, (cg & 7) * 8);
            float kk[8], qq[8], tmp[8];
            unpack8(*reinterpret_cast<const uint4*>(sm + GP_K + off), kk);
            unpack8(*reinterpret_cast<const uint4*>(sm + GP_Q + off), qq);
            const float eqs = ex2(sG[t]), egl = ex2(gl - sG[t]);
#pragma unroll
            for (int x = 0; x < 8; ++x) tmp[x] = qq[x] * eqs;
            *reinterpret_cast<uint4*>(img + IMG_QG + off) = pack8(tmp);
#pragma unroll
            for (int x = 0; x < 8; ++x) tmp[x] = kk[x] * egl;
            *reinterpret_cast<uint4*>(img + IMG_B2 + 8192 + off) = pack8(tmp);
        }
        if (tid < D) reinterpret_cast<float*>(img + IMG_GAM)[tid] = ex2(gl);
    }
    if (ok) ok = block_wait(&bar, 0, err, 2);
    fence_after_sync();
    float* sA = reinterpret_cast<float*>(sm + GP_A);
    float* sT = reinterpret_cast<float*>(sm + GP_T);
    if (ok) {
        // K e^G in place (the MMAs are done with k) for W = -T' (K e^G)
        for (int e = tid; e < C * 16; e += PT) {
            const int t = e >> 4, cg = e & 15;
            const uint32_t off = (cg >> 3) * 8192 + sw128_offset(t, (cg & 7) * 8);
            float kk[8];
            unpack8(*reinterpret_cast<const uint4*>(sm + GP_K + off), kk);
            const float eg = ex2(sG[t]);
#pragma unroll
            for (int x = 0; x < 8; ++x) kk[x] *= eg;
            *reinterpret_cast<uint4*>(sm + GP_K + off) = pack8(kk);
        }
        // extraction: thread (warp w, lane l < 16) takes key row j = 16 sp + l and query /
        // row columns i = 32 (w >> 2) .. +31: A (fp32, for the inverse) and Aqk^T (image)
        const int j = 16 * sp + l, ib = 32 * (w >> 2);
        float d1[2][16], d2[2][16];
        const uint32_t lane = (uint32_t)(32 * sp) << 16;
        tmem_ld16(tmem + lane + ib, d1[0]);
        tmem_ld16(tmem + lane + ib + 16, d1[1]);
        tmem_ld16(tmem + lane + 64 + ib, d2[0]);
        tmem_ld16(tmem + lane + 64 + ib + 16, d2[1]);
        tmem_wait_ld();
        if (l < 16) {
            const float gj = sG[j];
            float aq[32];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {
                    const int i = ib + 16 * x + cc;
                    const float e = (i >= j) ? ex2(sG[i] - gj) : 0.f;    // <= 1
                    sA[i * AP + j] = (j < i) ? sB[i] * e * d1[x][cc] : 0.f;
                    aq[16 * x + cc] = e * d2[x][cc];
                }
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<uint4*>(img + IMG_B2 + sw128_offset(j, ib + 8 * m)) = pack8(aq + 8 * m);
        }
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
        bool side_ok;
        ok = prep_tail<false>(sm, img, sA, sT, sB, tmem, &bar, 1, err, [] {}, [] { return true; }, side_ok);
    } else if (!ok) {
        // the input loads may still be in flight: let them land before leaving
        mbar_wait(&bar_in, 0, nullptr, 0, 200);
    }
    fence_before_sync();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// state kernel
// ---------------------------------------------------------------------------
constexpr uint32_t STAGE_V = IMG_BYTES;                  // v tile, MN-major A (2 blocks of 8 KB)
constexpr uint32_t STAGE_BYTES = IMG_BYTES + 16384;      // 81 KB
constexpr uint32_t S_SBF = 2 * STAGE_BYTES;              // S^T bf16, K-major A: 128 rows x 128 (2 K-blocks)
constexpr uint32_t S_UBF = S_SBF + 32768;                // U^T bf16, K-major A: 128 rows x 64
constexpr uint32_t S_BYTES = S_UBF + 16384;
constexpr uint32_t S_SMEM = S_BYTES + 1024;

constexpr int ST = 288;                                 // state-kernel threads: 8 worker warps + the issuer's

// What one CTA walks (kMode):
//   WALK_SEQ   a whole sequence from h0 (or zero): outputs and the final state;
//   WALK_VALUE one segment from a zero state: its final state is the segment's
//              offset B (no outputs);
//   WALK_MAP   one segment from the identity, with V = 0 (no v loads, no
//              V T'^T product): its final state is the segment's map M;
//   WALK_FINAL one segment from its entry state (SegPlan::starts): outputs, and
//              the final state when it is the sequence's last segment.
enum { WALK_SEQ = 0, WALK_VALUE = 1, WALK_MAP = 2, WALK_FINAL = 3 };

template <bool kHasH0, int kMode>
__global__ void __launch_bounds__(ST, 1)
chunk_state_tc_kernel(const unsigned char* __restrict__ ws, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap omap, float scale,
                      const float* __restrict__ h0, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ hT, SeqInfo si, int64_t H, int64_t h_base, int64_t Hg,
                      const int32_t* __restrict__ slots, int64_t P, int* __restrict__ err,
                      const __grid_constant__ SegPlan sp)
{
    constexpr bool kOut = kMode == WALK_SEQ || kMode == WALK_FINAL;   // outputs written
    constexpr bool kV = kMode != WALK_MAP;                            // v tiles used
    griddep_wait();
    griddep_launch_dependents();
    if (sp.skip && *sp.skip) return;               // the fused kernel takes this call over
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[2], bar1, bar2, barO, uready, sready;
    __shared__ uint32_t tmem_base;

    // blocks run heads-innermost over sequences ranked longest first (or over
    // segments in order)
    const int64_t hg = (H - h_base) < Hg ? (H - h_base) : Hg;
    const int hl = (int)((int64_t)blockIdx.x % hg);
    const int64_t h = h_base + hl;
    int64_t n, g = 0, sg = 0, nsg = 1;
    if constexpr (kMode == WALK_SEQ) {
        n = si.seq_of((int64_t)blockIdx.x / hg);
    } else {
        g = (int64_t)blockIdx.x / hg;
        if (!sp.locate(g, si.N, n, sg, nsg)) return;
    }
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int qt = w & 3, half = w >> 2;                // TMEM lane quarter, column half
    const int j = 32 * qt + l;                          // dv index = TMEM lane
    int64_t bos, eos;
    seq_range(si.cu, n, si.T_seq, si.T_total, bos, eos);
    int64_t nch = si.chunk_count(n, eos - bos);
    int64_t gc0 = si.chunk_start(n);
    if constexpr (kMode != WALK_SEQ) {                  // this segment's chunks
        const int64_t c0 = sg * sp.len;
        nch -= c0;
        nch = nch < 0 ? 0 : (nch > sp.len ? sp.len : nch);
        gc0 += c0;
        bos += c0 * C;
    }
    // state slot of this (sequence, head); -1: none (zero start, nothing stored)
    int64_t sidx = n * H + h;
    if (slots) {
        const int64_t sl = slots[n];
        sidx = (sl >= 0 && sl < P) ? sl * H + h : -1;
        if (sl >= P && tid == 0 && err) atomicOr(err, 1);
    }
    const int64_t sbuf = (g * sp.hstride + (sp.abs_head ? h : (int64_t)hl)) * (int64_t)D * D;
    const float* h0p = nullptr;
    float* hTp = nullptr;
    if constexpr (kMode == WALK_SEQ) {
        h0p = (kHasH0 && sidx >= 0) ? h0 + sidx * (int64_t)D * D : nullptr;
        hTp = (hT && sidx >= 0) ? hT + sidx * (int64_t)D * D : nullptr;
    } else if constexpr (kMode == WALK_VALUE) {
        hTp = sp.offs + sbuf;
    } else if constexpr (kMode == WALK_MAP) {
        hTp = sp.maps + sbuf;
    } else {
        h0p = sp.starts + sbuf;
        hTp = (sg + 1 == nsg && hT && sidx >= 0) ? hT + sidx * (int64_t)D * D : nullptr;
    }
    // entry state element (row c of S, column j)
    auto s_init = [&](int c) -> float {
        if constexpr (kMode == WALK_MAP) return c == j ? 1.f : 0.f;
        else return h0p ? h0p[c * D + j] : 0.f;
    };

    // Roles: warps 0-7 (workers) own the TMEM lanes and all SIMT work; one thread of warp 8
    // (the issuer) issues every MMA and stage copy.  They meet only on mbarriers: the MMA
    // commits (bar1: U^T of a chunk; bar2: its state update; barO: all of its MMAs), the stage
    // copies (full), and two worker arrivals per chunk (uready: U^T staged as an operand;
    // sready: the next state staged), so neither side ever waits for the other's unrelated work.
    const bool worker = w < 8;
    const bool issuer = tid == 8 * 32;
    if (nch == 0) {                                      // nothing to walk: final = entry state
        if (hTp && worker)
            for (int c = 64 * half; c < 64 * half + 64; ++c) hTp[c * D + j] = s_init(c);
        return;
    }
    auto load_stage = [&](int64_t ch, int s) {          // issuer
        unsigned char* st = sm + s * STAGE_BYTES;
        fence_smem_to_async();
        tma::expect_tx(&full[s], kV ? IMG_BYTES + 16384 : IMG_BYTES);
        tma::load_bulk(st, ws + ((gc0 + ch) * Hg + hl) * (int64_t)IMG_BYTES, IMG_BYTES, &full[s]);
        if constexpr (kV) {
            const int32_t y = (int32_t)(bos + ch * C), x = (int32_t)(h * D);
            tma::load_2d(st + STAGE_V, &vmap, x, y, &full[s]);
            tma::load_2d(st + STAGE_V + 8192, &vmap, x + 64, y, &full[s]);
        }
    };

    if (issuer) {
        mbar_init(&full[0], 1); mbar_init(&full[1], 1);
        mbar_init(&bar1, 1); mbar_init(&bar2, 1); mbar_init(&barO, 1);
        mbar_init(&uready, 8); mbar_init(&sready, 8);  // one arrival per worker warp
        fence_mbar_init();
        load_stage(0, 0);
        if (nch > 1) load_stage(1, 1);
    }
    if (w == 0) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t lane = (uint32_t)(32 * qt) << 16;
    const uint32_t tU = tmem, tS = tmem + 256;
    auto tO = [&](int64_t ch) { return tmem + 64 + 64 * (uint32_t)(ch & 1); };
    // a worker warp's arrival: its lanes' shared-memory writes visible to the tensor core and
    // their TMEM accesses ordered before the issuer's next MMA
    auto warp_arrive = [&](uint64_t* b) {
        fence_smem_to_async();
        fence_before_sync();
        __syncwarp();
        if (l == 0) mbar_arrive(b);
    };
    bool ok = true;

    if (w == 8) {
        // the issuer's warp: every lane takes the same branches (the waits' outcomes are shared
        // with __all_sync), lane 0 issues
        auto wait_all = [&](uint64_t* b, uint32_t parity, int bit) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_spin(b, parity, err, bit) ? 1 : 0) != 0;
        };
        // stage copies issued and waited for per stage (for the drain after an error)
        uint32_t issued[2] = {1u, nch > 1 ? 1u : 0u}, seen[2] = {0u, 0u};
        auto wait_stage = [&](int s) -> bool {
            if (!wait_all(&full[s], seen[s] & 1, 4)) return false;
            ++seen[s];
            return true;
        };
        // U^T = V^T T'^T + S^T (-W)^T (commit: bar1), then O^T = S^T (Q e^G)^T (the output takes
        // `scale` when it leaves TMEM)
        auto issue_mma1 = [&](int64_t ch) {
            unsigned char* st = sm + (ch & 1) * STAGE_BYTES;
            fence_after_sync();
            if constexpr (kV) {
                const uint32_t id0 = make_idesc_bf16(128, 64, true, false);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tU, make_desc(smem_u32(st + STAGE_V + ks * 2048), 8192, 1024),
                             make_desc(smem_u32(st + IMG_T + ks * 32), 16, 1024), id0, ks > 0);
            }
            const uint32_t id1 = make_idesc_bf16(128, 64, false, false);
            const uint32_t idW = make_idesc_bf16(128, 64, false, true);    // -W^T: MN-major B
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = make_desc(smem_u32(sm + S_SBF + (ks >> 2) * 16384 + (ks & 3) * 32), 16, 1024);
                mma_bf16(tU, ad, make_desc(smem_u32(st + IMG_W + ks * 2048), 8192, 1024), idW,
                         (kV || ks > 0) ? 1u : 0u);
            }
            commit(&bar1);
            if constexpr (kOut) {
                const uint32_t to = tO(ch);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = make_desc(smem_u32(sm + S_SBF + (ks >> 2) * 16384 + (ks & 3) * 32), 16, 1024);
                    mma_bf16(to, ad, make_desc(smem_u32(st + IMG_QG + (ks >> 2) * 8192 + (ks & 3) * 32), 16, 1024), id1, ks > 0);
                }
            }
        };
        ok = wait_all(&sready, 0, 6) && wait_stage(0);               // entry state staged
        if (ok && l == 0) issue_mma1(0);
        __syncwarp();
        for (int64_t ch = 0; ok && ch < nch; ++ch) {
            const int s = (int)(ch & 1);
            unsigned char* st = sm + s * STAGE_BYTES;
            const uint32_t ph = (uint32_t)(ch & 1);
            if (!(ok = wait_all(&uready, ph, 6))) break;               // U^T staged
            if (l == 0) {
                fence_after_sync();
                // S^T += U^T (K e^{Gl - G}) (N = 128; commit: bar2), then O^T += U^T Aqk^T
                // (N = 64); barO covers all MMAs of this chunk
                const uint32_t idO = make_idesc_bf16(128, 64, false, true);
                const uint32_t idS = make_idesc_bf16(128, 128, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tS, make_desc(smem_u32(sm + S_UBF + ks * 32), 16, 1024),
                             make_desc(smem_u32(st + IMG_B2 + 8192 + ks * 2048), 8192, 1024), idS, 1u);
                commit(&bar2);
                if constexpr (kOut) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tO(ch), make_desc(smem_u32(sm + S_UBF + ks * 32), 16, 1024),
                                 make_desc(smem_u32(st + IMG_B2 + ks * 2048), 8192, 1024), idO, 1u);
                }
                commit(&barO);
            }
            __syncwarp();
            if (ch + 2 < nch) {                                        // the stage takes chunk ch + 2
                if (!(ok = wait_all(&barO, ph, 5))) break;
                if (l == 0) load_stage(ch + 2, s);
                __syncwarp();
                ++issued[s];
            }
            if (ch + 1 < nch) {                                        // next state staged
                if (!(ok = wait_all(&sready, (uint32_t)((ch + 1) & 1), 6) && wait_stage(s ^ 1))) break;
                if (l == 0) issue_mma1(ch + 1);
                __syncwarp();
            }
        }
        if (!ok && l == 0)                                             // drain this CTA's copies
            for (int s = 0; s < 2; ++s)
                while (seen[s] < issued[s]) {
                    mbar_wait(&full[s], seen[s] & 1, nullptr, 0, 200);
                    ++seen[s];
                }
        __syncwarp();
    } else if (worker) {
        // every wait of the workers goes through one AND-barrier, so they leave together
        ok = bar_and_named(1, 256, mbar_wait_spin(&full[0], 0, err, 4));
        // entry state: bf16 copy (operand) and gamma_0-scaled fp32 in TMEM; this thread owns
        // columns 64*half .. +63 of row j of S^T
        if (ok) {
            const float* gam = reinterpret_cast<const float*>(sm + IMG_GAM);
            unsigned char* dst = sm + S_SBF + half * 16384;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                const int c0 = 64 * half + 16 * cb;
                float f[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) f[x] = s_init(c0 + x);
                *reinterpret_cast<uint4*>(dst + sw128_offset(j, 16 * cb)) = pack8(f);
                *reinterpret_cast<uint4*>(dst + sw128_offset(j, 16 * cb + 8)) = pack8(f + 8);
#pragma unroll
                for (int x = 0; x < 16; ++x) f[x] *= gam[c0 + x];
                tmem_st16(tS + lane + c0, f);
            }
            tmem_wait_st();
        }
        warp_arrive(&sready);
        for (int64_t ch = 0; ok && ch < nch; ++ch) {
            const int s = (int)(ch & 1);
            const int64_t t0 = bos + ch * C;
            const int len = (int)((eos - t0) < C ? (eos - t0) : C);
            const uint32_t ph = (uint32_t)(ch & 1);
            const bool last = (ch + 1 == nch);

            // U^T (fp32, TMEM) -> bf16 operand rows; this thread: tokens 32*half .. +31.  The
            // worker barrier also keeps the previous chunk's output copy-out (same buffer) ahead.
            if constexpr (kOut) {
                if (tid == 0) tma::bulk_wait_read();     // the previous chunk's output store
            }
            if (!(ok = bar_and_named(1, 256, mbar_wait_spin(&bar1, ph, err, 5)))) break;
            fence_after_sync();
            {
                float f[2][16];
                tmem_ld16(tU + lane + 32 * half, f[0]);
                tmem_ld16(tU + lane + 32 * half + 16, f[1]);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int c = 32 * half + 16 * x;
                    *reinterpret_cast<uint4*>(sm + S_UBF + sw128_offset(j, c)) = pack8(f[x]);
                    *reinterpret_cast<uint4*>(sm + S_UBF + sw128_offset(j, c + 8)) = pack8(f[x] + 8);
                }
            }
            warp_arrive(&uready);

            // next entry state: bf16 operand copy, then scaled by the next chunk's decay (two
            // rounds of 32 columns: register budget of nine warps per CTA)
            if (!(ok = bar_and_named(1, 256, mbar_wait_spin(&bar2, ph, err, 5) &&
                                               (last || mbar_wait_spin(&full[s ^ 1], (uint32_t)(((ch + 1) >> 1) & 1), err, 4)))))
                break;
            fence_after_sync();
            const float* gam_next =
                last ? nullptr : reinterpret_cast<const float*>(sm + (s ^ 1) * STAGE_BYTES + IMG_GAM);
#pragma unroll
            for (int rd = 0; rd < 2; ++rd) {
                float f[2][16];
#pragma unroll
                for (int x = 0; x < 2; ++x) tmem_ld16(tS + lane + 64 * half + 32 * rd + 16 * x, f[x]);
                tmem_wait_ld();
                if (last) {
                    if (hTp)
#pragma unroll
                        for (int x = 0; x < 2; ++x)
#pragma unroll
                            for (int y = 0; y < 16; ++y) hTp[(64 * half + 32 * rd + 16 * x + y) * D + j] = f[x][y];
                } else {
                    unsigned char* dst = sm + S_SBF + half * 16384;
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        const int cb = 2 * rd + x;
                        *reinterpret_cast<uint4*>(dst + sw128_offset(j, 16 * cb)) = pack8(f[x]);
                        *reinterpret_cast<uint4*>(dst + sw128_offset(j, 16 * cb + 8)) = pack8(f[x] + 8);
                        float g8[16];
                        ld8f(gam_next + 64 * half + 16 * cb, g8);
                        ld8f(gam_next + 64 * half + 16 * cb + 8, g8 + 8);
#pragma unroll
                        for (int y = 0; y < 16; ++y) f[x][y] *= g8[y];
                        tmem_st16(tS + lane + 64 * half + 16 * cb, f[x]);
                    }
                }
            }
            if (!last) {
                tmem_wait_st();
                warp_arrive(&sready);
            }

            // output rows of this chunk, staged through the U^T buffer (its MMAs are complete
            // once barO is) as a [token][dv] bf16 tile: a whole chunk leaves as one tensor store
            // (thread 0; its source is released before the buffer's next use, at the top of the
            // loop), a partial one row by row (the rows past it belong to the next sequence)
            if constexpr (kOut) {
                if (!(ok = bar_and_named(1, 256, mbar_wait_spin(&barO, ph, err, 5)))) break;
                fence_after_sync();
                unsigned char* stg = sm + S_UBF;
                float f[2][16];
                tmem_ld16(tO(ch) + lane + 32 * half, f[0]);
                tmem_ld16(tO(ch) + lane + 32 * half + 16, f[1]);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < 16; ++y) {
                        const int t = 32 * half + 16 * x + y;
                        *reinterpret_cast<__nv_bfloat16*>(stg + t * 256 + j * 2) = __float2bfloat16_rn(scale * f[x][y]);
                    }
                fence_smem_to_async();
                bar_sync_named(1, 256);
                if (len == C) {
                    if (tid == 0) {
                        tma::store_2d(&omap, (int32_t)(h * D), (int32_t)t0, stg);
                        tma::bulk_commit();
                    }
                } else {
                    for (int e = tid; e < len * 16; e += 256) {
                        const int r = e >> 4, c = e & 15;
                        *reinterpret_cast<uint4*>(out + ((t0 + r) * H + h) * D + 8 * c) =
                            *reinterpret_cast<const uint4*>(stg + r * 256 + c * 16);
                    }
                }
            }
            fence_before_sync();
        }
    }
    if (kOut && tid == 0) tma::bulk_wait_all();      // the last output store
    fence_before_sync();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc

int64_t tc_ws_bytes_per_chunk() { return tc::IMG_BYTES; }

int64_t tc_seg_bytes_per_head(const SegPlan& p)
{
    return p.len > 0 ? p.upper * 3 * (int64_t)tc::D * tc::D * (int64_t)sizeof(float) : 0;
}

template <bool kHasH0, int kMode>
static cudaError_t set_state_smem()
{
    return cudaFuncSetAttribute(tc::chunk_state_tc_kernel<kHasH0, kMode>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::S_SMEM);
}

cudaError_t run_prefill_tc(const PrefillArgs& a, unsigned char* ws, int64_t Hg, int* err,
                           cudaStream_t st)
{
    static std::atomic<uint64_t> attrs_done{0};
    cudaError_t e = once_per_device(attrs_done, [] {
        cudaError_t r;
        if ((r = cudaFuncSetAttribute(tc::chunk_prep_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::P_SMEM)))
            return r;
        if ((r = cudaFuncSetAttribute(tc::chunk_prep_gdn_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::GP_SMEM)))
            return r;
        if ((r = set_state_smem<true, tc::WALK_SEQ>())) return r;
        if ((r = set_state_smem<false, tc::WALK_SEQ>())) return r;
        if ((r = set_state_smem<false, tc::WALK_VALUE>())) return r;
        if ((r = set_state_smem<false, tc::WALK_MAP>())) return r;
        return set_state_smem<false, tc::WALK_FINAL>();
    });
    if (e) return e;
    // [tokens][H * d] views of the inputs; rows past the end read as zeros
    const uint64_t rows = (uint64_t)a.si.T_total, cols = (uint64_t)a.H * tc::D;
    tc::PrepMaps maps;
    CUtensorMap vmap;
    if ((e = make_tensor_map_2d(&maps.k, a.k, true, cols, rows, cols * 2, 64, 64, true))) return e;
    if ((e = make_tensor_map_2d(&maps.q, a.q, true, cols, rows, cols * 2, 64, 64, true))) return e;
    if (a.gate_scalar) maps.g = maps.k;        // unused: the gates are loaded per (token, head)
    else if ((e = make_tensor_map_2d(&maps.g, a.log_alpha, false, cols, rows, cols * 4, 32, 64, true)))
        return e;
    if ((e = make_tensor_map_2d(&vmap, a.v, true, cols, rows, cols * 2, 64, 64, true))) return e;
    // out as [tokens][H * D] bf16, boxes of one head's 128 columns x 64 tokens, unswizzled
    // (absent when no walk writes outputs: the segment-map entry point)
    CUtensorMap omap;
    memset(&omap, 0, sizeof(omap));
    if (a.out && (e = make_tensor_map_2d(&omap, a.out, true, cols, rows, cols * 2, tc::D, 64, false))) return e;

    auto launch_prep = [&](int64_t hb, int64_t hg, unsigned char* w, cudaStream_t s) -> cudaError_t {
        if (a.si.chunks_upper <= 0) return cudaSuccess;
        dim3 gp((unsigned)a.si.chunks_upper, (unsigned)hg);
        LaunchScope scope(s, K_PREP_TC);
        if (a.gate_scalar) {
            return launch_pdl(tc::chunk_prep_gdn_tc_kernel, gp, dim3(tc::PT), tc::GP_SMEM, s,
                              maps, a.beta, a.log_alpha, a.si, a.H, hb, Hg, w, err);
        } else {
            // persistent: two CTAs per SM walk the (chunk, head) items
            const int64_t items = a.si.chunks_upper * hg;
            if (items > INT32_MAX) return cudaErrorInvalidValue;   // items are 32-bit in the kernel
            const int64_t slots = 2 * device_sm_count();
            return launch_pdl(tc::chunk_prep_tc_kernel, dim3((unsigned)(items < slots ? items : slots)),
                              dim3(tc::PT), tc::P_SMEM, s, maps, a.beta, a.si, a.H, hb, Hg, hg, w, err,
                              a.range_flag);
        }
    };
    SegPlan none;
    memset(&none, 0, sizeof(none));
    none.skip = a.range_flag;
    auto launch_state = [&](int64_t hb, int64_t hg, unsigned char* w, cudaStream_t s) -> cudaError_t {
        dim3 gs((unsigned)(a.si.N * hg));
        LaunchScope scope(s, K_STATE_TC);
        if (a.h0)
            return launch_pdl(tc::chunk_state_tc_kernel<true, tc::WALK_SEQ>, gs, dim3(tc::ST), tc::S_SMEM, s,
                              w, vmap, omap, a.scale, a.h0, (__nv_bfloat16*)a.out, a.hT, a.si, a.H, hb, Hg,
                              a.slots, a.P, err, none);
        return launch_pdl(tc::chunk_state_tc_kernel<false, tc::WALK_SEQ>, gs, dim3(tc::ST), tc::S_SMEM, s,
                          w, vmap, omap, a.scale, (const float*)nullptr, (__nv_bfloat16*)a.out, a.hT, a.si,
                          a.H, hb, Hg, a.slots, a.P, err, none);
    };
    // one walk over every segment of the plan (grid: segment bound x heads)
    auto launch_walk = [&](int mode, const SegPlan& sp, int64_t hb, int64_t hg, unsigned char* w,
                           cudaStream_t s) -> cudaError_t {
        if (sp.upper <= 0) return cudaSuccess;
        dim3 gs((unsigned)(sp.upper * hg));
        LaunchScope scope(s, mode == tc::WALK_FINAL ? K_STATE_TC : K_STATE_SEG_TC);
        __nv_bfloat16* o = (__nv_bfloat16*)a.out;
        const float* no_h0 = nullptr;
        float* no_hT = nullptr;
        if (mode == tc::WALK_VALUE)
            return launch_pdl(tc::chunk_state_tc_kernel<false, tc::WALK_VALUE>, gs, dim3(tc::ST), tc::S_SMEM, s,
                              w, vmap, omap, a.scale, no_h0, o, no_hT, a.si, a.H, hb, Hg, a.slots, a.P, err, sp);
        if (mode == tc::WALK_MAP)
            return launch_pdl(tc::chunk_state_tc_kernel<false, tc::WALK_MAP>, gs, dim3(tc::ST), tc::S_SMEM, s,
                              w, vmap, omap, a.scale, no_h0, o, no_hT, a.si, a.H, hb, Hg, a.slots, a.P, err, sp);
        return launch_pdl(tc::chunk_state_tc_kernel<false, tc::WALK_FINAL>, gs, dim3(tc::ST), tc::S_SMEM, s,
                          w, vmap, omap, a.scale, no_h0, o, a.hT, a.si, a.H, hb, Hg, a.slots, a.P, err, sp);
    };

    // segment buffers sit after the operand images of one head group
    SegPlan sp = a.seg;
    sp.skip = a.tc_what == 0 ? a.range_flag : nullptr;
    if (a.tc_what == 0 && sp.len > 0) {
        const int64_t mat = (int64_t)tc::D * tc::D;
        float* segbuf = reinterpret_cast<float*>(
            ws + Hg * (a.si.chunks_upper > 0 ? a.si.chunks_upper : 1) * (int64_t)tc::IMG_BYTES);
        sp.maps = segbuf;
        sp.offs = segbuf + sp.upper * Hg * mat;
        sp.starts = segbuf + 2 * sp.upper * Hg * mat;
        sp.hstride = Hg;
        sp.abs_head = false;
    }

    for (int64_t hb = 0; hb < a.H; hb += Hg) {
        const int64_t hg = (a.H - hb) < Hg ? (a.H - hb) : Hg;
        if ((e = launch_prep(hb, hg, ws, st))) return e;
        if (a.tc_what == 2) continue;          // operand images only
        if (a.tc_what == 1) {                  // each sequence's (M, B) into the caller's buffers
            if ((e = launch_walk(tc::WALK_VALUE, sp, hb, hg, ws, st))) return e;
            if ((e = launch_walk(tc::WALK_MAP, sp, hb, hg, ws, st))) return e;
        } else if (sp.len > 0) {               // segment-parallel walk
            if ((e = launch_walk(tc::WALK_VALUE, sp, hb, hg, ws, st))) return e;
            if ((e = launch_walk(tc::WALK_MAP, sp, hb, hg, ws, st))) return e;
            PrefixArgs pa;
            pa.maps = sp.maps; pa.offs = sp.offs; pa.h0 = a.h0; pa.starts = sp.starts;
            pa.out = nullptr; pa.seg_off = sp.seg_off; pa.nseg = sp.nseg; pa.N = a.si.N;
            pa.H = a.H; pa.h_base = hb; pa.hg = hg; pa.hstride = Hg; pa.abs_head = false;
            pa.slots = a.slots; pa.P = a.P; pa.dk = tc::D; pa.dv = tc::D; pa.err = err;
            if ((e = launch_affine_prefix(pa, st))) return e;
            if ((e = launch_walk(tc::WALK_FINAL, sp, hb, hg, ws, st))) return e;
        } else {
            if ((e = launch_state(hb, hg, ws, st))) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace kda
