// Fused chunkwise KDA prefill on the sm_100a tensor cores (bf16 I/O, dk = dv = 128).
//
// The chunk equations are those of the two-kernel path (derived by unrolling the
// per-token step of "Kimi Delta Attention: la atencion lineal detras de Kimi K2 y
// Qwen3", section "Como funciona Kimi Delta Attention paso a paso"; the chunkwise
// form is the one "Kimi Linear acaba de superar a la atencion completa en sus
// propios terminos" says the method trains with), with T' = (I + A)^{-1} diag(beta):
//
//   A_ij   = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}   (i > j)
//   Aqk_ij = sum_c q_ic k_jc e^{G_ic - G_jc}          (i >= j)
//   W = T' (K e^G),  U = T' V - W S,  O = scale ((Q e^G) S + Aqk U),
//   S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T U
//
// One CTA per SM walks (sequence, head) chains, heads innermost, and computes
// every chunk's operands on chip: nothing but the inputs, the outputs and the
// final states crosses HBM.  Roles (448 threads):
//   warps 0-7   prep: thread (channel c, token half) -- cumulative decay in
//               registers, the exponential factors, the operand tiles [c][t]
//               (token-contiguous, 128B-swizzled), the A / Aqk read-out, the
//               blocked inverse of (I + A) (its block products split over all
//               eight warps; it also writes T') and the -W^T read-out; thread 0
//               issues the A / Aqk and -W^T MMAs itself;
//   warps 8-11  walk: thread = value column j (a TMEM lane of S^T) -- the
//               state's decay scaling, the U^T / S^T bf16 copies (kept in
//               tensor memory as MMA operands), the output tile;
//   warp 12     one thread issues the prep's TMA loads and the k / q transposes,
//               and (packed sequences) takes each CTA's next chain by ticket;
//   warp 13     one thread issues the walk's MMAs and v loads.
// Per chunk, k and q land by TMA as [t][c] tiles and are transposed into tensor
// memory by an MMA with the identity (exact), so each prep thread owns one
// channel's tokens; the next chunk's transposes are released only once the A / Aqk
// MMA of this one has completed, so that they never queue ahead of it on the tensor
// pipe.  The decay factors e^{G_i - G_j} are split as e^{G_i} e^{-G_j}
// when every |G| of the chunk stays within 2^100: the row operands of A and Aqk
// are then the image tiles K e^G and Q e^G themselves, the column operand is
// K e^{-G}, and A and Aqk are one MMA.  When instead every |G - s0| does (s0 = the
// channel's decay over the first 32 tokens), the same MMA takes e^{G_i - s0} and
// e^{s0 - G_j}, and the image rows are written again at the chunk start once it has
// completed.  Past that the lower triangle is taken level by level (blocks of 64,
// 32, ..., 2 rows; each pair i > j at the level where i and j fall in different
// halves, both factors referenced to the first row of the upper half and so <= 1),
// plus one product for the diagonal: exact at any decay rate.  The state walk of chunk c (U^T = V^T T'^T + S^T (-W^T),
// O^T = S^T (Q e^G)^T + U^T Aqk^T, S^T += U^T (K e^{Gl - G}), as three MMA groups:
// [O^T | U^T] = S^T [(Q e^G)^T | -W^T] with N = 128, U^T += V^T T'^T, and
// [S^T | O^T] += U^T [K e^{Gl - G} ; Aqk] with N = 192) overlaps the prep
// of chunk c + 1; the state's decay by the next chunk's e^{G_last} is applied
// as the walk copies the state for that chunk.  Operands whose producer and
// consumer overlap are double-buffered, the rest are handed over on mbarriers.  Every wait is
// bounded; a wait that gives up sets a bit in the error word and makes every
// role leave its loop, after which the CTA drains its copies and MMAs and
// frees its tensor memory.
#include <cstring>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc_util.cuh"
#include "kda_tma.cuh"
#include "kda_umma.cuh"

namespace kda {

using namespace umma;
using namespace tcu;

namespace fz {

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 448;
constexpr int AP = 68;                      // row pitch (floats) of the fp32 A and T
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRange = 100.f;             // one-product forms: every |G| or |G - s0| (log2) within
constexpr long long kWaitCycles = 4000000000LL;

constexpr int W_WALK = 8;                   // walk warps 8-11
constexpr int W_PI = 12;                    // prep issuer
constexpr int W_WI = 13;                    // walk issuer

constexpr int NB_PAIR = 1;                  // 1..4: prep warps w and w + 4
constexpr int NB_PREP = 5;                  // prep warps 0-7
constexpr int NB_WALK = 7;                  // walk warps

// Shared memory (bytes from a 1024-aligned base).  [c][t] tiles: 128 channel rows of
// 64 tokens (128 B), 128B-swizzled -- K-major when the tokens are the reduction index,
// MN-major when they are the M/N index.
constexpr uint32_t F_ID = 0;                // identity 16 x 16 bf16 (16 rows of 128 B)     2 KB
constexpr uint32_t F_G = 2048;              // log_alpha [t][c] fp32 (TMA, unswizzled)     32 KB
constexpr uint32_t F_KQ = 34816;            // k | q [t][c] (TMA)                          32 KB
constexpr uint32_t F_KD = 67584;            // (K e^{-G})^T, then T fp32 [64][AP]          17 KB
constexpr uint32_t F_KG = 84992;            // (K e^G)^T                                   16 KB
constexpr uint32_t F_QG = 101376;           // (Q e^G)^T x 2; after use the output tile    32 KB
constexpr uint32_t F_KLAQ = 134144;         // per slot: (K e^{Gl - G})^T, then Aqk [i][j]  48 KB
constexpr uint32_t F_TP = 183296;           // T' [i][j]                                    8 KB
constexpr uint32_t F_W = 191488;            // A fp32 [64][AP] for the inverse, then -W^T  17 KB
constexpr uint32_t F_V = 208896;            // v [t][dv] (TMA)                             16 KB
constexpr uint32_t F_GAM = 225280;          // e^{G_last} x 2
constexpr uint32_t F_BETA = 226304;         // beta of the chunk
constexpr uint32_t F_XCH = 226560;          // half sums of the decay [3][128]
constexpr uint32_t F_BYTES = F_XCH + 3 * 128 * 4;
constexpr uint32_t F_SMEM = F_BYTES + 1024;
static_assert(F_KD + 64 * AP * 4 <= F_KG, "T scratch overlaps (K e^G)^T");
static_assert(F_W + 64 * AP * 4 <= F_V, "A scratch overlaps v");

// Tensor memory columns (512 allocated)
constexpr uint32_t TM_KT = 0;               // k^T fp32 (prep)
constexpr uint32_t TM_QT = 64;              // q^T fp32
constexpr uint32_t TM_S = 128;              // S^T fp32 (state)
constexpr uint32_t TM_O = 256;              // O^T fp32 (right after S^T: one N = 192 update)
constexpr uint32_t TM_U = 320;              // U^T fp32 (right after O^T: one N = 128 product);
                                            // its first 32 columns then hold U^T bf16
constexpr uint32_t TM_SB = 384;             // S^T bf16 (operand)
constexpr uint32_t TM_D = 448;              // [K e^G; Q e^G] (K e^{-G})^T, then -W^T

struct Bars {
    uint64_t g, gc, kq, tr, ktf, gam, a, w, img;   // prep pipeline
    uint64_t v, u, s, o, ur, sr, orr;          // walk pipeline
    uint64_t m1, fr[2];                     // walk -> prep: MMA1 done, image slot free
    uint64_t fin_p, fin_w, fin_q;           // final drains: prep issuer, walk issuer, prep leader
};

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded poll of one phase; gives up when another role has given up (abort) or after
// about 2 s, then sets bit `bit` in *err and the abort flag.
__device__ __forceinline__ bool fwait(uint64_t* bar, uint32_t parity, int* err, int bit,
                                      volatile int* abort)
{
    const long long t0 = clock64();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (*abort) return false;
            if (clock64() - t0 > kWaitCycles) {
                if (err) atomicOr(err, 1 << bit);
                *abort = 1;
                return false;
            }
        }
    }
}

// A group's wait: `leader` polls, the group's barrier shares the outcome.
__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, bool leader, int barid,
                                      int count, int* err, int bit, volatile int* abort)
{
    bool ok = true;
    if (leader) ok = fwait(bar, parity, err, bit, abort);
    return bar_and_named(barid, count, ok);
}

// Where a CTA's chains come from.  Static: blockIdx.x, + gridDim.x, ... of the
// (sequence rank, head) list.  Dynamic (packed sequences of mixed lengths): chain
// blockIdx.x first, then whatever chain a ticket from the global counter names
// (gridDim.x + ticket), so the CTAs that finish early take the remaining chains and,
// with the sequences ranked longest first, the long chains start first.  In dynamic
// mode one thread (the prep issuer, the role furthest ahead) takes the tickets and
// publishes each chain it starts, in order, in a ring in shared memory; every other
// role reads the ring at the same position.
constexpr int kRing = 16;
struct Sched {
    int* ticket;                                // global counter (zeroed) or null: static
    volatile int* ring_val;                     // [kRing] chain index, -1: no more chains
    volatile int* ring_seq;                     // [kRing] position the entry was written for
};

// The chunks of one CTA, chain by chain, heads innermost; sequences ranked longest
// first when an order is known.  Chains without tokens are skipped (their final
// states are written separately).  Token rows and chain indices fit 32 bits (the
// launch checks both).
struct Items {
    int32_t r, h, n, bos, eos, nch, c;
    int64_t sidx;                               // state index, -1: none
    uint32_t q;                                 // chains started before this one
    bool ok;

    // Chain r's fields; false when r is past the end or the chain has no tokens.
    __device__ __forceinline__ bool set(int32_t r_, const SeqInfo& si, int32_t H, const int32_t* slots,
                                        int64_t P)
    {
        r = r_;
        if (r < 0 || r >= (int32_t)si.N * H) return false;
        const int32_t sr = r / H;
        h = r - sr * H;
        n = (int32_t)si.seq_of(sr);
        int64_t b, e;
        seq_range(si.cu, n, si.T_seq, si.T_total, b, e);
        bos = (int32_t)b;
        eos = (int32_t)e;
        nch = (eos - bos + C - 1) / C;
        c = 0;
        sidx = (int64_t)n * H + h;
        if (slots) {
            const int64_t sl = slots[n];
            sidx = (sl >= 0 && sl < P) ? sl * H + h : -1;
        }
        return nch > 0;
    }
    // The first chain with tokens from candidate `r` on, in the source's order, or -1.
    __device__ __forceinline__ int32_t resolve(int32_t r_, const Sched& sc, const SeqInfo& si, int32_t H,
                                               const int32_t* slots, int64_t P)
    {
        const int32_t rend = (int32_t)si.N * H;
        while (r_ < rend) {
            if (set(r_, si, H, slots, P)) return r_;
            r_ = sc.ticket ? (int32_t)gridDim.x + atomicAdd(sc.ticket, 1) : r_ + (int32_t)gridDim.x;
        }
        return -1;
    }
    // Publisher: ring entry q (dynamic mode).
    __device__ __forceinline__ void publish(const Sched& sc, uint32_t qq, int32_t val)
    {
        sc.ring_val[qq % kRing] = val;
        __threadfence_block();
        sc.ring_seq[qq % kRing] = (int)qq;
    }
    // Reader: ring entry q, polled with the same bounds as the mbarrier waits.
    __device__ __forceinline__ int32_t read(const Sched& sc, uint32_t qq, int* err, volatile int* abort)
    {
        const long long t0 = clock64();
        for (uint32_t i = 1;; ++i) {
            if (sc.ring_seq[qq % kRing] == (int)qq) {
                __threadfence_block();
                return sc.ring_val[qq % kRing];
            }
            if ((i & 31u) == 0) {
                if (*abort) return -1;
                if (clock64() - t0 > kWaitCycles) {
                    if (err) atomicOr(err, 1 << 6);
                    *abort = 1;
                    return -1;
                }
            }
        }
    }
    // Chain number q from the source: the publisher resolves and publishes it, the
    // other roles read it (dynamic) or resolve it themselves (static).
    __device__ __forceinline__ void take(int32_t cand, bool publisher, const Sched& sc, const SeqInfo& si,
                                         int32_t H, const int32_t* slots, int64_t P, int* err,
                                         volatile int* abort)
    {
        int32_t got;
        if (!sc.ticket || publisher) {
            got = resolve(cand, sc, si, H, slots, P);
            if (sc.ticket) publish(sc, q, got);
        } else {
            got = read(sc, q, err, abort);
        }
        ok = got >= 0 && set(got, si, H, slots, P);
    }
    __device__ __forceinline__ void init(bool publisher, const Sched& sc, const SeqInfo& si, int32_t H,
                                         const int32_t* slots, int64_t P, int* err, volatile int* abort)
    {
        q = 0;
        take((int32_t)blockIdx.x, publisher, sc, si, H, slots, P, err, abort);
    }
    __device__ __forceinline__ void next(bool publisher, const Sched& sc, const SeqInfo& si, int32_t H,
                                         const int32_t* slots, int64_t P, int* err, volatile int* abort)
    {
        if (++c >= nch) {
            ++q;
            if (sc.ticket && !publisher) {
                take(-1, false, sc, si, H, slots, P, err, abort);
                return;
            }
            const int32_t cand = sc.ticket ? (int32_t)gridDim.x + atomicAdd(sc.ticket, 1)
                                           : r + (int32_t)gridDim.x;
            take(cand, publisher, sc, si, H, slots, P, err, abort);
        }
    }
    __device__ __forceinline__ int32_t t0() const { return bos + c * C; }
    __device__ __forceinline__ int len() const
    {
        const int32_t l = eos - t0();
        return l < C ? l : C;
    }
    __device__ __forceinline__ bool first() const { return c == 0; }
    __device__ __forceinline__ bool last() const { return c + 1 == nch; }
};

// Byte offset of token t of channel row c in a [c][t] tile.
__device__ __forceinline__ uint32_t ct_off(int c, int t)
{
    return (uint32_t)c * 128u + ((uint32_t)(((t >> 3) ^ c) & 7) << 4);
}

// Byte offset of element (i, j) in the 128B-swizzled [i][j] bf16 T' tile (64 x 64).
__device__ __forceinline__ uint32_t tp_off(int i, int j)
{
    return sw128_offset(i, j & ~7) + 2u * (uint32_t)(j & 7);
}

// Columns 8 nh .. 8 nh + 7 of the 16 x 16 product X Y (fp32 blocks of pitch AP, tf32
// operands, fp32 accumulation): one m16n8k8 accumulator per k-step pair.
__device__ __forceinline__ void mma16x8x16_tf32(float (&acc)[4], const float* X, const float* Y, int nh,
                                                int lane)
{
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = tf32(X[g * AP + 8 * ks + q]);
        const uint32_t a1 = tf32(X[(g + 8) * AP + 8 * ks + q]);
        const uint32_t a2 = tf32(X[g * AP + 8 * ks + q + 4]);
        const uint32_t a3 = tf32(X[(g + 8) * AP + 8 * ks + q + 4]);
        const uint32_t b0 = tf32(Y[(8 * ks + q) * AP + 8 * nh + g]);
        const uint32_t b1 = tf32(Y[(8 * ks + q + 4) * AP + 8 * nh + g]);
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// Stores columns 8 nh .. + 7 of a 16 x 16 block (accumulator layout, times `s`) to Z.
__device__ __forceinline__ void store16x8(float* Z, const float (&acc)[4], float s, int nh, int lane)
{
    const int g = lane >> 2, q = lane & 3;
    Z[g * AP + 8 * nh + 2 * q] = s * acc[0];
    Z[g * AP + 8 * nh + 2 * q + 1] = s * acc[1];
    Z[(g + 8) * AP + 8 * nh + 2 * q] = s * acc[2];
    Z[(g + 8) * AP + 8 * nh + 2 * q + 1] = s * acc[3];
}

// Columns 8 nh .. + 7 of block (p, r) of T (times `s`): to the fp32 T (pitch AP) and,
// scaled by beta_j, to the bf16 T' tile.
__device__ __forceinline__ void store_t_half(float* sT, unsigned char* tp, const float* sB, int p, int r,
                                             int nh, const float (&acc)[4], float s, int lane)
{
    store16x8(sT + (16 * p) * AP + 16 * r, acc, s, nh, lane);
    const int g = lane >> 2, q = lane & 3;
    const int j = 16 * r + 8 * nh + 2 * q;
    const float b0 = sB[j], b1 = sB[j + 1];
    *reinterpret_cast<uint32_t*>(tp + tp_off(16 * p + g, j)) = pack_bf16(s * acc[0] * b0, s * acc[1] * b1);
    *reinterpret_cast<uint32_t*>(tp + tp_off(16 * p + g + 8, j)) = pack_bf16(s * acc[2] * b0, s * acc[3] * b1);
}

// T = (I + A)^{-1} for the strictly lower A (fp32, pitch AP), by all eight prep warps:
// 16 x 16 diagonal blocks from their 8 x 8 halves (threads 0-63), then
// the blocks below by tf32 block products in three levels, each 16 x 16 product split
// into its two 8-column halves on two warps (scratch blocks parked above the diagonal
// of A).  Every block of T on or below the diagonal is written twice: in fp32 to sT (the
// later levels read it) and as T' = T diag(beta) to the bf16 tile `tp` (the diagonal
// blocks by warps 4-7 during the first level), whose blocks above the diagonal stay zero
// (written once, when the kernel starts).
__device__ __forceinline__ void invert_unit_lower(float* sA, float* sT, unsigned char* tp, const float* sB,
                                                  int tid)
{
    const int w = tid >> 5, l = tid & 31;
    if (tid < C) {
        // each 16 x 16 diagonal block (16 threads of one warp): its two 8 x 8 diagonal
        // blocks by forward substitution (one column per thread), then the 8 x 8 block
        // below them, L = -T_hi A_lo,hi-lo T_lo, by two fp32 products; Y = A T_lo is parked
        // in the block's unused upper-right 8 x 8 quarter
        const int b = tid >> 4, cc = tid & 15, o = 16 * b + 8 * (cc >> 3), c8 = cc & 7;
        float tcol[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) acc += sA[(o + r) * AP + o + m] * tcol[m];
            tcol[r] = (r == c8) ? 1.f : ((r < c8) ? 0.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) sT[(o + r) * AP + o + c8] = tcol[r];
        __syncwarp();
        const int ob = 16 * b, i = cc >> 1, j0 = 4 * (cc & 1);   // this thread: row i, columns j0..j0+3
        float y[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {               // Y = A[8+i][0..7] T_lo[.][j]
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) acc += sA[(ob + 8 + i) * AP + ob + m] * sT[(ob + m) * AP + ob + j0 + x];
            y[x] = acc;
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) sA[(ob + i) * AP + ob + 8 + j0 + x] = y[x];
        __syncwarp();
#pragma unroll
        for (int x = 0; x < 4; ++x) {               // L = -T_hi Y  (T_hi unit lower)
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) acc += sT[(ob + 8 + i) * AP + ob + 8 + m] * sA[(ob + m) * AP + ob + 8 + j0 + x];
            sT[(ob + 8 + i) * AP + ob + j0 + x] = -acc;
        }
        // T's upper-right 8 x 8 quarter of the block is zero
#pragma unroll
        for (int x = 0; x < 4; ++x) sT[(ob + i) * AP + ob + 8 + j0 + x] = 0.f;
    }
    bar_sync_named(NB_PREP, 256);
    auto Ab = [&](int r, int c) { return sA + (16 * r) * AP + 16 * c; };
    auto Tb = [&](int r, int c) { return sT + (16 * r) * AP + 16 * c; };
    if (w < 4) {                                  // T_10 = -T_11 A_10 T_00, T_32 = -T_33 A_32 T_22
        const int p = 2 * (w & 1) + 1, r = p - 1, nh = w >> 1;
        float acc[4] = {};
        mma16x8x16_tf32(acc, Ab(p, r), Tb(r, r), nh, l);
        store16x8(Ab(r, p), acc, 1.f, nh, l);
        __syncwarp();
        float acc2[4] = {};
        mma16x8x16_tf32(acc2, Tb(p, p), Ab(r, p), nh, l);
        store_t_half(sT, tp, sB, p, r, nh, acc2, -1.f, l);
    } else {                                      // meanwhile, T' of the diagonal blocks
        const int t = tid - 128, o = 16 * (t >> 5), i = o + ((t >> 1) & 15), hlf = t & 1;
        float f[8], bt[8];
        ld8f(sT + i * AP + o + 8 * hlf, f);
        ld8f(sB + o + 8 * hlf, bt);
#pragma unroll
        for (int x = 0; x < 8; ++x) f[x] *= bt[x];
        *reinterpret_cast<uint4*>(tp + sw128_offset(i, o + 8 * hlf)) = pack8(f);
    }
    bar_sync_named(NB_PREP, 256);
    const int p = 2 + ((w >> 1) & 1), r = w & 1, nh = w >> 2;
    {                                             // X_pr = sum_{m = r..1} A_pm T_mr
        float acc[4] = {};
        for (int m = r; m < 2; ++m) mma16x8x16_tf32(acc, Ab(p, m), Tb(m, r), nh, l);
        store16x8(Ab(r, p), acc, 1.f, nh, l);
    }
    bar_sync_named(NB_PREP, 256);
    {                                             // T_pr = -sum_{m = 2..p} T_pm X_mr
        float acc[4] = {};
        for (int m = 2; m <= p; ++m) mma16x8x16_tf32(acc, Tb(p, m), Ab(r, m), nh, l);
        store_t_half(sT, tp, sB, p, r, nh, acc, -1.f, l);
    }
}

// Level-pass selection of the exact fallback: pair (i, j) is taken at pass `pass`
// (0..5: blocks of 2s rows, s = 32 >> pass) when i is in the upper half of its block
// and j in the lower half of the same block; pass 6 takes the diagonal (Aqk only).
__device__ __forceinline__ bool pass_pair(int pass, int i, int j)
{
    if (pass == 6) return i == j;
    const int s = 32 >> pass;
    const int f = (i & ~(2 * s - 1)) + s;       // first row of i's upper half
    return (i & (2 * s - 1)) >= s && j >= f - s && j < f;
}

__global__ void __launch_bounds__(NT, 1)
chunk_fused_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap,
                      const __grid_constant__ CUtensorMap gmap,
                      const float* __restrict__ log_alpha, const float* __restrict__ beta,
                      const float* __restrict__ h0, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ hT, float scale, SeqInfo si, int64_t H,
                      const int32_t* __restrict__ slots, int64_t P, int* __restrict__ err,
                      int* __restrict__ ticket, const int* __restrict__ run_if)
{
    if (run_if && *run_if == 0) return;           // the two-kernel form computed this call
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Bars bars;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort_raw;
    __shared__ int s_ring_val[kRing], s_ring_seq[kRing];
    volatile int* abort = &s_abort_raw;

    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int32_t H32 = (int32_t)H;
    const Sched sc{ticket, s_ring_val, s_ring_seq};
    const bool publisher = tid == W_PI * 32;
    if (tid < kRing) s_ring_seq[tid] = -1;

    if (tid == W_PI * 32) {
        mbar_init(&bars.g, 1); mbar_init(&bars.gc, 8);
        mbar_init(&bars.kq, 1); mbar_init(&bars.tr, 1); mbar_init(&bars.ktf, 8); mbar_init(&bars.gam, 8);
        mbar_init(&bars.a, 1); mbar_init(&bars.w, 1); mbar_init(&bars.img, 8);
        mbar_init(&bars.v, 1); mbar_init(&bars.u, 1); mbar_init(&bars.s, 1); mbar_init(&bars.o, 1);
        mbar_init(&bars.ur, 4); mbar_init(&bars.sr, 4); mbar_init(&bars.orr, 4);
        mbar_init(&bars.m1, 1); mbar_init(&bars.fr[0], 1); mbar_init(&bars.fr[1], 1);
        mbar_init(&bars.fin_p, 1); mbar_init(&bars.fin_w, 1); mbar_init(&bars.fin_q, 1);
        fence_mbar_init();
        s_abort_raw = 0;
    }
    if (w < 8) {                                  // the identity operand of the transposes
        for (int e = tid; e < 512; e += 256)      // T' tile: blocks above the diagonal stay 0
            reinterpret_cast<uint4*>(sm + F_TP)[e] = make_uint4(0, 0, 0, 0);
        if (tid < 128) {
            const int r = tid >> 3, cb = tid & 7;
            float f[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) f[x] = (8 * cb + x == r) ? 1.f : 0.f;
            *reinterpret_cast<uint4*>(sm + F_ID + sw128_offset(r, 8 * cb)) = pack8(f);
        }
        fence_smem_to_async();
    }
    if (w == W_PI) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    // every role's first chain (the publisher's entry is written before anyone reads it)
    Items it0;
    if (publisher) it0.init(true, sc, si, H32, slots, P, err, abort);
    __syncthreads();
    if (!publisher) it0.init(false, sc, si, H32, slots, P, err, abort);

    if (w < 8) {
        // ------------------------------------------------------------------ prep
        const int q4 = w & 3, ph = w >> 2;
        const int pc = 32 * q4 + l;               // channel (TMEM lane of k^T, q^T, -W^T)
        const uint32_t lane = (uint32_t)(32 * q4) << 16;
        const bool leader = tid == 0;
        float* sB = reinterpret_cast<float*>(sm + F_BETA);
        float* xch = reinterpret_cast<float*>(sm + F_XCH);
        float* sA = reinterpret_cast<float*>(sm + F_W);
        float* sT = reinterpret_cast<float*>(sm + F_KD);

        const float* sg = reinterpret_cast<const float*>(sm + F_G);
        // operand descriptors (the leader issues the prep's MMAs): A and Aqk take the rows
        // [K e^G; Q e^G] (the Q e^G block of slot s one LBO step after K e^G) against the
        // columns K e^{-G}; -W^T = -(K e^G)^T T'^T
        const uint64_t dRow0 = make_desc(smem_u32(sm + F_KG), F_QG - F_KG, 1024);
        const uint64_t dRow1 = make_desc(smem_u32(sm + F_KG), F_QG + 16384 - F_KG, 1024);
        const uint64_t dCol = make_desc(smem_u32(sm + F_KD), 16384, 1024);
        const uint64_t dKgT = make_desc(smem_u32(sm + F_KG), 16, 1024);
        const uint64_t dTp = make_desc(smem_u32(sm + F_TP), 16, 1024);
        constexpr uint32_t idA = make_idesc_bf16(128, 64, true, true);
        constexpr uint32_t idW = make_idesc_bf16(128, 64, false, false, true);
        Items it = it0;
        uint32_t n_a = 0;                         // completions of bars.a seen
        // -W^T of chunk kk from TMEM into the image, [c][i]; then the image is complete
        auto read_w = [&](uint32_t kk) -> bool {
            bool o = true;
            if (leader) o = fwait(&bars.w, kk & 1, err, 3, abort);
            if (!bar_and_named(NB_PREP, 256, o)) return false;
            fence_after_sync();
            float f[32];
            tmem_ld16(tmem + lane + TM_D + 32 * ph, f);
            tmem_ld16(tmem + lane + TM_D + 32 * ph + 16, f + 16);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<uint4*>(sm + F_W + sw128_offset(pc, 32 * ph + 8 * m)) = pack8(f + 8 * m);
            fence_smem_to_async();
            fence_before_sync();
            __syncwarp();
            if (l == 0) mbar_arrive(&bars.img);
            return true;
        };
        for (uint32_t k = 0; it.ok; ++k) {
            const int s = (int)(k & 1);
            const int len = it.len();
            // beta of row pc (threads of the first 64 channels), read at the extraction
            const float bcur = (q4 < 2 && pc < len) ? __ldg(beta + ((int64_t)it.t0() + pc) * H + it.h) : 0.f;
            // ---- (a) cumulative decay of channel pc over this half's tokens, log2 units
            // (rows past the chunk's end add nothing)
            bool ok = true;
            if (leader) ok = fwait(&bars.g, k & 1, err, 1, abort);
            if (!bar_and_named(NB_PREP, 256, ok)) break;
            float G[32];
            float run = 0.f;
#pragma unroll
            for (int y = 0; y < 32; ++y) {
                const float gy = sg[(32 * ph + y) * D + pc];
                run += (32 * ph + y < len) ? kLog2e * gy : 0.f;
                G[y] = run;
            }
            __syncwarp();
            if (l == 0) mbar_arrive(&bars.gc);    // the gate tile may take the next chunk's
            xch[ph * 128 + pc] = run;
            if (ph == 1) xch[256 + pc] = G[0];
            bar_sync_named(NB_PAIR + q4, 64);
            const float s0 = xch[pc], s1 = xch[128 + pc];
            const float G32 = s0 + xch[256 + pc];
            if (ph == 1) {
#pragma unroll
                for (int y = 0; y < 32; ++y) G[y] += s0;
            }
            const float Gl = s0 + s1;             // last row
            float mx = 0.f, mxw = 0.f;            // largest |G| and |G - s0| of these tokens
#pragma unroll
            for (int y = 0; y < 32; ++y) {
                mx = fmaxf(mx, fabsf(G[y]));
                mxw = fmaxf(mxw, fabsf(G[y] - s0));
            }

            // k^T, q^T of this chunk in TMEM; image slot s free (chunk k - 2 walked)
            if (leader) {
                ok = fwait(&bars.tr, k & 1, err, 1, abort);
                if (ok && k >= 2) ok = fwait(&bars.fr[s], ((k - 2) >> 1) & 1, err, 6, abort);
            }
            if (!bar_and_named(NB_PREP, 256, ok)) break;
            fence_after_sync();
            // T', -W^T and the A scratch (all in place of the previous chunk's): free once
            // MMA1 of chunk k - 1 has completed
            auto wait_m1 = [&]() -> bool {
                bool o = true;
                if (leader && k >= 1) o = fwait(&bars.m1, (k - 1) & 1, err, 6, abort);
                return bar_and_named(NB_PREP, 256, o);
            };
            // one exponent reference per chunk and channel: the chunk start while every |G|
            // is within kRange, else the first half's total s0 while every |G - s0| is (a
            // chunk decaying by up to twice the range); past that, the level passes
            bool fast = bar_and_named(NB_PREP, 256, !(mx > kRange));
            const bool wide = !fast && bar_and_named(NB_PREP, 256, !(mxw > kRange));
            fast = fast || wide;
            const float rref = wide ? s0 : 0.f;

            unsigned char* qg = sm + F_QG + s * 16384;
            unsigned char* kl = sm + F_KLAQ + s * 24576;
            unsigned char* aq = kl + 16384;
            auto load_kq = [&](int hb, float* kf, float* qf) {
                tmem_ld16(tmem + lane + TM_KT + 32 * ph + 16 * hb, kf);
                tmem_ld16(tmem + lane + TM_QT + 32 * ph + 16 * hb, qf);
                tmem_wait_ld();
                if (len < C) {
#pragma unroll
                    for (int y = 0; y < 16; ++y)
                        if (32 * ph + 16 * hb + y >= len) kf[y] = qf[y] = 0.f;
                }
            };
            auto warp_arrive = [&](uint64_t* b) {
                fence_smem_to_async();
                fence_before_sync();
                __syncwarp();
                if (l == 0) mbar_arrive(b);
            };
            auto wait_a = [&]() -> bool {
                bool o2 = true;
                if (leader) o2 = fwait(&bars.a, n_a & 1, err, 2, abort);
                ++n_a;
                o2 = bar_and_named(NB_PREP, 256, o2);
                fence_after_sync();
                return o2;
            };
            auto put_gamma = [&] {
                if (ph == 0) reinterpret_cast<float*>(sm + F_GAM + s * 512)[pc] = ex2(Gl);
            };
            // the operand tiles are complete: the leader issues [K e^G; Q e^G] (K e^{-G})^T
            // (`fenced`: this thread's tile writes already passed a proxy fence)
            auto issue_a = [&](bool fenced) {
                if (!fenced) fence_smem_to_async();
                fence_before_sync();
                bar_sync_named(NB_PREP, 256);
                if (leader) {
                    fence_after_sync();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tmem + TM_D, (s ? dRow1 : dRow0) + 128u * ks, dCol + 128u * ks, idA, ks > 0);
                    commit(&bars.a);
                }
            };

            if (fast) {
                // ---- (b1) e^{G_i - G_j} = e^{G_i - r} e^{r - G_j} with the reference r = 0 or s0:
                // K e^{G - r}, Q e^{G - r} (with r = 0 the image tiles K e^G, Q e^G) are the row
                // operands of A and Aqk, K e^{r - G} the column operand; K e^{Gl - G} =
                // K e^{r - G} e^{Gl - r}
                const float Egl = ex2(Gl - rref);
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    float kf[16], qf[16];
                    load_kq(hb, kf, qf);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        float a8[8], b8[8], c8[8], d8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int y = 8 * m + e;
                            const float gg = G[16 * hb + y] - rref;
                            const float e1 = ex2(gg), e2 = ex2(-gg);
                            a8[e] = kf[y] * e1;
                            b8[e] = qf[y] * e1;
                            c8[e] = kf[y] * e2;
                            d8[e] = c8[e] * Egl;
                        }
                        const uint32_t off = ct_off(pc, 32 * ph + 16 * hb + 8 * m);
                        *reinterpret_cast<uint4*>(sm + F_KG + off) = pack8(a8);
                        *reinterpret_cast<uint4*>(qg + off) = pack8(b8);
                        *reinterpret_cast<uint4*>(sm + F_KD + off) = pack8(c8);
                        *reinterpret_cast<uint4*>(kl + off) = pack8(d8);
                    }
                }
                put_gamma();
                // one proxy fence for the tiles; e^{G_last} is read by the walk warps (generic)
                // and k^T, q^T have been read (the next chunk's may land)
                fence_smem_to_async();
                fence_before_sync();
                __syncwarp();
                if (l == 0) mbar_arrive(&bars.gam);
                issue_a(true);
                if (!wait_m1()) break;
                if (!wait_a()) break;
                if (wide) {
                    // A has read the s0-referenced rows: the image tiles K e^G, Q e^G are
                    // written again at the chunk start (from k^T, q^T, still in TMEM), as the
                    // chunk-start reference writes them
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        float kf[16], qf[16];
                        load_kq(hb, kf, qf);
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            float a8[8], b8[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float e1 = ex2(G[16 * hb + 8 * m + e]);
                                a8[e] = kf[8 * m + e] * e1;
                                b8[e] = qf[8 * m + e] * e1;
                            }
                            const uint32_t off = ct_off(pc, 32 * ph + 16 * hb + 8 * m);
                            *reinterpret_cast<uint4*>(sm + F_KG + off) = pack8(a8);
                            *reinterpret_cast<uint4*>(qg + off) = pack8(b8);
                        }
                    }
                }
                // k^T, q^T were read before A was issued (and again just above for a chunk
                // referenced to s0); signalled only now so that the next chunk's transposes
                // do not queue ahead of A on the tensor pipe
                if (l == 0) mbar_arrive(&bars.ktf);
                // ---- A (fp32, beta-scaled rows, for the inverse) and Aqk (bf16 image)
                float d[32];
                tmem_ld16(tmem + lane + TM_D + 32 * ph, d);
                tmem_ld16(tmem + lane + TM_D + 32 * ph + 16, d + 16);
                tmem_wait_ld();
                if (q4 < 2) {
                    const int i = pc;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        float4 v4;
                        const int j = 32 * ph + 4 * m;
                        v4.x = (j + 0 < i) ? bcur * d[4 * m + 0] : 0.f;
                        v4.y = (j + 1 < i) ? bcur * d[4 * m + 1] : 0.f;
                        v4.z = (j + 2 < i) ? bcur * d[4 * m + 2] : 0.f;
                        v4.w = (j + 3 < i) ? bcur * d[4 * m + 3] : 0.f;
                        *reinterpret_cast<float4*>(sA + i * AP + j) = v4;
                    }
                    if (ph == 0) sB[i] = bcur;
                } else {
                    const int i = pc - 64;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float a8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) a8[e] = (32 * ph + 8 * m + e <= i) ? d[8 * m + e] : 0.f;
                        *reinterpret_cast<uint4*>(aq + sw128_offset(i, 32 * ph + 8 * m)) = pack8(a8);
                    }
                }
            } else {
                // ---- (b1') the level passes: every factor <= 1 (log_alpha <= 0).  The image
                // tiles K e^G and Q e^G hold each pass's row operands and are written last.
                if (!wait_m1()) break;
                for (int e = tid; e < 64 * AP / 4; e += 256)
                    reinterpret_cast<float4*>(sA)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int e = tid; e < 512; e += 256)
                    reinterpret_cast<uint4*>(aq)[e] = make_uint4(0, 0, 0, 0);
                if (q4 < 2 && ph == 0) sB[pc] = bcur;
                float Gs[32];                     // indexed at run time (local memory)
#pragma unroll
                for (int y = 0; y < 32; ++y) Gs[y] = G[y];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {  // K e^{Gl - G} (<= 1) and e^{G_last}
                    float kf[16], qf[16];
                    load_kq(hb, kf, qf);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        float c8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) c8[e] = kf[8 * m + e] * ex2(Gl - G[16 * hb + 8 * m + e]);
                        *reinterpret_cast<uint4*>(kl + ct_off(pc, 32 * ph + 16 * hb + 8 * m)) = pack8(c8);
                    }
                }
                put_gamma();
                warp_arrive(&bars.gam);
                bar_sync_named(NB_PREP, 256);     // zeroed A / Aqk before any pass writes
                bool pok = true;
                for (int pass = 0; pass < 8 && pok; ++pass) {
                    // passes 0-5: the levels; 6: the diagonal; 7: the image tiles K e^G, Q e^G
                    // (no MMA)
                    const int hs = 32 >> pass;    // half block of this level (pass < 6)
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        float kf[16], qf[16];
                        load_kq(hb, kf, qf);
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            float kin[8], qin[8], kd[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int y = 8 * m + e, t = 32 * ph + 16 * hb + y;
                                if (pass >= 6) {
                                    const float eg = pass == 7 ? ex2(G[16 * hb + y]) : 1.f;
                                    kin[e] = kf[y] * eg; qin[e] = qf[y] * eg; kd[e] = kf[y];
                                } else {
                                    const bool up = (t & (2 * hs - 1)) >= hs;
                                    const int f = (t & ~(2 * hs - 1)) + hs;
                                    const float Gf = (hs == 32) ? G32 : Gs[f - 32 * ph];
                                    const float x = G[16 * hb + y] - Gf;   // <= 0 up, >= 0 below
                                    const float ef = ex2(up ? x : -x);
                                    kin[e] = up ? kf[y] * ef : 0.f;
                                    qin[e] = up ? qf[y] * ef : 0.f;
                                    kd[e] = up ? 0.f : kf[y] * ef;
                                }
                            }
                            const uint32_t off = ct_off(pc, 32 * ph + 16 * hb + 8 * m);
                            *reinterpret_cast<uint4*>(sm + F_KG + off) = pack8(kin);
                            *reinterpret_cast<uint4*>(qg + off) = pack8(qin);
                            if (pass < 7) *reinterpret_cast<uint4*>(sm + F_KD + off) = pack8(kd);
                        }
                    }
                    if (pass == 7) break;
                    issue_a(false);
                    if (!(pok = wait_a())) break;
                    float d[32];
                    tmem_ld16(tmem + lane + TM_D + 32 * ph, d);
                    tmem_ld16(tmem + lane + TM_D + 32 * ph + 16, d + 16);
                    tmem_wait_ld();
                    if (q4 < 2) {
                        const int i = pc;
                        if (pass < 6)
                            for (int y = 0; y < 32; ++y)
                                if (pass_pair(pass, i, 32 * ph + y)) sA[i * AP + 32 * ph + y] = bcur * d[y];
                    } else {
                        const int i = pc - 64;
                        for (int y = 0; y < 32; ++y)
                            if (pass_pair(pass, i, 32 * ph + y))
                                *reinterpret_cast<__nv_bfloat16*>(aq + sw128_offset(i, 32 * ph + y)) =
                                    __float2bfloat16_rn(d[y]);
                    }
                    fence_before_sync();          // TMEM reads before the next pass's MMA
                }
                if (!pok) break;
                warp_arrive(&bars.ktf);           // k^T, q^T read (pass 7 was the last)
            }
            if (fast) {
                // the inverse starts with the diagonal 16 x 16 blocks: warp 0 solves rows and
                // columns 0-31, which it extracted itself; warp 1 solves 32-63, extracted by
                // warp 5 (the image tiles reach the async proxy through the fence after the
                // inverse; the inverse's first barrier completes A for the later levels)
                if (q4 == 1) bar_sync_named(NB_PAIR + 1, 64);
                else if (w == 0) __syncwarp();
            } else {
                fence_smem_to_async();            // Aqk, K e^G, Q e^G: read by the async proxy
                bar_sync_named(NB_PREP, 256);     // A complete
            }
            // ---- (b2) T = (I + A)^{-1} and the bf16 T' = T diag(beta)
            invert_unit_lower(sA, sT, sm + F_TP, sB, tid);
            // ---- (b3) -W^T = -(K e^G)^T T'^T: the leader's MMA into the A / Aqk columns
            // (read out above)
            fence_smem_to_async();
            fence_before_sync();
            bar_sync_named(NB_PREP, 256);
            if (leader) {
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_D, dKgT + 2u * ks, dTp + 2u * ks, idW, ks > 0);
                commit(&bars.w);
            }
            if (!read_w(k)) break;
            it.next(false, sc, si, H32, slots, P, err, abort);
        }
        // the leader's MMAs have completed before the CTA frees its tensor memory
        if (leader) {
            commit(&bars.fin_q);
            mbar_wait(&bars.fin_q, 0, nullptr, 0, 200);
        }
    } else if (w < W_PI) {
        // ------------------------------------------------------------------ walk
        const int q4 = w & 3;
        const int j = 32 * q4 + l;                // value column = TMEM lane of S^T, U^T, O^T
        const uint32_t lane = (uint32_t)(32 * q4) << 16;
        const bool wlead = tid == W_WALK * 32;
        // chains without tokens: final state = initial state
        for (int64_t r = blockIdx.x; hT && r < si.N * H; r += gridDim.x) {
            const int64_t sr = r / H, h = r - sr * H, n = si.seq_of(sr);
            int64_t bos, eos;
            seq_range(si.cu, n, si.T_seq, si.T_total, bos, eos);
            if (eos > bos) continue;
            int64_t sidx = n * H + h;
            if (slots) {
                const int64_t sl = slots[n];
                sidx = (sl >= 0 && sl < P) ? sl * H + h : -1;
            }
            if (sidx < 0) continue;
            for (int c = 0; c < D; ++c)
                hT[sidx * D * D + c * D + j] = h0 ? h0[sidx * D * D + c * D + j] : 0.f;
        }
        auto arrive4 = [&](uint64_t* b) {
            fence_before_sync();
            __syncwarp();
            if (l == 0) mbar_arrive(b);
        };
        auto wwait = [&](uint64_t* b, uint32_t par, int bit) -> bool {
            const bool o = gwait(b, par, wlead, NB_WALK, 128, err, bit, abort);
            fence_after_sync();
            return o;
        };
        // S^T fp32 -> bf16 operand copy; the fp32 state then decays by the next chunk's
        // e^{G_last} (slot g) before its update MMA accumulates onto it.  `src` (nullable:
        // zeros) replaces the TMEM state when a chain starts.
        auto stage_state = [&](const float* src, int g) {
            const float* gam = reinterpret_cast<const float*>(sm + F_GAM + g * 512);
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                float f[32];
                if (src) {
#pragma unroll
                    for (int y = 0; y < 32; ++y) f[y] = src[(32 * cb + y) * D + j];
                } else {
                    tmem_ld16(tmem + lane + TM_S + 32 * cb, f);
                    tmem_ld16(tmem + lane + TM_S + 32 * cb + 16, f + 16);
                    tmem_wait_ld();
                }
                uint32_t u[16];
#pragma unroll
                for (int y = 0; y < 16; ++y) u[y] = pack_bf16(f[2 * y], f[2 * y + 1]);
                tmem_st16u(tmem + lane + TM_SB + 16 * cb, u);
                float g8[32];
#pragma unroll
                for (int y = 0; y < 32; y += 8) ld8f(gam + 32 * cb + y, g8 + y);
#pragma unroll
                for (int y = 0; y < 32; ++y) f[y] *= g8[y];
                tmem_st16(tmem + lane + TM_S + 32 * cb, f);
                tmem_st16(tmem + lane + TM_S + 32 * cb + 16, f + 16);
            }
            tmem_wait_st();
            arrive4(&bars.sr);
        };
        Items it = it0;
        for (uint32_t k = 0; it.ok; ++k) {
            const int s = (int)(k & 1);
            if (it.first()) {                     // entry state (h0 or zeros), decayed by this chunk
                if (slots && wlead && err) {
                    const int64_t sl = slots[it.n];
                    if (sl >= P) atomicOr(err, 1);
                }
                if (!wwait(&bars.gam, k & 1, 6)) break;
                if (h0 && it.sidx >= 0) {
                    stage_state(h0 + it.sidx * D * D, s);
                } else {
                    float f[32];
#pragma unroll
                    for (int y = 0; y < 32; ++y) f[y] = 0.f;
#pragma unroll 1
                    for (int cb = 0; cb < 4; ++cb) {
                        tmem_st16(tmem + lane + TM_S + 32 * cb, f);
                        tmem_st16(tmem + lane + TM_S + 32 * cb + 16, f + 16);
                        uint32_t u[16];
#pragma unroll
                        for (int y = 0; y < 16; ++y) u[y] = 0u;
                        tmem_st16u(tmem + lane + TM_SB + 16 * cb, u);
                    }
                    tmem_wait_st();
                    arrive4(&bars.sr);
                }
            }
            // U^T -> bf16 operand (first 32 columns of its own TMEM range)
            if (!wwait(&bars.u, k & 1, 5)) break;
            {
                // all 64 columns are read before the packed halves overwrite the first 32
                float f[32], g[32];
                tmem_ld16(tmem + lane + TM_U, f);
                tmem_ld16(tmem + lane + TM_U + 16, f + 16);
                tmem_ld16(tmem + lane + TM_U + 32, g);
                tmem_ld16(tmem + lane + TM_U + 48, g + 16);
                tmem_wait_ld();
                uint32_t u[16];
#pragma unroll
                for (int y = 0; y < 16; ++y) u[y] = pack_bf16(f[2 * y], f[2 * y + 1]);
                tmem_st16u(tmem + lane + TM_U, u);
#pragma unroll
                for (int y = 0; y < 16; ++y) u[y] = pack_bf16(g[2 * y], g[2 * y + 1]);
                tmem_st16u(tmem + lane + TM_U + 16, u);
                tmem_wait_st();
                arrive4(&bars.ur);
            }
            // next entry state -> bf16 operand and decay, or the final state
            if (!wwait(&bars.s, k & 1, 5)) break;
            if (!it.last()) {
                if (!wwait(&bars.gam, (k + 1) & 1, 6)) break;
                stage_state(nullptr, s ^ 1);
            } else if (hT && it.sidx >= 0) {
                float* hp = hT + it.sidx * D * D;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    float f[16];
                    tmem_ld16(tmem + lane + TM_S + 16 * cb, f);
                    tmem_wait_ld();
#pragma unroll
                    for (int y = 0; y < 16; ++y) hp[(16 * cb + y) * D + j] = f[y];
                }
            }
            // output rows: [t][dv] bf16 tile in the consumed (Q e^G)^T slot, one tensor store
            // per whole chunk; the image slot is released once the store has read it
            if (!wwait(&bars.o, k & 1, 5)) break;
            unsigned char* stg = sm + F_QG + s * 16384;
            {
                float f[64];
#pragma unroll
                for (int x = 0; x < 4; ++x) tmem_ld16(tmem + lane + TM_O + 16 * x, f + 16 * x);
                tmem_wait_ld();
                arrive4(&bars.orr);
#pragma unroll
                for (int t = 0; t < 64; ++t)
                    *reinterpret_cast<__nv_bfloat16*>(stg + t * 256 + 2 * j) = __float2bfloat16_rn(scale * f[t]);
            }
            fence_smem_to_async();
            bar_sync_named(NB_WALK, 128);
            const int len = it.len();
            const int64_t t0 = it.t0();
            if (len == C) {
                if (wlead) {
                    tma::store_2d(&omap, (int32_t)(it.h * D), (int32_t)t0, stg);
                    tma::bulk_commit();
                    tma::bulk_wait_read();
                    mbar_arrive(&bars.fr[s]);
                }
            } else {
                for (int e = tid - W_WALK * 32; e < len * 16; e += 128) {
                    const int r = e >> 4, c = e & 15;
                    *reinterpret_cast<uint4*>(out + ((t0 + r) * H + it.h) * D + 8 * c) =
                        *reinterpret_cast<const uint4*>(stg + r * 256 + c * 16);
                }
                bar_sync_named(NB_WALK, 128);
                if (wlead) mbar_arrive(&bars.fr[s]);
            }
            it.next(false, sc, si, H32, slots, P, err, abort);
        }
        if (wlead) tma::bulk_wait_all();
    } else if (w == W_PI) {
        // ------------------------------------------------------------------ prep issuer
        if (l == 0) {
            auto issue_g = [&](const Items& x) {
                tma::expect_tx(&bars.g, 32768);
                tma::load_2d(sm + F_G, &gmap, (int32_t)(x.h * D), (int32_t)x.t0(), &bars.g);
            };
            auto issue_kq = [&](const Items& x) {
                const int32_t y = (int32_t)x.t0(), xc = (int32_t)(x.h * D);
                tma::expect_tx(&bars.kq, 32768);
                tma::load_2d(sm + F_KQ, &kmap, xc, y, &bars.kq);
                tma::load_2d(sm + F_KQ + 8192, &kmap, xc + 64, y, &bars.kq);
                tma::load_2d(sm + F_KQ + 16384, &qmap, xc, y, &bars.kq);
                tma::load_2d(sm + F_KQ + 24576, &qmap, xc + 64, y, &bars.kq);
            };
            Items it = it0;
            uint32_t kq_issued = 0, kq_seen = 0, g_issued = 0;
            // k^T, q^T: each 16-token block of the [t][c] tiles times I16 (exact)
            const uint32_t idT = make_idesc_bf16(128, 16, true, false);
            const uint64_t dI = make_desc(smem_u32(sm + F_ID), 16, 1024);
            const uint64_t dK = make_desc(smem_u32(sm + F_KQ), 8192, 1024);
            const uint64_t dQ = make_desc(smem_u32(sm + F_KQ + 16384), 8192, 1024);
            if (it.ok) { issue_g(it); ++g_issued; issue_kq(it); ++kq_issued; }
            for (uint32_t k = 0; it.ok; ++k) {
                Items nx = it;
                nx.next(true, sc, si, H32, slots, P, err, abort);
                if (!fwait(&bars.kq, k & 1, err, 1, abort)) break;
                ++kq_seen;
                // the prep threads have read chunk k - 1's k^T, q^T
                if (k > 0 && !fwait(&bars.ktf, (k - 1) & 1, err, 6, abort)) break;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    mma_bf16(tmem + TM_KT + 16 * ks, dK + 128u * ks, dI, idT, 0u);
                    mma_bf16(tmem + TM_QT + 16 * ks, dQ + 128u * ks, dI, idT, 0u);
                }
                commit(&bars.tr);
                // the k / q buffer is free once the transposes have read it, the gate tile once
                // the prep threads have scanned it
                if (!fwait(&bars.tr, k & 1, err, 1, abort)) break;
                if (nx.ok) { issue_kq(nx); ++kq_issued; }
                if (!fwait(&bars.gc, k & 1, err, 6, abort)) break;
                if (nx.ok) { issue_g(nx); ++g_issued; }
                it = nx;
            }
            // drain: this thread's MMAs and copies
            commit(&bars.fin_p);
            mbar_wait(&bars.fin_p, 0, nullptr, 0, 200);
            while (kq_seen < kq_issued) {
                mbar_wait(&bars.kq, kq_seen & 1, nullptr, 0, 200);
                ++kq_seen;
            }
            // gate tiles: the prep threads wait for each one they scan; at most the one issued
            // for a chunk that was never started is left in flight
            if (*abort) mbar_wait(&bars.g, (g_issued - 1) & 1, nullptr, 0, 200);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ walk issuer
        if (l == 0) {
            auto issue_v = [&](const Items& x) {
                const int32_t y = (int32_t)x.t0(), xc = (int32_t)(x.h * D);
                tma::expect_tx(&bars.v, 16384);
                tma::load_2d(sm + F_V, &vmap, xc, y, &bars.v);
                tma::load_2d(sm + F_V + 8192, &vmap, xc + 64, y, &bars.v);
            };
            Items it = it0;
            uint32_t v_issued = 0, v_seen = 0;
            if (it.ok) { issue_v(it); ++v_issued; }
            const uint32_t id_v = make_idesc_bf16(128, 64, true, false);   // V^T T'^T
            const uint64_t dV = make_desc(smem_u32(sm + F_V), 8192, 1024);
            const uint64_t dTp = make_desc(smem_u32(sm + F_TP), 16, 1024);
            // per image slot: the descriptors of slot 1 are those of slot 0 plus the slot
            // stride (16 KB for Q e^G and K e^{Gl - G}, 8 KB for Aqk) in 16-byte units
            // [(Q e^G)^T | -W^T] as one MN-major B of N = 128 (the -W^T block one LBO step
            // after the slot's Q e^G), [K e^{Gl - G} ; Aqk] as one K-major B of N = 192
            const uint64_t dQW0 = make_desc(smem_u32(sm + F_QG), F_W - F_QG, 1024);
            const uint64_t dQW1 = make_desc(smem_u32(sm + F_QG + 16384), F_W - F_QG - 16384, 1024);
            const uint64_t dKA0 = make_desc(smem_u32(sm + F_KLAQ), 16, 1024);
            const uint32_t id_uo = make_idesc_bf16(128, 128, false, true);
            const uint32_t id_so = make_idesc_bf16(128, 192, false, false);
            for (uint32_t k = 0; it.ok; ++k) {
                const int s = (int)(k & 1);
                const uint64_t dQW = s ? dQW1 : dQW0, dKA = dKA0 + (s ? 1536u : 0u);
                Items nx = it;
                nx.next(false, sc, si, H32, slots, P, err, abort);
                if (!fwait(&bars.img, k & 1, err, 6, abort)) break;
                if (!fwait(&bars.v, k & 1, err, 4, abort)) break;
                ++v_seen;
                if (!fwait(&bars.sr, k & 1, err, 6, abort)) break;
                if (k > 0 && !fwait(&bars.o, (k - 1) & 1, err, 5, abort)) break;
                // the output tile of the previous chunk has left TMEM
                if (k > 0 && !fwait(&bars.orr, (k - 1) & 1, err, 6, abort)) break;
                fence_after_sync();
                // [O^T | U^T] = S^T [(Q e^G)^T | -W^T], then U^T += V^T T'^T
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_SB + 8 * ks, dQW + 128u * ks, id_uo, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem + TM_U, dV + 128u * ks, dTp + 2u * ks, id_v, 1u);
                commit(&bars.u);
                if (!fwait(&bars.u, k & 1, err, 5, abort)) break;
                mbar_arrive(&bars.m1);            // T', -W^T and the v tile are free
                if (nx.ok) { issue_v(nx); ++v_issued; }
                if (!fwait(&bars.ur, k & 1, err, 6, abort)) break;
                fence_after_sync();
                // [S^T | O^T] += U^T [K e^{Gl - G} ; Aqk]
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) mma_bf16_ts(tmem + TM_S, tmem + TM_U + 8 * ks, dKA + 2u * ks, id_so, 1u);
                commit(&bars.s);
                commit(&bars.o);
                it = nx;
            }
            commit(&bars.fin_w);
            mbar_wait(&bars.fin_w, 0, nullptr, 0, 200);
            while (v_seen < v_issued) {
                mbar_wait(&bars.v, v_seen & 1, nullptr, 0, 200);
                ++v_seen;
            }
        }
        __syncwarp();
    }
    fence_before_sync();
    __syncthreads();
    if (w == W_PI) tmem_dealloc(tmem, 512);
}

}  // namespace fz

cudaError_t run_prefill_fused(const PrefillArgs& a, int* err, int* ticket, const int* run_if,
                              cudaStream_t st)
{
    static std::atomic<uint64_t> attrs_done{0};
    cudaError_t e = once_per_device(attrs_done, [] {
        return cudaFuncSetAttribute(fz::chunk_fused_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)fz::F_SMEM);
    });
    if (e) return e;
    const int64_t chains = a.si.N * a.H;
    if (chains <= 0 || a.si.T_total <= 0) {
        // no tokens: the final states are the initial ones
        if (a.hT && chains > 0) {
            // handled by the kernel's empty-chain pass (one CTA per SM at most)
        } else {
            return cudaSuccess;
        }
    }
    const uint64_t rows = (uint64_t)(a.si.T_total > 0 ? a.si.T_total : 1), cols = (uint64_t)a.H * fz::D;
    CUtensorMap kmap, qmap, vmap, omap;
    if ((e = make_tensor_map_2d(&kmap, a.k, true, cols, rows, cols * 2, 64, 64, true))) return e;
    if ((e = make_tensor_map_2d(&qmap, a.q, true, cols, rows, cols * 2, 64, 64, true))) return e;
    if ((e = make_tensor_map_2d(&vmap, a.v, true, cols, rows, cols * 2, 64, 64, true))) return e;
    if ((e = make_tensor_map_2d(&omap, a.out, true, cols, rows, cols * 2, fz::D, 64, false))) return e;
    CUtensorMap gmap;                             // log_alpha [tokens][H * D] fp32, 128 x 64 boxes
    if ((e = make_tensor_map_2d(&gmap, a.log_alpha, false, cols, rows, cols * 4, fz::D, 64, false))) return e;
    const int64_t sms = device_sm_count();
    const unsigned grid = (unsigned)(chains < sms ? chains : sms);
    // packed sequences of mixed lengths: chains handed out by tickets (the counter is
    // zeroed here, in stream order); equal-length chains: the static order balances
    if (ticket && (e = cudaMemsetAsync(ticket, 0, sizeof(int), st))) return e;
    LaunchScope scope(st, K_FUSED_TC);
    fz::chunk_fused_tc_kernel<<<grid, fz::NT, fz::F_SMEM, st>>>(
        kmap, qmap, vmap, omap, gmap, a.log_alpha, a.beta, a.h0, (__nv_bfloat16*)a.out, a.hT, a.scale, a.si,
        a.H, a.slots, a.P, err, ticket, run_if);
    return cudaGetLastError();
}

}  // namespace kda
