// Per-sequence chunk offsets for packed variable-length batches.
//
// One CTA scans the N sequence lengths (clamped into [0, T]) and writes
// chunk_off[n] = min(cap, sum_{m<n} ceil(L_m / 64)), n = 0..N, where cap is
// the number of chunk slots the workspace holds.  For well-formed offsets the
// sum never reaches past floor(T/64) + N = cap; for malformed ones (checked
// here: cu[0] == 0, non-decreasing, cu[N] == T; bit 0 of *err_flag is set
// otherwise) the cap keeps every chunk index the later kernels derive inside
// the workspace, so a malformed array cannot cause an out-of-bounds access.
//
// For the segment-parallel state walk it also writes seg_off[n], the first
// segment of sequence n when every sequence's chunk slots are cut into
// segments of seg_len chunks (an empty sequence still gets one segment, which
// carries its initial state through), capped at seg_cap like the chunk offsets.
#include <cub/block/block_scan.cuh>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kScanThreads = 512;    // 57 registers: no spill (1024 threads cap them at 64)

__global__ void __launch_bounds__(kScanThreads)
chunk_offsets_kernel(const int32_t* __restrict__ cu, int64_t N, int64_t T_total, int64_t cap,
                     int64_t* __restrict__ chunk_off, int32_t* __restrict__ order,
                     int* __restrict__ err, int64_t seg_len, int64_t seg_cap,
                     int64_t* __restrict__ seg_off)
{
    griddep_wait();
    griddep_launch_dependents();
    using Scan = cub::BlockScan<int64_t, kScanThreads>;
    __shared__ typename Scan::TempStorage tmp;
    __shared__ int64_t carry;
    if (threadIdx.x == 0) {
        carry = 0;
        if (cu[0] != 0 || cu[N] != T_total) atomicOr(err, 1);
    }
    __syncthreads();
    for (int64_t base = 0; base < N; base += kScanThreads) {
        const int64_t n = base + threadIdx.x;
        int64_t nc = 0;
        if (n < N) {
            int64_t bos, eos;
            seq_range(cu, n, 0, T_total, bos, eos);
            nc = (eos - bos + kChunk - 1) / kChunk;
            if (cu[n + 1] < cu[n]) atomicOr(err, 1);
        }
        int64_t excl, total;
        Scan(tmp).ExclusiveSum(nc, excl, total);
        if (n < N) chunk_off[n] = (carry + excl) < cap ? (carry + excl) : cap;
        __syncthreads();
        if (threadIdx.x == 0) carry += total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        if (carry > cap) atomicOr(err, 1);
        chunk_off[N] = carry < cap ? carry : cap;
    }
    if (seg_off != nullptr) {
        __syncthreads();
        if (threadIdx.x == 0) carry = 0;
        __syncthreads();
        for (int64_t base = 0; base < N; base += kScanThreads) {
            const int64_t n = base + threadIdx.x;
            int64_t ns = 0;
            if (n < N) {
                const int64_t c = chunk_off[n + 1] - chunk_off[n];
                ns = c > 0 ? (c + seg_len - 1) / seg_len : 1;
            }
            int64_t excl, total;
            Scan(tmp).ExclusiveSum(ns, excl, total);
            if (n < N) seg_off[n] = (carry + excl) < seg_cap ? (carry + excl) : seg_cap;
            __syncthreads();
            if (threadIdx.x == 0) carry += total;
            __syncthreads();
        }
        if (threadIdx.x == 0) seg_off[N] = carry < seg_cap ? carry : seg_cap;
    }
    if (order == nullptr) return;
    // rank sequences by chunk count, longest first (ties: lower index first):
    // order[rank] = sequence
    __syncthreads();
    for (int64_t n = threadIdx.x; n < N; n += kScanThreads) {
        const int64_t cn = chunk_off[n + 1] - chunk_off[n];
        int64_t rank = 0;
        for (int64_t m = 0; m < N; ++m) {
            const int64_t cm = chunk_off[m + 1] - chunk_off[m];
            rank += (cm > cn) || (cm == cn && m < n);
        }
        order[rank] = (int32_t)n;
    }
}

cudaError_t launch_chunk_offsets(const int32_t* cu, int64_t N, int64_t T_total, int64_t cap,
                                 int64_t* chunk_off, int32_t* order, int* err_flag,
                                 int64_t seg_len, int64_t seg_cap, int64_t* seg_off,
                                 cudaStream_t st)
{
    if (seg_off != nullptr && seg_len < 1) return cudaErrorInvalidValue;
    LaunchScope scope(st, K_CHUNK_OFFSETS);
    return launch_pdl(chunk_offsets_kernel, dim3(1), dim3(kScanThreads), 0, st, cu, N, T_total, cap,
                      chunk_off, order, err_flag, seg_len, seg_cap, seg_off);
}

}  // namespace kda
