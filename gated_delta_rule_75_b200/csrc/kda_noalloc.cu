// kda_chunk_fwd_noalloc: the chunkwise prefill without any device allocation.
//
// Who needs this: hosts that reserve all device memory up front and forbid
// allocation afterwards -- serving engines that carve the whole GPU into their
// own pools at start-up, or plugin interfaces that hand a plugin its tensors
// but no allocator -- cannot let a library call cudaMalloc (or a pool
// allocator) in the middle of a request: the call may fail because the memory
// is already reserved, or it may stall the request.  For them this entry point
// runs the fp32 SIMT chunk kernels on a fixed scratch area that lives in the
// library itself (a file-scope __device__ array), so a call allocates nothing.
//
// Rules of use (also stated in kda.h):
//  * the scratch is KDA_NOALLOC_SCRATCH_BYTES per GPU, held from the moment the
//    library's kernels are loaded on that GPU until the process exits;
//  * problems that do not fit are rejected with KDA_ERR_UNSUPPORTED before
//    anything is launched;
//  * every call on a GPU shares the one array and it keeps the previous call's
//    contents; calls whose work overlaps on the GPU (different streams without
//    ordering between them) race on it and must be serialised by the caller;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before any stream capture.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "kda.h"
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

// The scratch area.  In host code this name is only a host-side stand-in:
// its device address must come from cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current.
static cudaError_t noalloc_scratch_ptr(void** out)
{
    static std::mutex mu;
    static void* ptrs[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return cudaSuccess;
}

}  // namespace kda

using namespace kda;

extern "C" KDA_API kda_status_t kda_chunk_fwd_noalloc(
    const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
    const float* h0, void* out, float* hT, const int32_t* cu_seqlens, int64_t B, int64_t T,
    int64_t H, int64_t dk, int64_t dv, float scale, kda_io_dtype_t io_dtype, cudaStream_t stream)
{
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (io_dtype != KDA_IO_F32 && io_dtype != KDA_IO_BF16) return KDA_ERR_UNSUPPORTED;
    if (!(dk == 64 || dk == 128) || !(dv == 64 || dv == 128)) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens != nullptr && B < 1) return KDA_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return KDA_OK;
    const int64_t T_total = cu_seqlens ? T : B * T;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
    if (T_total > 0) {
        const void* ptrs[] = {q, k, v, log_alpha, out};
        for (const void* p : ptrs)
            if (p == nullptr || !a16(p)) return KDA_ERR_INVALID_ARG;
        if (beta == nullptr || !a4(beta)) return KDA_ERR_INVALID_ARG;
        if (out == q || out == k || out == v || out == log_alpha || out == beta)
            return KDA_ERR_INVALID_ARG;
    }
    if ((h0 && !a16(h0)) || (hT && !a16(hT))) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && !a4(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (T_total > (int64_t(1) << 40) || H > 65535) return KDA_ERR_UNSUPPORTED;
    if (B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;

    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.h0 = h0;
    a.out = out; a.hT = hT; a.H = H; a.dk = (int)dk; a.dv = (int)dv; a.scale = scale;
    a.io = io_dtype;
    a.slots = nullptr;
    a.P = 0;
    a.err = nullptr;
    a.gate_scalar = false;
    SeqInfo& si = a.si;
    si.cu = cu_seqlens;
    si.chunk_off = nullptr;
    si.N = B;
    si.T_seq = cu_seqlens ? 0 : T;
    si.T_total = T_total;
    si.nct = cu_seqlens ? 0 : (T + kChunk - 1) / kChunk;
    si.chunks_upper = cu_seqlens ? (T / kChunk + B) : B * si.nct;
    si.order = nullptr;

    // scratch layout: [256 B reserved | chunk offsets | per-(chunk, head) blocks];
    // at least one head's chunks must fit, heads then run in groups that fit
    const int64_t blk = simt_ws_floats_per_chunk((int)dk, (int)dv) * (int64_t)sizeof(float);
    const int64_t off_bytes = cu_seqlens ? ((B + 1) * 8 + 255) / 256 * 256 : 0;
    const int64_t per_head = blk * (si.chunks_upper > 0 ? si.chunks_upper : 1);
    const int64_t room = (int64_t)KDA_NOALLOC_SCRATCH_BYTES - 256 - off_bytes;
    if (room < per_head) return KDA_ERR_UNSUPPORTED;   // does not fit the fixed scratch
    int64_t Hg = room / per_head;
    if (Hg > H) Hg = H;

    void* base_v = nullptr;
    cudaError_t e = noalloc_scratch_ptr(&base_v);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    char* base = static_cast<char*>(base_v);
    // errors go to the library's device error word (kda_get_error); offsets and
    // blocks are fully written by the kernels before they are read
    int* err_flag = nullptr;
    if (library_error_word(&err_flag) != cudaSuccess) return KDA_ERR_CUDA;
    a.err = err_flag;
    if (cu_seqlens) {
        int64_t* chunk_off = reinterpret_cast<int64_t*>(base + 256);
        if (launch_chunk_offsets(cu_seqlens, B, T_total, si.chunks_upper, chunk_off, nullptr,
                                 err_flag, 0, 0, nullptr, stream) != cudaSuccess)
            return KDA_ERR_CUDA;
        si.chunk_off = chunk_off;
    }
    float* ws = reinterpret_cast<float*>(base + 256 + off_bytes);
    if (run_prefill_simt(a, ws, Hg, stream) != cudaSuccess) return KDA_ERR_CUDA;
    if (debug_mode_on()) {
        int flag = 0;
        if (take_error_word(stream, &flag) != cudaSuccess) return KDA_ERR_CUDA;
        return status_from_error_bits(flag);
    }
    return KDA_OK;
}
