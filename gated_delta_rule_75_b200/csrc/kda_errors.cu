// The library's device error word: one int per GPU that every kernel of the
// library ORs its error bits into (malformed cu_seqlens or a state slot out of
// range: bit 0; a bounded wait that gave up: bits 1-6).  Nothing on the device
// reads it, so a call never stops or skips work because of an earlier call's
// bits; they stay set until kda_get_error takes them (read and clear in one
// atomic exchange, ordered after the work already queued on its stream).
#include <cuda_runtime.h>

#include <mutex>

#include "kda.h"
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

static __device__ int g_error_word;
// where the exchange leaves the taken bits for the copy to the host
static __device__ int g_error_taken;

cudaError_t library_error_word(int** out)
{
    static std::mutex mu;
    static int* ptrs[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_error_word);
        if (e != cudaSuccess) return e;
        ptrs[dev] = static_cast<int*>(p);
    }
    *out = ptrs[dev];
    return cudaSuccess;
}

__global__ void take_error_kernel(int* __restrict__ word, int* __restrict__ taken)
{
    *taken = atomicExch(word, 0);
}

cudaError_t take_error_word(cudaStream_t st, int* host_out)
{
    // one taker at a time per process: the exchange result passes through one
    // device word per GPU
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    int* word = nullptr;
    cudaError_t e = library_error_word(&word);
    if (e != cudaSuccess) return e;
    void* taken = nullptr;
    if ((e = cudaGetSymbolAddress(&taken, g_error_taken)) != cudaSuccess) return e;
    take_error_kernel<<<1, 1, 0, st>>>(word, static_cast<int*>(taken));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int v = 0;
    if ((e = cudaMemcpyAsync(&v, taken, sizeof(int), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    *host_out = v;
    return cudaSuccess;
}

kda_status_t status_from_error_bits(int bits)
{
    if (bits & kErrTimeoutMask) return KDA_ERR_TIMEOUT;
    if (bits & kErrSeqlens) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

}  // namespace kda

extern "C" KDA_API kda_status_t kda_get_error(cudaStream_t stream, int32_t* word)
{
    if (word == nullptr) return KDA_ERR_INVALID_ARG;
    int v = 0;
    if (kda::take_error_word(stream, &v) != cudaSuccess) return KDA_ERR_CUDA;
    *word = v;
    return KDA_OK;
}
