// Self-test of the two bounded waits the kernels of this library use on their
// mbarriers (TMA copies, tensor-core MMAs, hand-offs between warps): one CTA waits
// on a barrier that nothing ever completes, first with the suspended poll (given up
// after `polls` polls; error bit 1), then with the spinning poll bounded by elapsed
// cycles (`polls` x 200000 cycles, about 0.1 ms per poll; error bit 2).  The CTA
// returns with no copy or MMA in flight, so the context stays usable.  Nothing here
// faults, traps or spins without a limit.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_umma.cuh"

namespace kda {

__global__ void bounded_wait_selftest_kernel(int* __restrict__ err, uint32_t polls)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);                 // one arrival expected; none comes
        umma::fence_mbar_init();
    }
    __syncthreads();
    int gave_up = 0;
    if (threadIdx.x == 0) {
        gave_up = umma::mbar_wait(&bar, 0, err, 1, polls) ? 0 : 1;
        gave_up += umma::mbar_wait_spin(&bar, 0, err, 2, (long long)polls * 200000LL) ? 0 : 1;
    }
    __syncthreads_or(gave_up);
}

cudaError_t launch_bounded_wait_selftest(int* err, uint32_t polls, cudaStream_t st)
{
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(err, polls);
    return cudaGetLastError();
}

}  // namespace kda

extern "C" {

kda_status_t kda_debug_bounded_wait(int32_t polls, int32_t* err_word, cudaStream_t stream)
{
    if (polls < 1 || polls > 20000 || (reinterpret_cast<uintptr_t>(err_word) & 3) != 0)
        return KDA_ERR_INVALID_ARG;
    if (err_word == nullptr) {                   // report into the library's error word
        int* lib_word = nullptr;
        if (kda::library_error_word(&lib_word) != cudaSuccess) return KDA_ERR_CUDA;
        if (kda::launch_bounded_wait_selftest(lib_word, (uint32_t)polls, stream) != cudaSuccess)
            return KDA_ERR_CUDA;
        return cudaStreamSynchronize(stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    if (cudaMemsetAsync(err_word, 0, sizeof(int32_t), stream) != cudaSuccess) return KDA_ERR_CUDA;
    if (kda::launch_bounded_wait_selftest(err_word, (uint32_t)polls, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    int32_t flag = 0;
    if (cudaMemcpyAsync(&flag, err_word, sizeof(int32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    return (flag & kda::kErrTimeoutMask) ? KDA_ERR_TIMEOUT : KDA_OK;
}

}  // extern "C"
