// C ABI of the KDA library: argument checks, workspace, dispatch.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kda.h"
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

bool debug_mode_on()
{
    static const bool on = [] {
        const char* s = std::getenv("KDA_DEBUG");
        return s != nullptr && s[0] == '1';
    }();
    return on;
}

static bool debug_mode() { return debug_mode_on(); }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

static bool head_ok(int64_t d) { return d == 64 || d == 128; }

// Library-owned, per-device CUDA memory pool for stream-ordered workspace.
// Memory freed with cudaFreeAsync stays cached in the pool (release threshold
// set to the maximum), so repeated calls do not go back to the driver.
static cudaMemPool_t workspace_pool(int dev)
{
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (pools[dev] == nullptr) {
        cudaMemPoolProps props;
        std::memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return nullptr;
        uint64_t thr = ~0ull;
        cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
        pools[dev] = p;
    }
    return pools[dev];
}

// Workspace budget per call (bytes); heads are processed in groups that fit.
// KDA_WORKSPACE_MB fixes it; otherwise it is 60 % of the device memory that
// was free when the library first ran on the device, but at least 4 GiB
// (queried once per device: the query is too slow for every call).
static int64_t workspace_budget()
{
    static const int64_t fixed = [] {
        const char* s = std::getenv("KDA_WORKSPACE_MB");
        if (!s) return int64_t(0);
        int64_t mb = std::atoll(s);
        if (mb < 64) mb = 64;
        return mb << 20;
    }();
    if (fixed) return fixed;
    static std::mutex mu;
    static int64_t cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return int64_t(4) << 30;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        size_t free_b = 0, total_b = 0;
        int64_t b = int64_t(4) << 30;
        if (cudaMemGetInfo(&free_b, &total_b) == cudaSuccess) {
            const int64_t f = (int64_t)(0.6 * (double)free_b);
            if (f > b) b = f;
        }
        cached[dev] = b;
    }
    return cached[dev];
}

static kda_status_t from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return KDA_OK;
    if (e == cudaErrorMemoryAllocation) return KDA_ERR_NO_MEMORY;
    return KDA_ERR_CUDA;
}

// Stream-ordered allocation that is always released on scope exit.
struct StreamBuffer {
    void* ptr = nullptr;
    cudaStream_t st = nullptr;
    cudaError_t alloc(size_t bytes, cudaStream_t s) {
        st = s;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e) return e;
        cudaMemPool_t pool = workspace_pool(dev);
        if (!pool) return cudaErrorMemoryAllocation;
        return cudaMallocFromPoolAsync(&ptr, bytes, pool, s);
    }
    ~StreamBuffer() {
        if (ptr) cudaFreeAsync(ptr, st);
    }
};

}  // namespace kda

using namespace kda;

extern "C" {

kda_status_t kda_workspace_high_water(int64_t* bytes, int reset)
{
    if (bytes == nullptr) return KDA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    cudaMemPool_t pool = workspace_pool(dev);
    if (!pool) return KDA_ERR_CUDA;
    uint64_t v = 0;
    if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &v) != cudaSuccess)
        return KDA_ERR_CUDA;
    *bytes = (int64_t)v;
    if (reset) {
        uint64_t zero = 0;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

const char* kda_status_string(kda_status_t s)
{
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_NO_MEMORY: return "workspace allocation failed";
    case KDA_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

int kda_version(void) { return 100; }

}  // extern "C"

namespace kda {

static kda_status_t recurrent_step_impl(const void* q, const void* k, const void* v,
                                        const float* log_alpha, const float* beta, float* state,
                                        const int32_t* slots, void* out, int64_t N, int64_t P,
                                        int64_t H, int64_t dk, int64_t dv, float scale,
                                        kda_io_dtype_t io_dtype, bool gate_scalar,
                                        cudaStream_t stream)
{
    if (N < 0 || H < 0 || P < 0) return KDA_ERR_INVALID_ARG;
    if (io_dtype != KDA_IO_F32 && io_dtype != KDA_IO_BF16) return KDA_ERR_UNSUPPORTED;
    if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return KDA_OK;
    const void* ptrs[] = {q, k, v, state, out};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (log_alpha == nullptr || !(gate_scalar ? aligned4(log_alpha) : aligned16(log_alpha)))
        return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (slots && !aligned4(slots)) return KDA_ERR_INVALID_ARG;
    if (out == q || out == k || out == v || out == state) return KDA_ERR_INVALID_ARG;
    DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.state = state;
    a.out = out; a.N = N; a.H = H; a.P = slots ? P : N; a.dk = (int)dk; a.dv = (int)dv;
    a.scale = scale; a.io = io_dtype; a.slots = slots; a.err = nullptr;
    a.gate_scalar = gate_scalar;
    cudaError_t e = cudaSuccess;
    // only a slot out of range sets a bit here
    if (slots && (e = library_error_word(&a.err))) return from_cuda(e);
    e = launch_decode(a, stream);
    if (e == cudaSuccess && debug_mode()) {
        int flag = 0;
        if ((e = take_error_word(stream, &flag))) return from_cuda(e);
        return status_from_error_bits(flag);
    }
    return from_cuda(e);
}

static kda_status_t chunk_fwd_impl(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, const float* h0,
                                   void* out, float* hT, const int32_t* slots, int64_t P,
                                   const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                                   int64_t dk, int64_t dv, float scale, kda_io_dtype_t io_dtype,
                                   kda_prefill_impl_t impl, bool gate_scalar, cudaStream_t stream,
                                   float* maps = nullptr, float* offs = nullptr);

}  // namespace kda

extern "C" {

kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, float* state,
                                void* out, int64_t N, int64_t H, int64_t dk, int64_t dv,
                                float scale, kda_io_dtype_t io_dtype, cudaStream_t stream)
{
    return recurrent_step_impl(q, k, v, log_alpha, beta, state, nullptr, out, N, N, H, dk, dv,
                               scale, io_dtype, false, stream);
}

kda_status_t kda_gdn_recurrent_step(const void* q, const void* k, const void* v,
                                    const float* log_a, const float* beta, float* state,
                                    void* out, int64_t N, int64_t H, int64_t dk, int64_t dv,
                                    float scale, kda_io_dtype_t io_dtype, cudaStream_t stream)
{
    return recurrent_step_impl(q, k, v, log_a, beta, state, nullptr, out, N, N, H, dk, dv,
                               scale, io_dtype, true, stream);
}

kda_status_t kda_recurrent_step_slots(const void* q, const void* k, const void* v,
                                      const float* log_alpha, const float* beta,
                                      float* state_pool, const int32_t* slots, void* out,
                                      int64_t N, int64_t P, int64_t H, int64_t dk, int64_t dv,
                                      float scale, kda_io_dtype_t io_dtype, cudaStream_t stream)
{
    if (slots == nullptr) return KDA_ERR_INVALID_ARG;
    return recurrent_step_impl(q, k, v, log_alpha, beta, state_pool, slots, out, N, P, H, dk,
                               dv, scale, io_dtype, false, stream);
}

kda_status_t kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta, const float* h0,
                              void* out, float* hT, const int32_t* cu_seqlens, int64_t B,
                              int64_t T, int64_t H, int64_t dk, int64_t dv, float scale,
                              kda_io_dtype_t io_dtype, kda_prefill_impl_t impl,
                              cudaStream_t stream)
{
    return chunk_fwd_impl(q, k, v, log_alpha, beta, h0, out, hT, nullptr, 0, cu_seqlens, B, T, H,
                          dk, dv, scale, io_dtype, impl, false, stream);
}

kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* log_a,
                               const float* beta, const float* h0, void* out, float* hT,
                               const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                               int64_t dk, int64_t dv, float scale, kda_io_dtype_t io_dtype,
                               kda_prefill_impl_t impl, cudaStream_t stream)
{
    return chunk_fwd_impl(q, k, v, log_a, beta, h0, out, hT, nullptr, 0, cu_seqlens, B, T, H,
                          dk, dv, scale, io_dtype, impl, true, stream);
}

kda_status_t kda_chunk_fwd_slots(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta, float* state_pool,
                                 const int32_t* slots, void* out, const int32_t* cu_seqlens,
                                 int64_t B, int64_t T, int64_t P, int64_t H, int64_t dk,
                                 int64_t dv, float scale, kda_io_dtype_t io_dtype,
                                 kda_prefill_impl_t impl, cudaStream_t stream)
{
    if (slots == nullptr || state_pool == nullptr || P < 0) return KDA_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, beta, state_pool, out, state_pool, slots, P,
                          cu_seqlens, B, T, H, dk, dv, scale, io_dtype, impl, false, stream);
}

}  // extern "C"

namespace kda {

// Streaming multiprocessors of the current device (queried once per device).
int64_t device_sm_count()
{
    static std::mutex mu;
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Segment plan of the tensor-core state walk.  A chain per (sequence, head)
// runs one CTA per SM at most, so with fewer chains than about a quarter of
// the SMs the walk is latency-bound on its longest chain; cutting the chains
// into segments costs about three walks' worth of work (value, map, final) but
// runs them side by side.  The plan aims at about one segment-CTA per SM.
// Segment plan of the two-kernel tensor-core form: forced by SEGMENTED; under AUTO and
// TENSORCORE (`guarded`: the two-kernel form with the fused kernel as its fallback)
// only when there are few chains (at most a quarter of the SMs) and, for fixed-length
// batches, at least four segments per chain.
static SegPlan plan_segments(const SeqInfo& si, int64_t H, kda_prefill_impl_t impl, bool guarded)
{
    SegPlan p;
    std::memset(&p, 0, sizeof(p));
    if (si.chunks_upper <= 0) return p;
    if (impl != KDA_PREFILL_TENSORCORE_SEGMENTED && !guarded) return p;
    const bool force = impl == KDA_PREFILL_TENSORCORE_SEGMENTED;
    const int64_t sms = device_sm_count();
    const int64_t chains = si.N * H;
    if (!force && chains * 4 > sms) return p;
    if (si.cu == nullptr) {
        int64_t per_chain = sms / chains;
        if (per_chain < 2) per_chain = 2;
        const int64_t len = (si.nct + per_chain - 1) / per_chain;
        const int64_t nseg = (si.nct + len - 1) / len;
        if (!force && nseg < 4) return p;
        p.len = len;
        p.nseg = nseg;
        p.upper = si.N * nseg;
    } else {
        int64_t total = sms / H;                 // segments wanted over all sequences
        if (total < 2 * si.N) total = 2 * si.N;
        const int64_t len = (si.chunks_upper + total - 1) / total;
        if (!force && si.chunks_upper < 4 * len * si.N) return p;
        p.len = len;
        p.nseg = 0;
        p.upper = (si.chunks_upper + len - 1) / len + si.N;
    }
    return p;
}

static kda_status_t chunk_fwd_impl(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, const float* h0,
                                   void* out, float* hT, const int32_t* slots, int64_t P,
                                   const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                                   int64_t dk, int64_t dv, float scale, kda_io_dtype_t io_dtype,
                                   kda_prefill_impl_t impl, bool gate_scalar, cudaStream_t stream,
                                   float* maps, float* offs)
{
    // segmap mode: each (sequence, head)'s affine map instead of outputs
    const bool segmap = maps != nullptr || offs != nullptr;
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (io_dtype != KDA_IO_F32 && io_dtype != KDA_IO_BF16) return KDA_ERR_UNSUPPORTED;
    if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (impl < KDA_PREFILL_AUTO || impl > KDA_PREFILL_TENSORCORE_FUSED)
        return KDA_ERR_INVALID_ARG;
    // the tensor-core kernels address token rows with 32-bit TMA coordinates
    const int64_t T_rows = cu_seqlens ? T : B * T;
    const bool tc_shape = io_dtype == KDA_IO_BF16 && dk == 128 && dv == 128 &&
                          T_rows < (int64_t(1) << 31);
    const bool tc_forced = impl != KDA_PREFILL_AUTO && impl != KDA_PREFILL_SIMT;
    if (tc_forced && !tc_shape) return KDA_ERR_UNSUPPORTED;
    const bool use_tc = tc_forced || (impl == KDA_PREFILL_AUTO && tc_shape);
    if (cu_seqlens != nullptr && B < 1) return KDA_ERR_INVALID_ARG;
    if (segmap) {
        if (maps == nullptr || offs == nullptr || !aligned16(maps) || !aligned16(offs))
            return KDA_ERR_INVALID_ARG;
        if (maps == offs) return KDA_ERR_INVALID_ARG;
    }
    if (B == 0 || H == 0) return KDA_OK;
    const int64_t T_total = cu_seqlens ? T : B * T;
    if (T_total > 0) {
        const void* ptrs[] = {q, k, v, segmap ? (const void*)maps : out};
        for (const void* p : ptrs)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
        if (log_alpha == nullptr || !(gate_scalar ? aligned4(log_alpha) : aligned16(log_alpha)))
            return KDA_ERR_INVALID_ARG;
        if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
        if (!segmap && (out == q || out == k || out == v || out == log_alpha || out == beta))
            return KDA_ERR_INVALID_ARG;
    }
    if ((h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return KDA_ERR_INVALID_ARG;
    if (slots && !aligned4(slots)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0))
        return KDA_ERR_INVALID_ARG;
    // every index must fit the kernels' 64-bit arithmetic and 32-bit grid limits
    if (T_total > (int64_t(1) << 40) || H > 65535) return KDA_ERR_UNSUPPORTED;
    if (B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;   // one state-kernel block per (seq, head, tile)

    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.h0 = h0;
    a.out = out; a.hT = hT; a.H = H; a.dk = (int)dk; a.dv = (int)dv; a.scale = scale;
    a.io = io_dtype;
    a.slots = slots;
    a.P = P;
    a.err = nullptr;
    a.gate_scalar = gate_scalar;
    a.tc_what = 0;
    SeqInfo& si = a.si;
    si.cu = cu_seqlens;
    si.chunk_off = nullptr;
    si.N = B;
    si.T_seq = cu_seqlens ? 0 : T;
    si.T_total = T_total;
    si.nct = cu_seqlens ? 0 : (T + kChunk - 1) / kChunk;
    si.chunks_upper = cu_seqlens ? (T / kChunk + B) : B * si.nct;
    si.order = nullptr;

    // segment plan (tensor-core path): the segment-parallel walk, or in
    // segmap mode one segment per sequence written to the caller's buffers
    SegPlan& plan = a.seg;
    std::memset(&plan, 0, sizeof(plan));
    if (use_tc && segmap) {
        a.tc_what = 1;
        plan.len = int64_t(1) << 40;
        plan.nseg = 1;
        plan.upper = B;
        plan.maps = maps;
        plan.offs = offs;
        plan.hstride = H;
        plan.abs_head = true;
    }
    // AUTO / TENSORCORE (KDA form, outputs wanted, tokens present): the fused kernel,
    // which builds every chunk's operands on chip (no per-chunk workspace) and is exact
    // at any decay rate.  With few chains (at most half the SMs) the two-kernel form,
    // whose prep spreads over every SM, goes first: its prep flags any 16-token block
    // outside its decay range, its walks then do nothing, and the fused kernel launched
    // after them computes the call only in that case.
    const bool auto_tc = use_tc && !segmap && !gate_scalar && T_total > 0 &&
                         (impl == KDA_PREFILL_AUTO || impl == KDA_PREFILL_TENSORCORE);
    bool guarded = auto_tc && si.N * H * 2 <= device_sm_count();
    if (use_tc && !segmap) {
        plan = plan_segments(si, H, impl, guarded);
        if (plan.upper > 0x7fffffffLL / H) std::memset(&plan, 0, sizeof(plan));
    }
    // ... and only when every head fits one head group: with several groups, a group's walks
    // finish (writing hT, which may alias h0) before a later group's prep can flag a block,
    // and the fused kernel would then start those heads from overwritten states
    if (guarded) {
        const bool st = plan.len > 0 && cu_seqlens != nullptr;
        const int64_t ob =
            cu_seqlens ? ((B + 1) * 8 + (st ? (B + 1) * 8 : (B <= kMaxOrderedSeqs ? B * 4 : 0)) + 1023) /
                             1024 * 1024
                       : 0;
        const int64_t ph = tc_ws_bytes_per_chunk() * (si.chunks_upper > 0 ? si.chunks_upper : 1) +
                           tc_seg_bytes_per_head(plan);
        if ((workspace_budget() - 1024 - ob) / ph < H) {
            guarded = false;
            std::memset(&plan, 0, sizeof(plan));
        }
    }
    const bool seg_table = use_tc && !segmap && plan.len > 0 && cu_seqlens != nullptr;
    const bool use_fused = auto_tc ? !guarded : (impl == KDA_PREFILL_TENSORCORE_FUSED && !gate_scalar &&
                                                 !segmap && T_total > 0);

    // workspace: [1 KiB header (words 64, 65: see below) | chunk offsets (+ length order,
    // + segment offsets) | per head group: per-(chunk, head) blocks, segment
    // buffers | SIMT segmap extras]
    const int64_t blk_bytes =
        use_fused ? 0
        : use_tc ? tc_ws_bytes_per_chunk()
               : simt_ws_floats_per_chunk((int)dk, (int)(segmap && dk > dv ? dk : dv)) *
                     (int64_t)sizeof(float);
    const bool ordered = cu_seqlens != nullptr && B <= kMaxOrderedSeqs && !seg_table;
    const int64_t off_bytes =
        cu_seqlens ? ((B + 1) * 8 + (ordered ? B * 4 : 0) + (seg_table ? (B + 1) * 8 : 0) + 1023) /
                         1024 * 1024
                   : 0;
    const int64_t seg_bytes = (use_tc && !segmap && !use_fused) ? tc_seg_bytes_per_head(plan) : 0;
    const int64_t per_head = blk_bytes * (si.chunks_upper > 0 ? si.chunks_upper : 1) + seg_bytes;
    // SIMT segmap: zero values [T, H, dk], scratch outputs [T, H, max(dk, dv)],
    // identity initial states [N, H, dk, dk]
    const int64_t es = io_dtype == KDA_IO_BF16 ? 2 : 4;
    int64_t extra = 0, ex_v0 = 0, ex_out = 0, ex_eye = 0;
    if (segmap && !use_tc) {
        const int64_t dm = dk > dv ? dk : dv;
        ex_v0 = 0;
        ex_out = (T_total * H * dk * es + 1023) / 1024 * 1024;
        ex_eye = ex_out + (T_total * H * dm * es + 1023) / 1024 * 1024;
        extra = ex_eye + B * H * dk * dk * 4;
    }
    const int64_t budget = workspace_budget() - 1024 - off_bytes - extra;
    int64_t Hg = per_head > 0 ? budget / per_head : H;
    if (Hg < 1) Hg = 1;
    if (Hg > H) Hg = H;
    const int64_t ws_bytes = 1024 + off_bytes + Hg * per_head + (extra ? extra + 1024 : 0);

    StreamBuffer buf;
    cudaError_t e = buf.alloc((size_t)ws_bytes, stream);
    if (e) return from_cuda(e);
    char* base = static_cast<char*>(buf.ptr);
    int* err_flag = nullptr;
    if ((e = library_error_word(&err_flag))) return from_cuda(e);
    a.err = err_flag;
    if (cu_seqlens) {
        int64_t* chunk_off = reinterpret_cast<int64_t*>(base + 1024);
        int32_t* order = ordered ? reinterpret_cast<int32_t*>(chunk_off + B + 1) : nullptr;
        int64_t* seg_off = seg_table ? chunk_off + B + 1 : nullptr;
        if ((e = launch_chunk_offsets(cu_seqlens, B, T_total, si.chunks_upper, chunk_off, order,
                                      err_flag, plan.len, plan.upper, seg_off, stream)))
            return from_cuda(e);
        si.chunk_off = chunk_off;
        si.order = order;
        plan.seg_off = seg_off;
    }
    unsigned char* ws = reinterpret_cast<unsigned char*>(base + 1024 + off_bytes);
    // header words: 64, the fused kernel's chain tickets (packed sequences); 65, the
    // two-kernel form's decay-range flag
    int* ticket = cu_seqlens ? reinterpret_cast<int*>(base) + 64 : nullptr;
    if (use_fused) {
        e = run_prefill_fused(a, err_flag, ticket, nullptr, stream);
    } else if (guarded) {
        a.range_flag = reinterpret_cast<int*>(base) + 65;
        e = cudaMemsetAsync(a.range_flag, 0, sizeof(int), stream);
        if (!e) e = run_prefill_tc(a, ws, Hg, err_flag, stream);
        if (!e) e = run_prefill_fused(a, err_flag, ticket, a.range_flag, stream);
    } else if (use_tc) {
        e = run_prefill_tc(a, ws, Hg, err_flag, stream);
    } else if (!segmap) {
        e = run_prefill_simt(a, reinterpret_cast<float*>(ws), Hg, stream);
    } else {
        // B: the final states from zero; M: from the identity with zero values
        char* ex = reinterpret_cast<char*>(
            (reinterpret_cast<uintptr_t>(ws) + Hg * per_head + 1023) & ~uintptr_t(1023));
        void* v0 = ex + ex_v0;
        void* scratch = ex + ex_out;
        float* eye = reinterpret_cast<float*>(ex + ex_eye);
        PrefillArgs b = a;
        b.out = scratch; b.h0 = nullptr; b.hT = offs;
        e = run_prefill_simt(b, reinterpret_cast<float*>(ws), Hg, stream);
        if (!e) e = cudaMemsetAsync(v0, 0, (size_t)(T_total * H * dk * es), stream);
        if (!e) e = launch_fill_identity(eye, B * H, (int)dk, stream);
        if (!e) {
            PrefillArgs m = a;
            m.v = v0; m.dv = (int)dk; m.out = scratch; m.h0 = eye; m.hT = maps;
            e = run_prefill_simt(m, reinterpret_cast<float*>(ws), Hg, stream);
        }
    }
    if (e) return from_cuda(e);
    if (debug_mode()) {
        int flag = 0;
        if ((e = take_error_word(stream, &flag))) return from_cuda(e);
        return status_from_error_bits(flag);
    }
    return KDA_OK;
}

}  // namespace kda

extern "C" {

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* h0, void* out, float* hT,
                           const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                           int64_t dk, int64_t dv, float scale, kda_io_dtype_t io_dtype,
                           cudaStream_t stream)
{
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, h0, out, hT, cu_seqlens, B, T, H, dk, dv,
                            scale, io_dtype, KDA_PREFILL_AUTO, stream);
}

}  // extern "C"

extern "C" {

kda_status_t kda_chunk_fwd_segmap(const void* q, const void* k, const void* v,
                                  const float* log_alpha, const float* beta, float* maps,
                                  float* offs, const int32_t* cu_seqlens, int64_t B, int64_t T,
                                  int64_t H, int64_t dk, int64_t dv, kda_io_dtype_t io_dtype,
                                  cudaStream_t stream)
{
    if (maps == nullptr || offs == nullptr) return KDA_ERR_INVALID_ARG;
    if (B < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (B > 0 && H > 0 && (cu_seqlens ? T : B * T) == 0) {
        // no tokens: M = I, B = 0 for every sequence
        if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
        if (!aligned16(maps) || !aligned16(offs)) return KDA_ERR_INVALID_ARG;
        cudaError_t e = cudaMemsetAsync(offs, 0, (size_t)(B * H * dk * dv * 4), stream);
        if (!e) e = launch_fill_identity(maps, B * H, (int)dk, stream);
        return from_cuda(e);
    }
    return chunk_fwd_impl(q, k, v, log_alpha, beta, nullptr, nullptr, nullptr, nullptr, 0,
                          cu_seqlens, B, T, H, dk, dv, 1.f, io_dtype, KDA_PREFILL_AUTO, false,
                          stream, maps, offs);
}

kda_status_t kda_affine_prefix(const float* maps, const float* offs, const float* h0,
                               float* out, int64_t nseg, int64_t NH, int64_t dk, int64_t dv,
                               cudaStream_t stream)
{
    if (nseg < 0 || NH < 0) return KDA_ERR_INVALID_ARG;
    if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (NH == 0) return KDA_OK;
    if (NH > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (out == nullptr || !aligned16(out)) return KDA_ERR_INVALID_ARG;
    if (h0 && !aligned16(h0)) return KDA_ERR_INVALID_ARG;
    if (nseg > 0) {
        if (maps == nullptr || offs == nullptr || !aligned16(maps) || !aligned16(offs))
            return KDA_ERR_INVALID_ARG;
        if ((const void*)maps == (const void*)out || (const void*)offs == (const void*)out)
            return KDA_ERR_INVALID_ARG;
    }
    PrefixArgs p;
    std::memset(&p, 0, sizeof(p));
    p.maps = maps; p.offs = offs; p.h0 = h0; p.starts = nullptr; p.out = out;
    p.seg_off = nullptr; p.nseg = nseg; p.N = 1; p.H = NH; p.h_base = 0; p.hg = NH;
    p.hstride = NH; p.abs_head = true; p.slots = nullptr; p.P = 0;
    p.dk = (int)dk; p.dv = (int)dv; p.err = nullptr;
    return from_cuda(launch_affine_prefix(p, stream));
}

}  // extern "C"

namespace kda {

static kda_status_t chunk_bwd_impl(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta, const float* h0,
                                   const void* dout, const float* dhT, void* dq, void* dk, void* dv,
                                   float* dlog_alpha, float* dbeta, float* dh0,
                                   const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                                   int64_t dk_, int64_t dv_, float scale, kda_io_dtype_t io_dtype,
                                   bool gate_scalar, cudaStream_t stream)
{
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_INVALID_ARG;
    if (io_dtype != KDA_IO_F32 && io_dtype != KDA_IO_BF16) return KDA_ERR_UNSUPPORTED;
    if (!head_ok(dk_) || !head_ok(dv_)) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens != nullptr && B < 1) return KDA_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return KDA_OK;
    const int64_t T_total = cu_seqlens ? T : B * T;
    if (T_total > 0) {
        const void* ptrs[] = {q, k, v, dout, dq, dk, dv};
        for (const void* p : ptrs)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
        const void* gates[] = {log_alpha, dlog_alpha};
        for (const void* p : gates)
            if (p == nullptr || !(gate_scalar ? aligned4(p) : aligned16(p))) return KDA_ERR_INVALID_ARG;
        if (beta == nullptr || !aligned4(beta) || dbeta == nullptr || !aligned4(dbeta))
            return KDA_ERR_INVALID_ARG;
        // outputs must not alias inputs (or one another)
        const void* outs[] = {dq, dk, dv, dlog_alpha, dbeta};
        const void* ins[] = {q, k, v, log_alpha, beta, dout};
        for (const void* o : outs)
            for (const void* i : ins)
                if (o == i) return KDA_ERR_INVALID_ARG;
        for (int a = 0; a < 5; ++a)
            for (int c = a + 1; c < 5; ++c)
                if (outs[a] == outs[c]) return KDA_ERR_INVALID_ARG;
    }
    if ((h0 && !aligned16(h0)) || (dhT && !aligned16(dhT)) || (dh0 && !aligned16(dh0)))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && !aligned4(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (T_total > (int64_t(1) << 40) || H > 65535) return KDA_ERR_UNSUPPORTED;
    if (B * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;

    BackwardArgs b;
    std::memset(&b, 0, sizeof(b));
    b.q = q; b.k = k; b.v = v; b.log_alpha = log_alpha; b.beta = beta; b.h0 = h0;
    b.dout = dout; b.dhT = dhT; b.dq = dq; b.dk = dk; b.dv = dv; b.dlog_alpha = dlog_alpha;
    b.dbeta = dbeta; b.dh0 = dh0; b.H = H; b.dk_ = (int)dk_; b.dv_ = (int)dv_; b.scale = scale;
    b.io = io_dtype;
    b.gate_scalar = gate_scalar;
    SeqInfo& si = b.si;
    si.cu = cu_seqlens;
    si.chunk_off = nullptr;
    si.N = B;
    si.T_seq = cu_seqlens ? 0 : T;
    si.T_total = T_total;
    si.nct = cu_seqlens ? 0 : (T + kChunk - 1) / kChunk;
    si.chunks_upper = cu_seqlens ? (T / kChunk + B) : B * si.nct;
    si.order = nullptr;

    // workspace: [1 KiB header (reserved) | chunk offsets | per-(chunk, head) backward blocks]
    const int64_t off_bytes = cu_seqlens ? ((B + 1) * 8 + 1023) / 1024 * 1024 : 0;
    const int64_t per_head = bwd_ws_floats_per_chunk((int)dk_, (int)dv_) * (int64_t)sizeof(float) *
                             (si.chunks_upper > 0 ? si.chunks_upper : 1);
    int64_t Hg = (workspace_budget() - 1024 - off_bytes) / per_head;
    if (Hg < 1) Hg = 1;
    if (Hg > H) Hg = H;
    StreamBuffer buf;
    cudaError_t e = buf.alloc((size_t)(1024 + off_bytes + Hg * per_head), stream);
    if (e) return from_cuda(e);
    char* base = static_cast<char*>(buf.ptr);
    int* err_flag = nullptr;
    if ((e = library_error_word(&err_flag))) return from_cuda(e);
    if (cu_seqlens) {
        int64_t* chunk_off = reinterpret_cast<int64_t*>(base + 1024);
        if ((e = launch_chunk_offsets(cu_seqlens, B, T_total, si.chunks_upper, chunk_off, nullptr,
                                      err_flag, 0, 0, nullptr, stream)))
            return from_cuda(e);
        si.chunk_off = chunk_off;
    }
    e = run_backward_simt(b, reinterpret_cast<float*>(base + 1024 + off_bytes), Hg, stream);
    if (e) return from_cuda(e);
    if (debug_mode()) {
        int flag = 0;
        if ((e = take_error_word(stream, &flag))) return from_cuda(e);
        return status_from_error_bits(flag);
    }
    return KDA_OK;
}

}  // namespace kda

extern "C" {

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* h0, const void* dout, const float* dhT,
                           void* dq, void* dk, void* dv, float* dlog_alpha, float* dbeta,
                           float* dh0, const int32_t* cu_seqlens, int64_t B, int64_t T, int64_t H,
                           int64_t dk_, int64_t dv_, float scale, kda_io_dtype_t io_dtype,
                           cudaStream_t stream)
{
    return chunk_bwd_impl(q, k, v, log_alpha, beta, h0, dout, dhT, dq, dk, dv, dlog_alpha, dbeta,
                          dh0, cu_seqlens, B, T, H, dk_, dv_, scale, io_dtype, false, stream);
}

kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* log_a,
                               const float* beta, const float* h0, const void* dout,
                               const float* dhT, void* dq, void* dk, void* dv, float* dlog_a,
                               float* dbeta, float* dh0, const int32_t* cu_seqlens, int64_t B,
                               int64_t T, int64_t H, int64_t dk_, int64_t dv_, float scale,
                               kda_io_dtype_t io_dtype, cudaStream_t stream)
{
    return chunk_bwd_impl(q, k, v, log_a, beta, h0, dout, dhT, dq, dk, dv, dlog_a, dbeta, dh0,
                          cu_seqlens, B, T, H, dk_, dv_, scale, io_dtype, true, stream);
}

}  // extern "C"

extern "C" {

kda_status_t kda_debug_prep_image(const void* q, const void* k, const float* log_alpha,
                                  const float* beta, void* image, int64_t B, int64_t T, int64_t H,
                                  int gate_scalar, cudaStream_t stream)
{
    if (B < 0 || T < 0 || H < 0 || H > 65535) return KDA_ERR_INVALID_ARG;
    if (B * T >= (int64_t(1) << 31)) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0 || H == 0) return KDA_OK;
    const void* ptrs[] = {q, k, image};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (log_alpha == nullptr || !(gate_scalar ? aligned4(log_alpha) : aligned16(log_alpha)))
        return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = k;                 // v is not read by the prep
    a.log_alpha = log_alpha; a.beta = beta; a.H = H; a.dk = 128; a.dv = 128;
    a.scale = 1.f; a.io = KDA_IO_BF16; a.gate_scalar = gate_scalar != 0; a.tc_what = 2;
    SeqInfo& si = a.si;
    si.N = B;
    si.T_seq = T;
    si.T_total = B * T;
    si.nct = (T + kChunk - 1) / kChunk;
    si.chunks_upper = B * si.nct;
    return from_cuda(run_prefill_tc(a, static_cast<unsigned char*>(image), H, nullptr, stream));
}

}  // extern "C"
