// Internal declarations shared by the KDA library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "kda.h"

namespace kda {

// Where the tokens of each sequence live, and how chunks are numbered.
// Chunks are numbered sequence after sequence: sequence n owns global chunks
// [chunk_start(n), chunk_start(n+1)).  Without cu_seqlens every sequence has
// T_seq tokens and nct = ceil(T_seq / 64) chunks; with cu_seqlens the
// per-sequence chunk offsets are computed on the device (chunk_off, N+1
// entries) from the clamped offsets.
struct SeqInfo {
    const int32_t* cu;          // device, N+1 entries, or nullptr
    const int64_t* chunk_off;   // device, N+1 entries (only with cu)
    int64_t N;                  // number of sequences
    int64_t T_seq;              // tokens per sequence (fixed-length case)
    int64_t T_total;            // packed token count (B*T, or T with cu)
    int64_t nct;                // chunks per sequence (fixed-length case)
    int64_t chunks_upper;       // upper bound on the number of chunks (grid size)
    const int32_t* order;       // device, N entries: sequences longest first, or nullptr

#ifdef __CUDACC__
    // Sequence handled by the r-th sequential chain: the longest sequences
    // first when an order is known, so their chains start in the first wave.
    __device__ __forceinline__ int64_t seq_of(int64_t r) const {
        return order ? (int64_t)order[r] : r;
    }
    __device__ __forceinline__ int64_t chunk_start(int64_t n) const {
        return cu ? chunk_off[n] : n * nct;
    }
    // Chunks of sequence n that have workspace slots: ceil(len/64), capped by
    // the (capped) device offsets when cu_seqlens is malformed.
    __device__ __forceinline__ int64_t chunk_count(int64_t n, int64_t len) const {
        const int64_t c = (len + 63) / 64;
        if (!cu) return c;
        const int64_t slots = chunk_off[n + 1] - chunk_off[n];
        return c < slots ? c : slots;
    }
    // Map a global chunk index to (sequence, first token, length); false when
    // the index is past the last chunk.
    __device__ __forceinline__ bool locate(int64_t gc, int64_t& n, int64_t& t0,
                                           int64_t& len) const {
        if (cu == nullptr) {
            n = gc / nct;
            if (n >= N) return false;
            const int64_t c = gc - n * nct;
            const int64_t bos = n * T_seq;
            t0 = bos + c * 64;
            len = bos + T_seq - t0;
            len = len > 64 ? 64 : len;
            return len > 0;
        }
        if (gc >= chunk_off[N]) return false;
        int64_t lo = 0, hi = N;                  // chunk_off[lo] <= gc < chunk_off[hi]
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (chunk_off[mid] <= gc) lo = mid; else hi = mid;
        }
        n = lo;
        int64_t a = cu[n], b = cu[n + 1];
        a = a < 0 ? 0 : (a > T_total ? T_total : a);
        b = b < a ? a : (b > T_total ? T_total : b);
        t0 = a + (gc - chunk_off[n]) * 64;
        len = b - t0;
        len = len > 64 ? 64 : len;
        return len > 0;
    }
#endif
};

// Segment-parallel walk of the state chains (tensor-core path).  The chunks of
// each sequence are cut into segments of `len` chunks.  A segment maps its
// entry state affinely, S -> M S + B, so each segment's M (walk from the
// identity with V = 0) and B (walk from zero) are computed independently, the
// entry states follow from a short sequential composition, and a last walk per
// segment writes the outputs.  Buffers hold one dk x dk (maps) or dk x dv
// (offs, starts) fp32 matrix per (segment, head), at (g * hstride + head) where
// head is the index within the head group (or the absolute head when
// abs_head is set).
struct SegPlan {
    int64_t len;              // chunks per segment; 0: segmentation off
    int64_t nseg;             // segments per sequence (fixed-length batches)
    int64_t upper;            // bound on the number of segments (grid, buffers)
    const int64_t* seg_off;   // device [N+1]: first segment of each sequence (packed), or nullptr
    float* maps;
    float* offs;
    float* starts;
    int64_t hstride;
    bool abs_head;
    // device word or nullptr: when it is nonzero at launch, the state walks do nothing
    // (the prep found a chunk outside the two-kernel form's decay range and the fused
    // kernel, launched after them, computes the whole call instead)
    const int* skip;

#ifdef __CUDACC__
    // Segment g -> (sequence n, index s within it, segments of n); false past the end.
    __device__ __forceinline__ bool locate(int64_t g, int64_t N, int64_t& n, int64_t& s,
                                           int64_t& count) const {
        if (seg_off == nullptr) {
            n = g / nseg;
            if (n >= N) return false;
            s = g - n * nseg;
            count = nseg;
            return true;
        }
        if (g >= seg_off[N]) return false;
        int64_t lo = 0, hi = N;                  // seg_off[lo] <= g < seg_off[hi]
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (seg_off[mid] <= g) lo = mid; else hi = mid;
        }
        n = lo;
        s = g - seg_off[n];
        count = seg_off[n + 1] - seg_off[n];
        return true;
    }
#endif
};

struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const float* h0;
    void* out;
    float* hT;
    SeqInfo si;
    int64_t H;
    int dk, dv;
    float scale;
    kda_io_dtype_t io;
    // pooled states: when `slots` is set, sequence n's initial and final states
    // live at index slots[n] of h0 / hT ([P, H, dk, dv]); a negative slot means
    // zero initial state and no final state; slots >= P are reported and skipped
    const int32_t* slots;
    int64_t P;
    int* err;
    // Gated DeltaNet form: one gate per (token, head), log_alpha [.., H],
    // broadcast over the key channels
    bool gate_scalar;
    // tensor-core path: segment-parallel state walk (len == 0: one chain per
    // (sequence, head)); the buffers are placed by run_prefill_tc
    SegPlan seg;
    // two-kernel tensor-core path: device word the prep sets (bit 0) when a 16-token
    // block of some channel decays by more than its exponent range allows, or nullptr
    int* range_flag;
    // what the tensor-core path produces: outputs and final states (0), only each
    // sequence's affine map into seg.maps / seg.offs (1), or only the operand images of
    // the prep kernel, left in the workspace (2; the test hook kda_debug_prep_image)
    int tc_what;

#ifdef __CUDACC__
    // Flat (slot, head) index of sequence n's state, or -1 when it has none.
    __device__ __forceinline__ int64_t state_index(int64_t n, int64_t h) const {
        if (!slots) return n * H + h;
        const int64_t sl = slots[n];
        if (sl < 0) return -1;
        if (sl >= P) {
            if (err) atomicOr(err, 1);
            return -1;
        }
        return sl * H + h;
    }
#endif
};

// Backward pass (chunkwise gradients), fp32 SIMT kernels.
struct BackwardArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const float* h0;          // nullable: zero initial state
    const void* dout;         // [.., H, dv] io dtype
    const float* dhT;         // nullable: zero gradient of the final state
    void* dq;                 // [.., H, dk] io dtype
    void* dk;
    void* dv;                 // [.., H, dv] io dtype
    float* dlog_alpha;        // [.., H, dk] ([.., H] with gate_scalar)
    float* dbeta;             // [.., H]
    float* dh0;               // nullable
    SeqInfo si;
    int64_t H;
    int dk_, dv_;
    float scale;
    kda_io_dtype_t io;
    // Gated DeltaNet: log_alpha [.., H] broadcast over the key channels; dlog_alpha [.., H]
    // receives the channel sum of the per-channel gradient
    bool gate_scalar;
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    float* state;
    void* out;
    int64_t N, H, P;
    int dk, dv;
    float scale;
    kda_io_dtype_t io;
    const int32_t* slots;    // nullptr: state index = n * H + h
    int* err;
    bool gate_scalar;        // log_alpha [N, H] (one gate per head) instead of [N, H, dk]
};

// Runs `f` (a per-device setup such as raising a kernel's shared-memory
// limit) once per device: the bit of the current device in `done` is set after
// the first success.  Devices past 63 run it every time.
// Streaming multiprocessors of the current device (queried once per device).
int64_t device_sm_count();

template <typename F>
inline cudaError_t once_per_device(std::atomic<uint64_t>& done, F f)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = f();
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Kernel identities for launch counting and timing (kda_profiler.cu).
enum KernelId {
    K_CHUNK_OFFSETS = 0,
    K_PREP_SIMT,
    K_STATE_SIMT,
    K_DECODE,
    K_PREP_TC,
    K_STATE_TC,
    K_STATE_SEG_TC,
    K_AFFINE_PREFIX,
    K_FILL,
    K_BWD_STATE,
    K_BWD_DENSE1,
    K_BWD_DENSE2,
    K_BWD_PARAM,
    K_FUSED_TC,
    K_KERNEL_COUNT
};

// Launch with programmatic stream serialization: the grid may start while the
// previous kernel on `st` drains (the kernel itself calls griddep_wait before it
// touches global memory).  Used for the launches of one prefill call, which
// follow each other back to back on one stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    const cudaError_t g = cudaGetLastError();   // clears the launch error it may have set
    return e != cudaSuccess ? e : g;
}

// Opened around every kernel launch: counts it and, while the profiler is
// enabled, records start/stop CUDA events on the launching stream.
class LaunchScope {
public:
    LaunchScope(cudaStream_t st, KernelId id);
    ~LaunchScope();
    LaunchScope(const LaunchScope&) = delete;
    LaunchScope& operator=(const LaunchScope&) = delete;

private:
    cudaStream_t st_;
    KernelId id_;
    void* start_ = nullptr;
    void* stop_ = nullptr;
};

// kda_decode.cu
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// kda_chunk_simt.cu
int64_t simt_ws_floats_per_chunk(int dk, int dv);
cudaError_t run_prefill_simt(const PrefillArgs& a, float* ws, int64_t Hg, cudaStream_t st);

// kda_chunk_bwd.cu
int64_t bwd_ws_floats_per_chunk(int dk, int dv);
cudaError_t run_backward_simt(const BackwardArgs& b, float* ws, int64_t Hg, cudaStream_t st);

// kda_chunk_tc.cu (bf16, dk = dv = 128)
int64_t tc_ws_bytes_per_chunk();
// Workspace bytes per head for the segment buffers of a plan.
int64_t tc_seg_bytes_per_head(const SegPlan& p);
cudaError_t run_prefill_tc(const PrefillArgs& a, unsigned char* ws, int64_t Hg, int* err,
                           cudaStream_t st);

// kda_fused_tc.cu (bf16, dk = dv = 128, T_total > 0): the whole prefill in one
// kernel.  `ticket` (device int, or null): the counter that hands out chains to
// CTAs as they free up (zeroed by the call); null keeps the static order.
// `run_if` (device int, or null): the kernel does nothing unless it is nonzero at launch.
cudaError_t run_prefill_fused(const PrefillArgs& a, int* err, int* ticket, const int* run_if,
                              cudaStream_t st);

// Device error word bits (workspace header): malformed cu_seqlens, and bounded
// waits that gave up in the tensor-core kernels (bit 1: input copies of the prep;
// 2, 3: its MMAs; 4: state-walk stage copies; 5: state-walk MMAs; 6: the state
// walk's worker/issuer hand-offs).
constexpr int kErrSeqlens = 1 << 0;
constexpr int kErrTimeoutMask = 0x7e;

// kda_errors.cu: the library's per-GPU device error word (the current device's),
// taking it (read and clear, ordered on `st`, waits for `st`), and the status its
// bits map to in debug mode.
cudaError_t library_error_word(int** out);
cudaError_t take_error_word(cudaStream_t st, int* host_out);
kda_status_t status_from_error_bits(int bits);
// KDA_DEBUG=1 in the environment (read once): every call waits for its stream and
// returns the status of the error bits it finds (kda_api.cu).
bool debug_mode_on();

// Self-test of the bounded mbarrier wait (kda_selftest.cu).
cudaError_t launch_bounded_wait_selftest(int* err, uint32_t polls, cudaStream_t st);

// kda_seqinfo.cu.  With seg_off set, also the first segment of each sequence
// for segments of seg_len chunks (at least one per sequence), capped at seg_cap.
cudaError_t launch_chunk_offsets(const int32_t* cu, int64_t N, int64_t T_total, int64_t cap,
                                 int64_t* chunk_off, int32_t* order, int* err_flag,
                                 int64_t seg_len, int64_t seg_cap, int64_t* seg_off,
                                 cudaStream_t st);

// kda_segscan.cu.  Entry states of consecutive segments: for every chain
// (sequence n, head h of the group h_base .. h_base + hg - 1) with segments
// s = 0 .. count-1 (count from seg_off, else nseg), X_0 = h0 (or zero),
// X_{s+1} = M_s X_s + B_s.  starts (nullable) receives every X_s, out
// (nullable) the state after the last segment at the chain's state index.
struct PrefixArgs {
    const float* maps;       // [(base(n) + s) * hstride + head][dk][dk]
    const float* offs;       // [(base(n) + s) * hstride + head][dk][dv]
    const float* h0;         // nullable; at the chain's state index
    float* starts;           // nullable; indexed like offs
    float* out;              // nullable; at the chain's state index
    const int64_t* seg_off;  // nullable: nseg segments per sequence
    int64_t nseg, N, H, h_base, hg, hstride;
    bool abs_head;           // buffer head index = h (else h - h_base)
    const int32_t* slots;    // pooled states, as in PrefillArgs
    int64_t P;
    int dk, dv;
    int* err;
};
cudaError_t launch_affine_prefix(const PrefixArgs& p, cudaStream_t st);
// count consecutive d x d identity matrices at dst.
cudaError_t launch_fill_identity(float* dst, int64_t count, int d, cudaStream_t st);
// Sequences are ranked by length (for `order`) when there are at most this many.
constexpr int64_t kMaxOrderedSeqs = 2048;

}  // namespace kda
