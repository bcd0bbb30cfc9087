// libkda C-ABI: argument checking, workspace sizing and dispatch to the kernels.
// Everything here is host code; the kernels live in the included .cuh files so the
// whole library is one translation unit (one device status word, no relocatable code).
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "libkda.h"
#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_prefill_simt.cuh"
#include "kda_prefill_tc.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int32_t dk, int32_t dv) { return dk == dv && (dk == 64 || dk == 128); }

// bf16 runs on the tensor cores (d = 64 as the first 64 channels of a 128-channel problem);
// fp32 on CUDA cores.
bool tensor_core_path(kda_dtype dt, int32_t dk) { return dt == KDA_BF16 && (dk == 128 || dk == 64); }

bool valid_chunk(kda_dtype dt, int32_t C) {
    if (dt == KDA_BF16) return C == 64;
    return C == 16 || C == 32 || C == 64;
}

template <typename T>
cudaError_t dispatch_simt(int32_t dk, int32_t C, const void* q, const void* k, const void* v,
                          const float* g, const float* beta, const float* s0, const int32_t* cu,
                          int num_seqs, int64_t total, int H, void* out, float* sf,
                          cudaStream_t st, uint32_t in_flags) {
#define KDA_SIMT_CASE(D, CC)                                                                  \
    if (dk == D && C == CC)                                                                   \
        return kda::launch_prefill_simt<T, D, CC>(q, k, v, g, beta, s0, cu, num_seqs, total, H, \
                                                  out, sf, st, in_flags);
    KDA_SIMT_CASE(64, 16) KDA_SIMT_CASE(64, 32) KDA_SIMT_CASE(64, 64)
    KDA_SIMT_CASE(128, 16) KDA_SIMT_CASE(128, 32) KDA_SIMT_CASE(128, 64)
#undef KDA_SIMT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

extern "C" {

int32_t kda_abi_version(void) { return 8; }

const char* kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported problem size or chunk size";
        case KDA_ERR_CUDA: return "CUDA runtime error";
        case KDA_ERR_TIMEOUT: return "a bounded device wait expired";
        case KDA_ERR_BAD_SEQLENS: return "cu_seqlens inconsistent with total_tokens";
        case KDA_ERR_BAD_EMIT_POS: return "an emission position is not a chunk boundary of a sequence";
    }
    return "unknown status";
}

size_t kda_prefill_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                                  int32_t dv, int32_t C, kda_dtype dt) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || !supported_dim(dk, dv) ||
        !valid_chunk(dt, C))
        return 0;
    if (!tensor_core_path(dt, dk)) return 0;
    size_t bytes = 0;
    return kda::tc::workspace_bytes_checked(total_tokens, num_seqs, H, &bytes) ? bytes : 0;
}

size_t kda_prefill_workspace_size_min(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                                      int32_t dv, int32_t C, kda_dtype dt) {
    if (kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv, C, dt) == 0) return 0;
    return kda::tc::workspace_bytes_min(total_tokens, num_seqs, H);
}

int64_t kda_prefill_windows(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk, int32_t dv,
                            int32_t C, kda_dtype dt, size_t ws_bytes) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || !supported_dim(dk, dv) || !valid_chunk(dt, C))
        return -1;
    if (!tensor_core_path(dt, dk) || num_seqs == 0) return 1;
    if (kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv, C, dt) == 0) return -1;
    const int64_t w = kda::tc::window_chunks(total_tokens, num_seqs, H, ws_bytes);
    if (w <= 0) return -1;
    const int64_t mc = kda::tc::max_chunks(total_tokens, num_seqs);
    return w >= mc ? 1 : (mc + w - 1) / w;
}

int32_t kda_prefill_launches(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                             int32_t dv, int32_t C, kda_dtype dt, uint32_t in_flags, int32_t num_emit) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || !supported_dim(dk, dv) || !valid_chunk(dt, C))
        return -1;
    if (num_seqs == 0) return 0;
    if (!tensor_core_path(dt, dk)) return 1;
    // chunk table, [recurrence order of several sequences], [emission slots], preparation,
    // strongly decayed chunks, recurrence
    int32_t n = 1 + (num_seqs > 1 ? 1 : 0) + (num_emit > 0 ? 1 : 0) + (total_tokens > 0 ? 2 : 0) + 1;
    if (!(in_flags & KDA_IN_SERIAL_CHAINS) && kda::tc::scan_segment_chunks(total_tokens, num_seqs, H) > 0)
        n += 3;   // segment table, segment transitions, starting states
    return n;
}

// A tensor-core problem whose workspace or launch grids cannot be addressed (see
// workspace_bytes_checked) is rejected before anything is launched.
static bool tc_problem_fits(int64_t total_tokens, int32_t num_seqs, int32_t H) {
    size_t bytes = 0;
    return kda::tc::workspace_bytes_checked(total_tokens, num_seqs, H, &bytes);
}

static kda_status prefill_common(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, const float* initial_state,
                                 const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                 int32_t H, int32_t dk, int32_t dv, kda_dtype dt, void* out,
                                 float* final_state, int32_t C, const int64_t* emit_pos,
                                 int32_t num_emit, float* emit_states, void* workspace,
                                 size_t ws_bytes, kda_stream_t stream, uint32_t in_flags) {
    if (num_seqs < 0 || total_tokens < 0 || H <= 0 || dk <= 0 || dv <= 0 || num_emit < 0)
        return KDA_ERR_INVALID_ARG;
    if (in_flags & ~(uint32_t)(KDA_IN_NORMALIZE_QK | KDA_IN_G_LOGITS | KDA_IN_BETA_LOGITS |
                               KDA_IN_G_SCALAR | KDA_IN_STRONG_DECAY | KDA_IN_SERIAL_CHAINS))
        return KDA_ERR_INVALID_ARG;
    if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return KDA_ERR_UNSUPPORTED;  // cu_seqlens is int32
    if (!supported_dim(dk, dv) || !valid_chunk(dt, C)) return KDA_ERR_UNSUPPORTED;
    if (num_emit > 0) {
        if (!emit_pos || !emit_states || (reinterpret_cast<uintptr_t>(emit_pos) & 7u) != 0 ||
            !aligned16(emit_states) || num_seqs == 0)
            return KDA_ERR_INVALID_ARG;
        if (!tensor_core_path(dt, dk)) return KDA_ERR_UNSUPPORTED;
    }
    if (tensor_core_path(dt, dk) && !tc_problem_fits(total_tokens, num_seqs, H)) return KDA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return KDA_OK;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, out, initial_state, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return KDA_ERR_INVALID_ARG;
    // A workspace below the full size runs the chunks in windows (window_chunks), down to
    // kda_prefill_workspace_size_min.
    const size_t need = kda_prefill_workspace_size_min(total_tokens, num_seqs, H, dk, dv, C, dt);
    if (ws_bytes < need || (need > 0 && (!workspace ||
                                         (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)))
        return KDA_ERR_INVALID_ARG;
    int64_t window = INT64_MAX;
    if (tensor_core_path(dt, dk) && need > 0) {
        window = kda::tc::window_chunks(total_tokens, num_seqs, H, ws_bytes);
        if (window <= 0) return KDA_ERR_INVALID_ARG;
    }

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (tensor_core_path(dt, dk))
        err = kda::tc::launch_prefill(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs,
                                      total_tokens, H, out, final_state, workspace, st, emit_pos,
                                      num_emit, emit_states, in_flags, window, dk);
    else if (dt == KDA_F32)
        err = dispatch_simt<float>(dk, C, q, k, v, g, beta, initial_state, cu_seqlens, num_seqs,
                                   total_tokens, H, out, final_state, st, in_flags);
    else
        return KDA_ERR_UNSUPPORTED;   // unreachable: every bf16 problem takes the tensor cores
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_prefill(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                       kda_dtype dt, void* out, float* final_state, int32_t C, void* workspace,
                       size_t ws_bytes, kda_stream_t stream) {
    return prefill_common(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, H, dk,
                          dv, dt, out, final_state, C, nullptr, 0, nullptr, workspace, ws_bytes, stream,
                          0u);
}

kda_status kda_prefill_gdn(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                           int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                           kda_dtype dt, void* out, float* final_state, int32_t C, void* workspace,
                           size_t ws_bytes, kda_stream_t stream) {
    return prefill_common(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, H, dk,
                          dv, dt, out, final_state, C, nullptr, 0, nullptr, workspace, ws_bytes, stream,
                          (uint32_t)KDA_IN_G_SCALAR);
}

kda_status kda_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                          int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                          kda_dtype dt, void* out, float* final_state, int32_t C, uint32_t in_flags,
                          const int64_t* emit_pos, int32_t num_emit, float* emit_states,
                          void* workspace, size_t ws_bytes, kda_stream_t stream) {
    return prefill_common(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, H, dk,
                          dv, dt, out, final_state, C, emit_pos, num_emit, emit_states, workspace,
                          ws_bytes, stream, in_flags);
}

kda_status kda_prefill_emit(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, const float* initial_state,
                            const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                            int32_t H, int32_t dk, int32_t dv, kda_dtype dt, void* out,
                            float* final_state, int32_t C, const int64_t* emit_pos,
                            int32_t num_emit, float* emit_states, void* workspace,
                            size_t ws_bytes, kda_stream_t stream) {
    return prefill_common(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, H, dk,
                          dv, dt, out, final_state, C, emit_pos, num_emit, emit_states, workspace,
                          ws_bytes, stream, 0u);
}

// Checks shared by the staged tensor-core entry points.
static kda_status check_staged(const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                               int32_t H, int32_t dk, int32_t dv, kda_dtype dt, int32_t C,
                               const void* workspace, size_t ws_bytes) {
    if (num_seqs < 0 || total_tokens < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (!tensor_core_path(dt, dk) || !supported_dim(dk, dv) || !valid_chunk(dt, C))
        return KDA_ERR_UNSUPPORTED;
    if (!tc_problem_fits(total_tokens, num_seqs, H)) return KDA_ERR_UNSUPPORTED;
    if (num_seqs > 0 && (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0))
        return KDA_ERR_INVALID_ARG;
    const size_t need = kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv, C, dt);
    if (ws_bytes < need || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

kda_status kda_prefill_prepare(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const int32_t* cu_seqlens, int32_t num_seqs,
                               int64_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                               kda_dtype dt, int32_t C, void* workspace, size_t ws_bytes,
                               kda_stream_t stream) {
    kda_status st = check_staged(cu_seqlens, num_seqs, total_tokens, H, dk, dv, dt, C, workspace, ws_bytes);
    if (st != KDA_OK || num_seqs == 0) return st;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    return kda::tc::launch_prepare(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, H, workspace,
                                   reinterpret_cast<cudaStream_t>(stream), nullptr, 0, 0u, dk) == cudaSuccess
               ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_prefill_scan(const float* initial_state, float* final_state, void* out,
                            const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                            int32_t H, int32_t dk, int32_t dv, kda_dtype dt, int32_t C,
                            void* workspace, size_t ws_bytes, kda_stream_t stream) {
    kda_status st = check_staged(cu_seqlens, num_seqs, total_tokens, H, dk, dv, dt, C, workspace, ws_bytes);
    if (st != KDA_OK || num_seqs == 0) return st;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!out || !aligned16(out))) return KDA_ERR_INVALID_ARG;
    return kda::tc::launch_scan(initial_state, final_state, out, num_seqs, total_tokens, H,
                                workspace, reinterpret_cast<cudaStream_t>(stream), nullptr, 0u, dk) == cudaSuccess
               ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_selftest_bounded_wait(uint64_t limit_ns, kda_stream_t stream) {
    if (limit_ns < 1000ull || limit_ns > 2000000000ull) return KDA_ERR_INVALID_ARG;
    kda::tc::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

static kda_status decode_common(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* state_inout, void* out, int32_t N, int32_t H,
                                int32_t dk, int32_t dv, kda_dtype dt, kda_stream_t stream, uint32_t in_flags) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (in_flags & ~(uint32_t)(KDA_IN_NORMALIZE_QK | KDA_IN_G_LOGITS | KDA_IN_BETA_LOGITS |
                               KDA_IN_G_SCALAR | KDA_IN_STRONG_DECAY | KDA_IN_SERIAL_CHAINS))
        return KDA_ERR_INVALID_ARG;
    in_flags &= ~(uint32_t)(KDA_IN_STRONG_DECAY | KDA_IN_SERIAL_CHAINS);   // no effect on one token
    if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if ((int64_t)N * H > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !state_inout || !out) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, state_inout, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (dt == KDA_F32)
        err = dk == 64 ? kda::launch_decode<64, float>(q, k, v, g, beta, state_inout, out, N, H, st, in_flags)
                       : kda::launch_decode<128, float>(q, k, v, g, beta, state_inout, out, N, H, st, in_flags);
    else
        err = dk == 64 ? kda::launch_decode<64, __nv_bfloat16>(q, k, v, g, beta, state_inout, out, N, H, st,
                                                               in_flags)
                       : kda::launch_decode<128, __nv_bfloat16>(q, k, v, g, beta, state_inout, out, N, H,
                                                                st, in_flags);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* state_inout, void* out, int32_t N, int32_t H,
                      int32_t dk, int32_t dv, kda_dtype dt, kda_stream_t stream) {
    return decode_common(q, k, v, g, beta, state_inout, out, N, H, dk, dv, dt, stream, 0u);
}

kda_status kda_decode_gdn(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state_inout, void* out, int32_t N, int32_t H,
                          int32_t dk, int32_t dv, kda_dtype dt, kda_stream_t stream) {
    return decode_common(q, k, v, g, beta, state_inout, out, N, H, dk, dv, dt, stream,
                         (uint32_t)KDA_IN_G_SCALAR);
}

kda_status kda_decode_ex(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, float* state_inout, void* out, int32_t N, int32_t H,
                         int32_t dk, int32_t dv, kda_dtype dt, uint32_t in_flags, kda_stream_t stream) {
    return decode_common(q, k, v, g, beta, state_inout, out, N, H, dk, dv, dt, stream, in_flags);
}

#ifdef KDA_TRACE
// Trace builds only: copy the first n clock stamps to host memory.
int kda_debug_read_trace(unsigned long long* host, int n) {
    if (n > kTraceSlots) n = kTraceSlots;
    return cudaMemcpyFromSymbol(host, g_kda_trace, sizeof(unsigned long long) * n) == cudaSuccess ? n : -1;
}
#endif

kda_status kda_get_device_status(kda_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_kda_status, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_kda_status, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    }
    return static_cast<kda_status>(v);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Allocation-free prefill: the tensor-core prefill with its workspace taken from a static
// device array inside this library instead of from the caller (for callers that cannot
// allocate device memory where they run).  Every GPU that loads the library holds the
// array until the process exits; all calls on a device share it.
static __device__ __align__(256) uint8_t g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry point (no link against libcuda).
CtxGetCurrentFn ctx_get_current() {
    static const CtxGetCurrentFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<CtxGetCurrentFn>(p);
        return static_cast<CtxGetCurrentFn>(nullptr);
    }();
    return fn;
}

// Last looked-up scratch address per CUDA context.  The array's name is only a host-side
// stand-in; the kernels must get the device address, which belongs to the context that
// loaded the module: a new primary context after cudaDeviceReset, or another context made
// current, has its own.
struct ScratchEntry {
    CUcontext ctx;
    void* ptr;
};
constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mutex;
ScratchEntry g_noalloc_cache[kMaxContexts] = {};

// Device address of the scratch array in the current context.  Outside stream capture the
// address is looked up on every call (cudaGetSymbolAddress, a host-side query once the
// module is loaded) and the cache refreshed; while `stream` is capturing only the cache
// of this context is used, so the first call in a context must come before any capture.
cudaError_t noalloc_scratch(cudaStream_t stream, void** ptr) {
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return cudaErrorNotSupported;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t err = cudaStreamIsCapturing(stream, &cap);
    if (err != cudaSuccess) return err;
    void* p = nullptr;
    if (cap == cudaStreamCaptureStatusNone) {
        // also makes the device's primary context current if nothing was yet
        err = cudaGetSymbolAddress(&p, g_kda_noalloc_scratch);
        if (err != cudaSuccess) return err;
    }
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    int slot = -1;
    for (int i = 0; i < kMaxContexts; ++i)
        if (g_noalloc_cache[i].ctx == ctx) { slot = i; break; }
    if (cap != cudaStreamCaptureStatusNone) {
        if (slot < 0) return cudaErrorStreamCaptureUnsupported;
        *ptr = g_noalloc_cache[slot].ptr;
        return cudaSuccess;
    }
    if (slot < 0) {
        for (int i = 0; i < kMaxContexts && slot < 0; ++i)
            if (g_noalloc_cache[i].ctx == nullptr) slot = i;
        if (slot < 0) slot = 0;   // table full: reuse the first entry
    }
    g_noalloc_cache[slot] = {ctx, p};
    *ptr = p;
    return cudaSuccess;
}
}  // namespace

extern "C" kda_status kda_prefill_noalloc(const void* q, const void* k, const void* v,
                                          const float* g, const float* beta,
                                          const float* initial_state, const int32_t* cu_seqlens,
                                          int32_t num_seqs, int64_t total_tokens, int32_t H,
                                          int32_t dk, int32_t dv, kda_dtype dt, void* out,
                                          float* final_state, int32_t C, kda_stream_t stream) {
    if (num_seqs < 0 || total_tokens < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_BF16 || !tensor_core_path(dt, dk) || dv != dk || C != 64) return KDA_ERR_UNSUPPORTED;
    if (total_tokens > INT32_MAX || !tc_problem_fits(total_tokens, num_seqs, H)) return KDA_ERR_UNSUPPORTED;
    const size_t need = kda_prefill_workspace_size_min(total_tokens, num_seqs, H, dk, dv, C, dt);
    if (need == 0 || need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return KDA_OK;
    void* scratch = nullptr;
    if (noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch) != cudaSuccess)
        return KDA_ERR_CUDA;
    return kda_prefill(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, H,
                       dk, dv, dt, out, final_state, C, scratch, KDA_NOALLOC_SCRATCH_BYTES, stream);
}
