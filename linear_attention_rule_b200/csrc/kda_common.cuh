// Shared device helpers for the libkda kernels (one translation unit: libkda.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "libkda.h"

// First error a kernel detected since the host last read it (kda_get_device_status).
__device__ int g_kda_status;

__device__ __forceinline__ void kda_set_status(int s) { atomicCAS(&g_kda_status, 0, s); }

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization
// may start before the kernel ahead of it in the stream has finished: it waits for that
// kernel's completion (and its memory) at kda_grid_wait, before its first access to anything
// that kernel writes or reads.  Every kernel of such a chain waits on every path, so each
// one completing implies that all before it have completed.  Without the attribute both
// calls do nothing.
__device__ __forceinline__ void kda_grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel of the stream be scheduled (its blocks wait at kda_grid_wait).
__device__ __forceinline__ void kda_grid_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Input prologue (the layer's elementwise steps in front of KDA, fused into the kernels):
// bit flags as in include/libkda.h (KDA_IN_*).
constexpr uint32_t kInNormQK = 1u, kInGLogits = 2u, kInBetaLogits = 4u, kInGScalar = 8u,
                   kInStrongDecay = 16u, kInSerialChains = 32u;
// log(sigmoid(x)) = min(x, 0) - log(1 + e^{-|x|}), without overflow for either sign
__device__ __forceinline__ float kda_logsigmoid(float x) { return fminf(x, 0.f) - log1pf(__expf(-fabsf(x))); }
__device__ __forceinline__ float kda_sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }
// 1 / max(||x||, 1e-12) from the squared norm (the clamp of torch's F.normalize)
__device__ __forceinline__ float kda_inv_norm(float sumsq) { return rsqrtf(fmaxf(sumsq, 1e-24f)); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Checks the part of cu_seqlens that sequence n depends on; records KDA_ERR_BAD_SEQLENS
// and returns false when it is inconsistent.
__device__ __forceinline__ bool kda_seq_bounds(const int32_t* cu, int n, int num_seqs,
                                               int64_t total, int64_t& t_begin, int64_t& t_end) {
    t_begin = cu[n];
    t_end = cu[n + 1];
    bool ok = t_begin >= 0 && t_end >= t_begin && t_end <= total;
    if (n == 0) ok = ok && t_begin == 0;
    if (n == num_seqs - 1) ok = ok && t_end == total;
    if (!ok) kda_set_status(KDA_ERR_BAD_SEQLENS);
    return ok;
}

// Optional phase tracing (compile with -DKDA_TRACE): SM clock stamps of chosen points of
// chosen CTAs, read back with kda_debug_read_trace.  Compiled out by default.
#ifdef KDA_TRACE
constexpr int kTraceSlots = 1 << 16;
__device__ unsigned long long g_kda_trace[kTraceSlots];
#define KDA_TRACE_POINT(cond, slot)                                                \
    do {                                                                           \
        if ((cond) && (slot) < kTraceSlots) g_kda_trace[(slot)] = clock64();       \
    } while (0)
#else
#define KDA_TRACE_POINT(cond, slot) \
    do {                            \
    } while (0)
#endif
