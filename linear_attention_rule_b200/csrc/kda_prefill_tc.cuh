// KDA chunkwise prefill on the sm_100a tensor cores (bf16 operands, fp32 accumulation,
// fp32 state), d_k = d_v = 128 (64 runs as the first 64 channels of 128), chunk C = 64.
//
// "SemiAnalysis Kimi K3", FlashKDA section: a chunk-parallel preparation kernel (K1)
// and a chunk-serial recurrence kernel (K2).  With the state stored S[key][value], a the
// inclusive chunk-relative cumulative log-decay and gamma = e^{a_last}, one chunk is
//   U' = U - W S_in,   O = Q_dec S_in + Aqk U',   S_out = diag(gamma) S_in + K_res^T U'.
// Substituting U' moves every product that does not involve S_in into the parallel
// preparation:
//   S_out = diag(gamma) S_in + M S_in + K_res^T U,   M = -K_res^T W
//   O     = P S_in + Aqk U,                          P = Q_dec - Aqk W
// so the serial chain carries ONE tensor-core product per chunk, [M | K_res^T] [S_in ; U]
// (K = 128 + 64), and the output product [P | Aqk] [S_in ; U] runs beside it: the terms
// without S_in ride in the same accumulators as extra K steps.
//
//   chunk_index_kernel  cu_seqlens -> first chunk of every sequence and the chunk table
//                       (first token, rows) (device side, no host sync); validates cu_seqlens.
//   order_kernel        (several sequences) the order in which the recurrence takes them:
//                       most chunks first.
//   prep_kernel         one CTA of 8 warps per (chunk, head), fully parallel, 2 CTAs per SM:
//                         TMA: g, then q and k, then v tiles (128-byte swizzled) into
//                              shared memory, each group on its own barrier
//                         a, gamma, Q_dec = q e^a, K_dec = k e^a, K_inv = k e^-a      (FFMA/MUFU)
//                         K_res = K_inv gamma (held in registers until the product below
//                                              has read K_inv)
//                         [K_dec; Q_dec] K_inv^T                                      (MMA 128x64x128)
//                         L = strict_tril(beta K_dec K_inv^T), Aqk = tril(Q_dec K_inv^T)
//                         INV = (I + L)^-1: 16x16 diagonal blocks by forward substitution,
//                                               block doubling 16 -> 32 (fp32, CUDA cores),
//                                               32 -> 64 as two chained products     (MMA tf32)
//                         [W | U] = INV diag(beta) [K_dec | V]                       (MMA 128x256x64)
//                         -M = K_res^T W                                             (MMA 128x128x64)
//                         Aqk W -> P = Q_dec - Aqk W                                 (MMA 128x128x64)
//                       and writes one record per (chunk, head): the shared-memory
//                       operand images of P, M, K_res, U (4 value slices), Aqk, and gamma.
//   emit_index_kernel   (kda_prefill_emit only) chunk boundaries at which to emit states.
//   rec_kernel<NV>      one CTA per (sequence, head, NV = 32 or 64 value channels): the
//                       chunk chain with the fp32 state slice in registers and, beside it,
//                       the chunk outputs O = P S_in + Aqk U; a loader warp streams the
//                       records in (bulk copies, 2 stages) and two issuer warps launch the
//                       tensor-core products, hand-offs through mbarriers only.
#pragma once

#include <cuda.h>
#include <algorithm>
#include <atomic>
#include <type_traits>
#include <utility>

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace kda::sm100;

constexpr int D = 128;   // d_k = d_v
constexpr int C = 64;    // chunk

// ---- record of one (chunk, head) ---------------------------------------------------------
// Shared-memory operand images (bf16, rows of 128 B, 128-byte swizzle unless said), each
// 1024-byte aligned.  The recurrence reads two of them as the B operands of one product
// stream of N = 192 (its state columns and its output columns together):
constexpr uint32_t kRecSB = 0;          // [M ; P]  K-major, rows n: M's rows i (0..127), then P's rows r
                                        //          (128..191); key channels 0..63 / 64..127 in two halves
constexpr uint32_t kRecSBHalf = 24576;  //          of 24 KB
constexpr uint32_t kRecP = 16384;       //          P's first row inside each half
constexpr uint32_t kRecUB = 49152;      // K_res  rows t (64 tokens), key channels i 0..63 / 64..127 (2 x 8 KB):
                                        //        the MN-major A operand K_res^T
constexpr uint32_t kRecAQ = 65536;      // Aqk    K-major rows r (64), tokens s (8 KB)
constexpr uint32_t kRecU = 73728;       // U  rows t (64), value channels 32 s .. 32 s + 31 for 4 slices s
                                        //    (4 x 4 KB, rows of 64 B, 64-byte swizzle): MN-major U^T
constexpr uint32_t kRecGamma = 90112;   // gamma fp32 [128]
constexpr uint32_t kRecBytes = 90624;

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ inline int64_t max_chunks(int64_t total_tokens, int num_seqs) {
    return total_tokens / C + num_seqs;
}
// Workspace: [chunk offsets int32 (N+1)] [recurrence order of the sequences int32 (N+1)]
// [chunk table int2 (max_chunks)] [emission slot per chunk int32 (max_chunks)] [strong-decay
// count int32, pad] [strong-decay units int2 (max_chunks x H)] [records (max_chunks x H)]
__host__ inline size_t ws_table_offset(int num_seqs) {
    return align_up(sizeof(int32_t) * 2 * (size_t)(num_seqs + 1), 16);
}
__host__ inline size_t ws_emit_offset(int64_t total_tokens, int num_seqs) {
    return align_up(ws_table_offset(num_seqs) + sizeof(int2) * (size_t)max_chunks(total_tokens, num_seqs), 16);
}
__host__ inline size_t ws_strong_offset(int64_t total_tokens, int num_seqs) {
    return align_up(ws_emit_offset(total_tokens, num_seqs) +
                        sizeof(int32_t) * (size_t)max_chunks(total_tokens, num_seqs),
                    16);
}
// Chunk-parallel scan over long chains ("SemiAnalysis Kimi K3", FlashKDA section: the
// recurrence unrolled from S_in over a span of tokens is affine in S_in).  When few
// (sequence, head) chains are long, each sequence is cut into segments of `seg` chunks:
// every segment but the last runs from a zero state and composes its transition
// T = prod (diag(gamma) + M) over its chunks (seg_kernel), the segments' starting states
// follow as S_in(p+1) = T_p S_in(p) + S_local(p) (combine_kernel), and the recurrence then
// runs every segment from its starting state (rec_kernel over segments).
constexpr int kScanTargetCtas = 148;     // segments x heads aimed at (a B200's SM count)
constexpr int kScanMinSegChunks = 64;    // shortest segment worth the extra passes (measured)
// Chunks per segment, or 0 for one chain per (sequence, head).  The recurrence runs every
// chain (or segment) as four value-slice CTAs, so segments pay while chains x 4 leave at least
// half of the SMs idle.  Depends on the sizes only.
__host__ inline int scan_segment_chunks(int64_t total_tokens, int num_seqs, int H) {
    const int64_t chains = (int64_t)num_seqs * H;
    if (num_seqs <= 0) return 0;
    const int64_t segs = kScanTargetCtas / (chains * 4);   // segments per chain
    if (segs < 2) return 0;
    const int64_t per_chain = (total_tokens / num_seqs + C - 1) / C;   // mean chunks per sequence
    const int64_t len = (per_chain + segs - 1) / segs;
    return len >= kScanMinSegChunks && len < per_chain ? (int)len : 0;
}
__host__ inline int64_t max_segments(int64_t total_tokens, int num_seqs, int seg) {
    return seg > 0 ? max_chunks(total_tokens, num_seqs) / seg + num_seqs : 0;
}
constexpr size_t kSegStateBytes = 3 * sizeof(float) * D * D;   // S_local, T, S_in per (segment, head)
// [segment offsets int32 (N+1)] [segment count int32, pad] [segment table int4 (max_segs)]
// [segment states (max_segs x H)]
__host__ inline size_t ws_scan_offset(int64_t total_tokens, int num_seqs, int H) {
    return align_up(ws_strong_offset(total_tokens, num_seqs) + 16 +
                        sizeof(int2) * (size_t)max_chunks(total_tokens, num_seqs) * H,
                    16);
}
__host__ inline size_t ws_scan_bytes(int64_t total_tokens, int num_seqs, int H) {
    const int seg = scan_segment_chunks(total_tokens, num_seqs, H);
    if (seg == 0) return 0;
    const size_t ms = (size_t)max_segments(total_tokens, num_seqs, seg);
    return align_up(sizeof(int32_t) * (num_seqs + 1), 16) + 16 + align_up(sizeof(int4) * ms, 1024) +
           ms * H * kSegStateBytes;
}
__host__ inline size_t ws_records_offset(int64_t total_tokens, int num_seqs, int H) {
    return align_up(ws_scan_offset(total_tokens, num_seqs, H) + ws_scan_bytes(total_tokens, num_seqs, H),
                    1024);
}
__host__ inline size_t workspace_bytes(int64_t total_tokens, int num_seqs, int H) {
    return ws_records_offset(total_tokens, num_seqs, H) +
           (size_t)max_chunks(total_tokens, num_seqs) * H * kRecBytes;
}
// The same size, or false when the problem exceeds what the launches can address: H above
// 65535, a grid (chunks x heads, or sequences x heads x value slices) beyond 2^31 - 1 CTAs,
// or a byte count that does not fit in size_t.
__host__ inline bool workspace_bytes_checked(int64_t total_tokens, int num_seqs, int H, size_t* bytes) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || H > 65535) return false;
    const int64_t mc = max_chunks(total_tokens, num_seqs);
    if (mc > INT32_MAX || mc * H > INT32_MAX || (int64_t)num_seqs * H * 4 > INT32_MAX) return false;
    size_t rec = 0, total = 0;
    if (__builtin_mul_overflow((size_t)mc * (size_t)H, (size_t)kRecBytes + sizeof(int2), &rec)) return false;
    if (__builtin_add_overflow(rec, ws_records_offset(total_tokens, num_seqs, H), &total)) return false;
    total = workspace_bytes(total_tokens, num_seqs, H);
    *bytes = total;
    return true;
}

// Windowed workspace: when the caller's workspace is smaller than workspace_bytes, the chunks
// run in windows of W global chunks, each prepared and then run through the recurrence
// before the next; a sequence crossing a window boundary carries its fp32 state from one
// window to the next through one of two slots per head.
// [chunk offsets (N+1)] [chunk table (max_chunks)] [emission slot per chunk] [strong-decay
// count per window (max_chunks)] [strong-decay units (W x H)] [carry 2 x H x D x D fp32]
// [records (W x H)]
constexpr int64_t kMinWindowChunks = 8;
struct WindowLayout {
    size_t counts, list, carry, records, bytes;
};
__host__ inline WindowLayout window_layout(int64_t total_tokens, int num_seqs, int H, int64_t W) {
    const size_t mc = (size_t)max_chunks(total_tokens, num_seqs);
    WindowLayout l;
    l.counts = align_up(ws_emit_offset(total_tokens, num_seqs) + sizeof(int32_t) * mc, 16);
    l.list = align_up(l.counts + sizeof(int32_t) * mc, 16);
    l.carry = align_up(l.list + sizeof(int2) * (size_t)W * H, 1024);
    l.records = align_up(l.carry + 2 * sizeof(float) * (size_t)H * D * D, 1024);
    l.bytes = l.records + (size_t)W * H * kRecBytes;
    return l;
}
// Chunks per window for a workspace of ws_bytes: max_chunks (one window, the layout of
// workspace_bytes) when that fits, else the most that fit, 0 when not even kMinWindowChunks do.
__host__ inline int64_t window_chunks(int64_t total_tokens, int num_seqs, int H, size_t ws_bytes) {
    const int64_t mc = max_chunks(total_tokens, num_seqs);
    if (ws_bytes >= workspace_bytes(total_tokens, num_seqs, H)) return mc;
    const WindowLayout l0 = window_layout(total_tokens, num_seqs, H, 0);
    if (ws_bytes < l0.bytes) return 0;
    int64_t W = (int64_t)((ws_bytes - l0.bytes) / ((size_t)H * (kRecBytes + sizeof(int2))));
    if (W >= mc) W = mc - 1;   // a full window takes the one-window layout, which did not fit
    while (W >= kMinWindowChunks && window_layout(total_tokens, num_seqs, H, W).bytes > ws_bytes) --W;
    return W >= kMinWindowChunks ? W : 0;
}
// The least workspace the prefill accepts (a window of kMinWindowChunks, or one window when
// the whole problem is not larger than that).
__host__ inline size_t workspace_bytes_min(int64_t total_tokens, int num_seqs, int H) {
    const size_t full = workspace_bytes(total_tokens, num_seqs, H);
    const size_t win = window_layout(total_tokens, num_seqs, H, kMinWindowChunks).bytes;
    return win < full ? win : full;
}

// ------------------------------------------------------------------ chunk index
// Sequence containing global chunk c: the largest n with off[n] <= c.
__device__ __forceinline__ int find_seq(const int32_t* off, int num_seqs, int c) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Single CTA of 1024 threads: off[n] = sum_{m<n} ceil(len_m / C), off[N] = total chunks,
// and the chunk table tab[c] = (first token, rows) of every chunk c < off[N], so that the
// chunk-parallel kernels find their tokens with one load; also empties the strong-decay list.
// Inconsistent cu_seqlens -> KDA_ERR_BAD_SEQLENS and every count 0 (nothing downstream runs).
__global__ void __launch_bounds__(1024)
chunk_index_kernel(const int32_t* __restrict__ cu, int num_seqs, int64_t total,
                   int32_t* __restrict__ off, int2* __restrict__ tab, int32_t* __restrict__ etab,
                   int32_t* __restrict__ strong_count, int num_counts) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    kda_grid_launch_next();   // the preparation's blocks may start loading their inputs
    if (tid == 0) { carry = 0; bad = 0; }
    for (int i = tid; i < num_counts; i += blockDim.x) strong_count[i] = 0;   // one per window
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + tid;
        int cnt = 0;
        if (n < num_seqs) {
            const int64_t a = cu[n], b = cu[n + 1];
            bool ok = a >= 0 && b >= a && b <= total;
            if (n == 0 && a != 0) ok = false;
            if (n == num_seqs - 1 && b != total) ok = false;
            if (!ok) bad = 1;
            cnt = ok ? (int)((b - a + C - 1) / C) : 0;
        }
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;  // inclusive over warps
        }
        __syncthreads();
        const int before = (w > 0 ? warp_tot[w - 1] : 0) + x - cnt;
        if (n < num_seqs) off[n] = carry + before;
        __syncthreads();
        if (tid == 0) carry += warp_tot[31];
        __syncthreads();
    }
    if (tid == 0) off[num_seqs] = carry;
    __syncthreads();   // off[] (global, written by this CTA) is visible to all its threads
    if (bad) {
        if (tid == 0) kda_set_status(KDA_ERR_BAD_SEQLENS);
        for (int n = tid; n <= num_seqs; n += 1024) off[n] = 0;
        return;
    }
    const int nch = carry;
    for (int c = tid; c < nch; c += 1024) {
        const int n = find_seq(off, num_seqs, c);
        const int t0 = cu[n] + (c - off[n]) * C;
        tab[c] = make_int2(t0, min(C, cu[n + 1] - t0));
        if (etab) etab[c] = -1;
    }
}

// The order in which the recurrence's CTAs take several sequences, written after the chunk
// offsets (order = off + N + 1): most chunks first, ties by index, so that a long chain does
// not start last and set the launch's tail; the identity beyond kOrderMax sequences.  Single
// CTA of 1024 threads, a bitonic sort in its dynamic shared memory (order_smem_bytes).  Bad
// cu_seqlens left every count 0: the identity.
constexpr int kOrderMax = 2048;
__host__ __device__ inline int order_pow2(int num_seqs) {
    int p = 2;
    while (p < num_seqs) p <<= 1;
    return p;
}
__host__ inline size_t order_smem_bytes(int num_seqs) {
    return num_seqs <= kOrderMax ? 2 * sizeof(int32_t) * (size_t)order_pow2(num_seqs) : 0;
}
__global__ void __launch_bounds__(1024) order_kernel(int32_t* __restrict__ off, int num_seqs) {
    kda_grid_launch_next();   // the preparation's blocks may start loading their inputs
    kda_grid_wait();          // the chunk offsets
    const int tid = threadIdx.x;
    int32_t* order = off + num_seqs + 1;
    if (num_seqs > kOrderMax) {
        for (int n = tid; n < num_seqs; n += 1024) order[n] = n;
        return;
    }
    extern __shared__ int32_t order_smem[];
    const int P = order_pow2(num_seqs);
    int32_t* s_cnt = order_smem;
    int32_t* s_idx = order_smem + P;
    for (int i = tid; i < P; i += 1024) {
        s_cnt[i] = i < num_seqs ? off[i + 1] - off[i] : -1;   // padding sorts last
        s_idx[i] = i;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += 1024) {
                const int m = i ^ j;
                if (m > i) {
                    const int ci = s_cnt[i], cm = s_cnt[m], xi = s_idx[i], xm = s_idx[m];
                    const bool m_first = cm > ci || (cm == ci && xm < xi);   // m precedes i
                    if (((i & k) == 0) == m_first) {   // ascending runs want i first, descending m
                        s_cnt[i] = cm; s_cnt[m] = ci;
                        s_idx[i] = xm; s_idx[m] = xi;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int n = tid; n < num_seqs; n += 1024) order[n] = s_idx[n];
}

// Emission slots: etab[c] = e for the chunk c that ends at emission boundary e (the state
// after tokens cu[n] .. emit_pos[e] - 1 of its sequence n).  A boundary must end a chunk:
// cu[n] < t <= cu[n+1] with (t - cu[n]) a multiple of C, or t = cu[n+1].  Anything else is
// reported as KDA_ERR_BAD_EMIT_POS and emits nothing.
__global__ void emit_index_kernel(const int32_t* __restrict__ cu, int num_seqs,
                                  const int32_t* __restrict__ off, const int64_t* __restrict__ emit_pos,
                                  int num_emit, int32_t* __restrict__ etab) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= num_emit || off[num_seqs] == 0) return;   // nothing to emit when cu_seqlens were bad
    const int64_t t = emit_pos[e];
    // sequence n: the last with cu[n] < t
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] < t) lo = mid; else hi = mid - 1;
    }
    const int64_t a = cu[lo], b = cu[lo + 1];
    if (!(a < t && t <= b) || ((t - a) % C != 0 && t != b)) {
        kda_set_status(KDA_ERR_BAD_EMIT_POS);
        return;
    }
    etab[off[lo] + (int)((t - a - 1) / C)] = e;
}

// 2-D tiled TMA load (no multicast) of box (x, y) of `tmap` into shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tmap, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x),
        "r"(y), "r"(bar)
        : "memory");
}

// ------------------------------------------------------------------ chunk preparation
constexpr int kPrepThreads = 256;
constexpr int kPrepCtasPerSm = 2;
struct PrepSmem {
    // operand region: 128-byte-swizzled tiles of 64 rows (tokens) x 64 channels
    static constexpr uint32_t KD0 = 0, QD0 = 8192, KD1 = 16384, QD1 = 24576;
    static constexpr uint32_t V0 = 32768, KI0 = 40960, V1 = 49152, KI1 = 57344;
    static constexpr uint32_t BLK = 16384;   // stride between the channel halves
    // g tile fp32 [64][128] (plain); after the decay: Abar image, Aqk image, L / INV fp32
    static constexpr uint32_t GR = 65536;
    // L / INV as 32 x 32 fp32 tiles with 128-byte swizzled rows (the tf32 K-major operand
    // layout): TB the lower-right block (L22, then B^{-1}), T10 the lower-left block of L
    // stored transposed (L21^T), T00 the upper-left block (L11, then A^{-1}), TAT = A^{-T}.
    // The upper-right block is zero and not stored.
    static constexpr uint32_t ABAR = GR, AQK = GR + 8192, LI = GR + 16384;
    static constexpr uint32_t TB = LI, T10 = LI + 4096, T00 = LI + 8192, TAT = LI + 12288;
    static constexpr uint32_t XCH = GR + 33792;      // decay partials [8][128]; later T [32][36]
    static constexpr uint32_t BETA = XCH + 4608;     // [64]
    static constexpr uint32_t DIAG = BETA + 256;      // [64] q_r . k_r in fp32 (Aqk's diagonal)
    static constexpr uint32_t BAR = DIAG + 256;       // g's TMA, then the products in order
    static constexpr uint32_t BAR2 = BAR + 8;         // the UT's first product, then the last (Aqk W)
    static constexpr uint32_t BARQK = BAR2 + 8;       // TMA of q and k
    static constexpr uint32_t BARV = BARQK + 8;       // TMA of v
    static constexpr uint32_t TMEM = BARV + 8;
    static constexpr uint32_t STRONG = TMEM + 4;       // some channel's chunk decay is below kStrongDecay
    static constexpr uint32_t BYTES = TMEM + 8 + 1024;  // + alignment slack
};
constexpr int kTP = 36;                                   // row pitch of the product scratch
constexpr uint32_t kPrepTmemCols = 256;
constexpr uint32_t kPrepTxG = 32768, kPrepTxQK = 2 * 16384, kPrepTxV = 16384;   // bytes per barrier

__device__ __forceinline__ bool prep_sync_ok(bool ok, int tid) {
    if (__syncthreads_or(!ok)) {
        if (tid == 0) kda_set_status(KDA_ERR_TIMEOUT);
        return false;
    }
    return true;
}

// 4 KB staging slot of warp w for the record drains; all of them lie in operand space that
// is dead by then (K_res after its product, the Abar image, the L / INV buffer).
__device__ __forceinline__ uint32_t stage_slot(int w) {
    const uint32_t base = w < 2 ? PrepSmem::KI0 : w < 4 ? PrepSmem::KI1 : w < 6 ? PrepSmem::ABAR : PrepSmem::LI;
    return base + (w & 1) * 4096;
}

// A chunk whose cumulative log-decay falls below this in some channel is not prepared here:
// K_inv = k e^{-a} would leave the range of bf16 (~e^{88}).  The CTA lists it for
// prep_strong_kernel, which forms the products with K_inv without a positive exponent.
constexpr float kStrongDecay = -64.f;

// One CTA per (chunk, head) unit, 2 CTAs per SM.  kScalarG: the gate is one log-decay per
// (token, head), g [T, H] (Gated DeltaNet, the scalar forget gate that KDA makes diagonal):
// the same decay on every channel, loaded like beta instead of through the g tensor map.
// kPrologue: in_flags may hold KDA_IN_* prologue bits (the plain path compiles without them).
// DIN: channels per head of q, k, v and g, 128 or 64.  With 64 the chunk is prepared as the
// first 64 channels of a 128-channel one whose other channels are zero (q = k = v = 0 and no
// decay there): those channels add nothing to any product, so the records are the 128-channel
// ones with zero halves, and the state's rows and columns from 64 on stay zero.
template <bool kScalarG, bool kPrologue, int DIN>
__global__ void __launch_bounds__(kPrepThreads, kPrepCtasPerSm)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
            const float* __restrict__ g_scalar, const float* __restrict__ beta, int num_seqs, int H,
            const int32_t* __restrict__ off, const int2* __restrict__ tab, uint8_t* __restrict__ records,
            int32_t* __restrict__ strong_count, int2* __restrict__ strong_units,
            uint32_t in_flags_arg, int64_t total, int c_base) {
    const uint32_t in_flags = kPrologue ? in_flags_arg : 0u;
    using S = PrepSmem;
    // chunk c of the problem and head h, heads fastest: the CTAs that run at once cover a few
    // chunks of every head, so their input boxes tile whole token rows of q, k, v and g
    // (chunk-fastest, each read 256-byte pieces of thousands of rows, 3-6% slower).  Records
    // are indexed from the window's first chunk c_base.
    const int c = c_base + (int)(blockIdx.x / (unsigned)H), h = (int)(blockIdx.x % (unsigned)H);
    kda_grid_launch_next();
    // One sequence: chunk c is tokens 64 c .., and the input copies are issued before the wait
    // for the chunk table (whose kernel also resets the strong-decay count used below).
    const bool one_seq = num_seqs == 1;
    int total_chunks, t0, nrow;
    if (one_seq) {
        total_chunks = (int)((total + C - 1) / C);
        t0 = c * C;
        nrow = (int)(total - t0 < C ? total - t0 : C);
    } else {
        kda_grid_wait();
        total_chunks = off[num_seqs];
        t0 = nrow = 0;
        if (c < total_chunks) {
            const int2 e = tab[c];
            t0 = e.x;
            nrow = e.y;
        }
    }
    if (c >= total_chunks) {
        if (one_seq) kda_grid_wait();
        return;
    }
    uint8_t* rec = records + ((size_t)(c - c_base) * H + h) * kRecBytes;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar = sb + S::BAR;
    float* sBeta = reinterpret_cast<float*>(sm + S::BETA);
    float* sX = reinterpret_cast<float*>(sm + S::XCH);
    // element (r, c) of a tile of L / INV, and 4 of them from a column c divisible by 4
    auto lt = [&](uint32_t tile, int r, int c) -> float& {
        return *reinterpret_cast<float*>(sm + tile + sw128_off(r, c >> 2) + (c & 3) * 4);
    };
    auto lt4 = [&](uint32_t tile, int r, int c) -> float4& {
        return *reinterpret_cast<float4*>(sm + tile + sw128_off(r, c >> 2));
    };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;   // TMEM lane quarter, column half
    bool ok = true, v_ok = true;
    uint32_t phase = 0;
    volatile int* strong_flag = reinterpret_cast<volatile int*>(sm + S::STRONG);

    // ---- (0) TMA: rows t0..t0+63 of g, then q and k, then v (two 64-channel boxes each),
    // on three barriers in the order of use: the decay's prefix sums start once g is in, the
    // decayed operands once q and k are, and v is first read by the product of step (4).  The
    // barriers are initialised and the copies issued by the same thread, before anything else.
    const uint32_t barqk = sb + S::BARQK, barv = sb + S::BARV;
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 8, 1);
        mbar_init(barqk, 1);
        mbar_init(barv, 1);
        fence_mbar_init();
        *strong_flag = 0;
        constexpr uint32_t halves = DIN / 64;   // 64-channel boxes per tensor
        const int x0 = h * DIN;
        if (!kScalarG) {   // the g tile lands as [64 rows][DIN] fp32
            mbar_arrive_expect_tx(bar, kPrepTxG / 2 * halves);
            tma_load_2d(sb + S::GR, &tm_g, x0, t0, bar);
        }
        mbar_arrive_expect_tx(barqk, kPrepTxQK / 2 * halves);
        tma_load_2d(sb + S::QD0, &tm_q, x0, t0, barqk);
        if (DIN == 128) tma_load_2d(sb + S::QD1, &tm_q, x0 + 64, t0, barqk);
        tma_load_2d(sb + S::KD0, &tm_k, x0, t0, barqk);
        if (DIN == 128) tma_load_2d(sb + S::KD1, &tm_k, x0 + 64, t0, barqk);
        mbar_arrive_expect_tx(barv, kPrepTxV / 2 * halves);
        tma_load_2d(sb + S::V0, &tm_v, x0, t0, barv);
        if (DIN == 128) tma_load_2d(sb + S::V1, &tm_v, x0 + 64, t0, barv);
    }
    if (warp == 1) tmem_alloc(sb + S::TMEM, kPrepTmemCols);
    if (tid < C) {
        const float b = tid < nrow ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        sBeta[tid] = tid < nrow && (in_flags & kInBetaLogits) ? kda_sigmoid(b) : b;
    }
    if (kScalarG && tid >= 64 && tid < 64 + C) {   // scalar gate of each row, in the g tile's place
        const int r = tid - 64;
        const float x = r < nrow ? g_scalar[(size_t)(t0 + r) * H + h] : 0.f;
        reinterpret_cast<float*>(sm + S::GR)[r] = r < nrow && (in_flags & kInGLogits) ? kda_logsigmoid(x) : x;
    }
    if (one_seq) kda_grid_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + S::TMEM);
    const uint32_t tl = tmem + ((uint32_t)(32 * wq) << 16);   // this warp's TMEM lanes
    const bool ptr_ = c == 37 && h == 3 && tid == 0;
    (void)ptr_;
    KDA_TRACE_POINT(ptr_, 8192 + 0);
    if constexpr (!kScalarG) {   // a scalar gate came with plain loads, before the barrier above
        ok = mbar_wait(bar, phase);
        phase ^= 1;
        if (!prep_sync_ok(ok, tid)) goto done;
    }
    KDA_TRACE_POINT(ptr_, 8192 + 1);

    {
        // ---- (1) decay: thread = (block of 4 tokens rb, group of 8 channels cg) ----
        const int cg = lane & 15, half = lane >> 4, rb = 2 * warp + half;
        const int kb = cg >> 3, c8 = cg & 7;
        // fp32 rows of 8 channels per lane: the 8 lanes of a quarter warp sit 32 bytes apart,
        // so a 16-byte access of the same half by all of them meets every other bank twice.
        // Groups 4..7 of each eight take their upper half first (byte offsets o1, then o2):
        // each access instruction then covers the 32 banks once.
        const bool swp = (cg & 4) != 0;
        const uint32_t o1 = swp ? 16u : 0u, o2 = 16u - o1;
        float loc[4][8], acc[8], gam[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.f;
        const float* gt = reinterpret_cast<const float*>(sm + S::GR);
        // Rows past the chunk's last token are masked; a full chunk (the common case) runs a
        // copy of the row loops without the masks.
        auto decay_rows = [&](auto full_c) {
            constexpr bool kFull = decltype(full_c)::value;
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = 4 * rb + rr;
                float gv[8];
                if constexpr (kScalarG) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) gv[u] = gt[r];
                } else if (DIN == 128 || cg < 8) {
                    const uint32_t ga = smem_u32(gt + r * DIN + 8 * cg);
                    const float4 f1 = lds_f4(ga + o1), f2 = lds_f4(ga + o2);
                    const float4 g0 = swp ? f2 : f1, g1 = swp ? f1 : f2;
                    gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w;
                    gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
                    if (in_flags & kInGLogits) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) gv[u] = kda_logsigmoid(gv[u]);
                    }
                } else {   // channels without input: no decay
#pragma unroll
                    for (int u = 0; u < 8; ++u) gv[u] = 0.f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    acc[u] += kFull || r < nrow ? gv[u] : 0.f;
                    loc[rr][u] = acc[u];
                }
            }
        };
        if (nrow == C) decay_rows(std::true_type{});
        else decay_rows(std::false_type{});
        float other[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) other[u] = __shfl_xor_sync(0xffffffffu, acc[u], 16);
        if (half == 0) {   // the same access order as the g reads
            const float4 v0 = make_float4(acc[0] + other[0], acc[1] + other[1], acc[2] + other[2], acc[3] + other[3]);
            const float4 v1 = make_float4(acc[4] + other[4], acc[5] + other[5], acc[6] + other[6], acc[7] + other[7]);
            const uint32_t xa = smem_u32(sX + warp * D + 8 * cg);
            sts_f4(xa + o1, swp ? v1 : v0);
            sts_f4(xa + o2, swp ? v0 : v1);
        }
        KDA_TRACE_POINT(ptr_, 8192 + 20);
        __syncthreads();
        KDA_TRACE_POINT(ptr_, 8192 + 21);
        // sums over the warps' partials, held with the halves in access order (bp, tp), then
        // put back in channel order.  The two half-warps hold the same channels: half 0 reads
        // the partials of warps 0..3, half 1 those of warps 4..7, and they swap their sums.
        float base[8], tot[8], bp[8], tp[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) bp[u] = tp[u] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int w = 4 * half + k;
            const uint32_t xa = smem_u32(sX + w * D + 8 * cg);
            const float4 x1 = lds_f4(xa + o1), x2 = lds_f4(xa + o2);
            const float xv[8] = {x1.x, x1.y, x1.z, x1.w, x2.x, x2.y, x2.z, x2.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                tp[u] += xv[u];
                if (w < warp) bp[u] += xv[u];
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // a + b on one side, b + a on the other: the same sums
            tp[u] += __shfl_xor_sync(0xffffffffu, tp[u], 16);
            bp[u] += __shfl_xor_sync(0xffffffffu, bp[u], 16);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {   // the rows of half 0 of this warp precede those of half 1
            bp[u] += half ? (swp ? other[u + 4] : other[u]) : 0.f;
            bp[u + 4] += half ? (swp ? other[u] : other[u + 4]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            tot[u] = swp ? tp[u + 4] : tp[u];
            tot[u + 4] = swp ? tp[u] : tp[u + 4];
            base[u] = swp ? bp[u + 4] : bp[u];
            base[u + 4] = swp ? bp[u] : bp[u + 4];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) gam[u] = __expf(tot[u]);
        KDA_TRACE_POINT(ptr_, 8192 + 22);
        if (rb == 0) {
            float4* gdst = reinterpret_cast<float4*>(rec + kRecGamma + 32 * cg);
            gdst[0] = make_float4(gam[0], gam[1], gam[2], gam[3]);
            gdst[1] = make_float4(gam[4], gam[5], gam[6], gam[7]);
        }
        {   // strong decay: acted on at the barrier after the decayed images (which may then
            // hold infinities, never used)
            bool strong = false;
#pragma unroll
            for (int u = 0; u < 8; ++u) strong |= tot[u] < kStrongDecay;
            if (strong) *strong_flag = 1;
        }
        ok = mbar_wait(barqk, 0);   // q, k in (a failure is acted on at the barrier below)
        // K_res = K_inv gamma of this thread's rows, from the bf16 K_inv image's values; stored
        // in K_inv's place once the first product has read it
        uint4 kres[4];
        auto image_rows = [&](auto full_c) {
            constexpr bool kFull = decltype(full_c)::value;
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = 4 * rb + rr;
                const uint32_t o = kb * S::BLK + sw128_off(r, c8);
                float qv[8], kv[8], qd[8], kd[8], ki[8];
                if (DIN == 128 || kb == 0) {
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + S::QD0 + o), qv);
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + S::KD0 + o), kv);
                } else {   // channels 64..127 of a 64-channel input: zero, and so is v there
#pragma unroll
                    for (int u = 0; u < 8; ++u) qv[u] = kv[u] = 0.f;
                    *reinterpret_cast<uint4*>(sm + S::V0 + o) = make_uint4(0u, 0u, 0u, 0u);
                }
                if (in_flags & kInNormQK) {   // the 16 lanes of this half-warp hold the row's 128 channels
                    float sq = 0.f, sk = 0.f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) { sq += qv[u] * qv[u]; sk += kv[u] * kv[u]; }
#pragma unroll
                    for (int o2 = 1; o2 < 16; o2 <<= 1) {
                        sq += __shfl_xor_sync(0xffffffffu, sq, o2);
                        sk += __shfl_xor_sync(0xffffffffu, sk, o2);
                    }
                    const float iq = kda_inv_norm(sq), ik = kda_inv_norm(sk);
#pragma unroll
                    for (int u = 0; u < 8; ++u) { qv[u] *= iq; kv[u] *= ik; }
                }
                const bool live = kFull || r < nrow;
                {   // Aqk's diagonal needs no decay (e^{a_r - a_r} = 1): q_r . k_r in fp32 from the
                    // inputs, where the bf16 images' roundings would spoil a q . k that cancels
                    float dg = 0.f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) dg = fmaf(qv[u], kv[u], dg);
#pragma unroll
                    for (int o2 = 1; o2 < 16; o2 <<= 1) dg += __shfl_xor_sync(0xffffffffu, dg, o2);
                    if (cg == 0) reinterpret_cast<float*>(sm + S::DIAG)[r] = live ? dg : 0.f;
                }
                // a scalar gate gives every channel the same decay: two exponentials per row
                const float ep0 = __expf(base[0] + loc[rr][0]), em0 = __expf(-(base[0] + loc[rr][0]));
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float a = base[u] + loc[rr][u];
                    const float ep = kScalarG ? ep0 : __expf(a), em = kScalarG ? em0 : __expf(-a);
                    qd[u] = live ? qv[u] * ep : 0.f;
                    kd[u] = live ? kv[u] * ep : 0.f;
                    ki[u] = live ? kv[u] * em : 0.f;
                }
                *reinterpret_cast<uint4*>(sm + S::QD0 + o) = pack_bf16x8(qd);
                *reinterpret_cast<uint4*>(sm + S::KD0 + o) = pack_bf16x8(kd);
                const uint4 kiw = pack_bf16x8(ki);
                *reinterpret_cast<uint4*>(sm + S::KI0 + o) = kiw;
                float kr[8];
                unpack_bf16x8(kiw, kr);
#pragma unroll
                for (int u = 0; u < 8; ++u) kr[u] *= gam[u];
                kres[rr] = pack_bf16x8(kr);
            }
        };
        if (nrow == C) image_rows(std::true_type{});
        else image_rows(std::false_type{});
        fence_proxy_async_smem();
        if (!prep_sync_ok(ok, tid)) goto done;
        if (*strong_flag) {   // every thread sees the flag after the barrier
            if (tid == 0) {
                const int slot = atomicAdd(strong_count, 1);
                strong_units[slot] = make_int2(c, h);
            }
            goto done;
        }
        KDA_TRACE_POINT(ptr_, 8192 + 2);

        // ---- (2) [K_dec ; Q_dec] K_inv^T -> TMEM [0, 64) ----
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t ko = (ks >> 2) * S::BLK + (ks & 3) * 32;
                umma_bf16(tmem, smem_desc(sb + S::KD0 + ko, 16, 1024, kSwizzle128),
                          smem_desc(sb + S::KI0 + ko, 16, 1024, kSwizzle128), id, ks > 0);
            }
            umma_commit(bar);
        }
        // Each thread learns of the product's completion from the barrier itself; what follows
        // up to the next block barrier depends on nothing another warp writes first.  A wait
        // that gave up records the timeout and the CTA runs on (every later wait is bounded too).
        if (!mbar_wait(bar, phase)) kda_set_status(KDA_ERR_TIMEOUT);
        phase ^= 1;
        tc_fence_after();
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)   // the first product has read K_inv
            *reinterpret_cast<uint4*>(sm + S::KI0 + kb * S::BLK + sw128_off(4 * rb + rr, c8)) = kres[rr];
        if (wq != 0 || wh != 1) {   // (warp 4 would hold L's upper-right block: zero, not stored)
            float d[32];
            tmem_ld32(tl + 32 * wh, d);
            tmem_wait_ld();
            if (wq < 2) {   // L[r][s] = beta_r (K_dec K_inv^T)[r][s] for s < r, fp32
                const float br = sBeta[32 * wq + lane];
                if (wh == 0 && wq == 1) {   // L21, transposed: row s, column lane; then warp 5 may use it
#pragma unroll
                    for (int s2 = 0; s2 < 32; ++s2) lt(S::T10, s2, lane) = br * d[s2];
                    fence_proxy_async_smem();
                    bar_arrive_fixed<1>(64);
                } else {   // diagonal block L11 (warp 0) or L22 (warp 5): row lane, zero from the diagonal on
                    const uint32_t tile = wq ? S::TB : S::T00;
#pragma unroll
                    for (int u4 = 0; u4 < 8; ++u4) {
                        float e[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) e[u] = 4 * u4 + u < lane ? br * d[4 * u4 + u] : 0.f;
                        lt4(tile, lane, 4 * u4) = make_float4(e[0], e[1], e[2], e[3]);
                    }
                }
            } else {        // Aqk[r][s] = (Q_dec K_inv^T)[r][s] for s < r, q_r . k_r for s = r (bf16 image)
                const int r = 32 * (wq - 2) + lane;
                const float dg = reinterpret_cast<const float*>(sm + S::DIAG)[r];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    float e[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int s = 32 * wh + 8 * qq + u;
                        e[u] = s < r ? d[8 * qq + u] : (s == r ? dg : 0.f);
                    }
                    *reinterpret_cast<uint4*>(sm + S::AQK + sw128_off(r, 4 * wh + qq)) = pack_bf16x8(e);
                }
            }
        }
        // First step of the UT transform INV = (I + L)^{-1}: the two 16x16 diagonal blocks D_b
        // of a diagonal tile, inverted in place by the warp that drained it (warp 0: T00,
        // warp 5: TB), lane = (block b, column j).  Column-oriented forward substitution: once
        // x[s] is final it is subtracted from every later row, so the dependent chain is 15
        // FMAs long.
        if (warp == 0 || warp == 5) {
            __syncwarp();
            const uint32_t tile = warp == 5 ? S::TB : S::T00;
            const int b = lane >> 4, j = lane & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 15; ++s2) {
#pragma unroll
                for (int r = s2 + 1; r < 16; ++r) x[r] -= lt(tile, 16 * b + r, 16 * b + s2) * x[s2];
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 16; ++r) lt(tile, 16 * b + r, 16 * b + j) = x[r];
            if (warp == 0) {   // A^{-T} for the 32 -> 64 product: column j of D_b is its row 16 b + j,
                               // and the block left of D_1^T is zero (8 columns per lane)
#pragma unroll
                for (int r4 = 0; r4 < 16; r4 += 4)
                    lt4(S::TAT, 16 * b + j, 16 * b + r4) = make_float4(x[r4], x[r4 + 1], x[r4 + 2], x[r4 + 3]);
                lt4(S::TAT, 16 + j, 8 * b) = make_float4(0.f, 0.f, 0.f, 0.f);
                lt4(S::TAT, 16 + j, 8 * b + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __syncwarp();
            // 16 -> 32 in the same tile: X = -D_1 (L_10 D_0) into rows 16..31, columns 0..15;
            // lane = (row r, 8 columns); the product L_10 D_0 through the scratch rows
            // 16 p .. 16 p + 15
            {
                float* sT = sX;
                const int p = warp == 5 ? 1 : 0, r = lane >> 1, c8 = 8 * (lane & 1);
                float t[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) t[u] = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < 16; ++s2) {
                    const float l = lt(tile, 16 + r, s2);
                    const float4 d0 = lt4(tile, s2, c8);
                    const float4 d1 = lt4(tile, s2, c8 + 4);
                    t[0] += l * d0.x; t[1] += l * d0.y; t[2] += l * d0.z; t[3] += l * d0.w;
                    t[4] += l * d1.x; t[5] += l * d1.y; t[6] += l * d1.z; t[7] += l * d1.w;
                }
                *reinterpret_cast<float4*>(sT + (16 * p + r) * kTP + c8) = make_float4(t[0], t[1], t[2], t[3]);
                *reinterpret_cast<float4*>(sT + (16 * p + r) * kTP + c8 + 4) = make_float4(t[4], t[5], t[6], t[7]);
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) t[u] = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < 16; ++s2) {   // D_1 is lower triangular: its zeros add nothing
                    const float dh = lt(tile, 16 + r, 16 + s2);
                    const float4 t0 = *reinterpret_cast<const float4*>(sT + (16 * p + s2) * kTP + c8);
                    const float4 t1 = *reinterpret_cast<const float4*>(sT + (16 * p + s2) * kTP + c8 + 4);
                    t[0] -= dh * t0.x; t[1] -= dh * t0.y; t[2] -= dh * t0.z; t[3] -= dh * t0.w;
                    t[4] -= dh * t1.x; t[5] -= dh * t1.y; t[6] -= dh * t1.z; t[7] -= dh * t1.w;
                }
                lt4(tile, 16 + r, c8) = make_float4(t[0], t[1], t[2], t[3]);
                lt4(tile, 16 + r, c8 + 4) = make_float4(t[4], t[5], t[6], t[7]);
                if (warp == 0) {   // and into A^{-T}, transposed
#pragma unroll
                    for (int u = 0; u < 8; ++u) lt(S::TAT, c8 + u, 16 + r) = t[u];
                }
            }
            if (warp == 5) {
                // B^{-1} is final, and L21^T once warp 1 has arrived: the first product of the
                // 32 -> 64 step, D1 = B^{-1} (L21^T)^T -> TMEM [64, 96), runs while warp 0 still
                // inverts A.  (Its A operand has M = 128 rows: those past B^{-1} are the other
                // tiles, whatever they hold; product rows 32-127 are never read.)
                fence_proxy_async_smem();
                bar_sync_fixed<1>(64);
                if (lane == 0) {
                    tc_fence_after();
                    constexpr uint32_t id = idesc_tf32(128, 32);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)   // K = 8 per product: 32 bytes of a tile row
                        umma_tf32(tmem + 64, smem_desc(sb + S::TB + ks * 32, 16, 1024, kSwizzle128),
                                  smem_desc(sb + S::T10 + ks * 32, 16, 1024, kSwizzle128), id, ks > 0);
                    umma_commit(bar + 8);
                }
            }
        }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    KDA_TRACE_POINT(ptr_, 8192 + 3);
    // K_res and Aqk are final: their images go to the record as they are (thread 0 waits for
    // these copies to have read K_res before the K_res space is reused for staging)
    if (tid == 0) {
        bulk_s2g(rec + kRecUB, sb + S::KI0, 8192);
        bulk_s2g(rec + kRecUB + 8192, sb + S::KI1, 8192);
        bulk_s2g(rec + kRecAQ, sb + S::AQK, 8192);
    }

    // ---- (3) UT transform, 32 -> 64: INV = [[A^{-1}, 0], [X, B^{-1}]] with
    // X = -B^{-1} L21 A^{-1} (A, B the diagonal 32-blocks of I + L), on the tensor cores in
    // tf32: D1 = B^{-1} (L21^T)^T (issued by warp 5 above, committed to the second barrier),
    // then D2 = D1 (A^{-T})^T -> TMEM [96, 128) with D1 read from Tensor Memory, once D1 is
    // complete (products into different accumulators are not ordered); lanes 0-31
    // meaningful; X = -D2.  The entries of the tiles above their diagonals are 0 (L strictly
    // lower triangular, the inverse lower triangular), so the products need no masks.
    KDA_TRACE_POINT(ptr_, 8192 + 18);
    if (tid == 0) {
        v_ok = mbar_wait(bar + 8, 0);
        tc_fence_after();
        constexpr uint32_t id = idesc_tf32(128, 32);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            umma_tf32_tmem_a(tmem + 96, tmem + 64 + 8 * ks, smem_desc(sb + S::TAT + ks * 32, 16, 1024, kSwizzle128),
                             id, ks > 0);
        umma_commit(bar);
    }
    {   // meanwhile Abar = INV diag(beta) as a bf16 K-major A image, the blocks without X:
        // this thread writes columns c4..c4+3 and 32+c4..32+c4+3 of row r and columns 32+c4..
        // of row 32 + r
        const int r = tid >> 3, c4 = 4 * (tid & 7);
        const float4 b_lo = *reinterpret_cast<const float4*>(sBeta + c4);
        const float4 b_hi = *reinterpret_cast<const float4*>(sBeta + 32 + c4);
        auto put4 = [&](int row, int col, float4 x4, float4 b4) {
            *reinterpret_cast<uint2*>(sm + S::ABAR + sw128_off(row, col >> 3) + (col & 4) * 2) =
                make_uint2(pack_bf16x2(x4.x * b4.x, x4.y * b4.y), pack_bf16x2(x4.z * b4.z, x4.w * b4.w));
        };
        put4(r, c4, lt4(S::T00, r, c4), b_lo);
        put4(r, 32 + c4, make_float4(0.f, 0.f, 0.f, 0.f), b_hi);
        put4(32 + r, 32 + c4, lt4(S::TB, r, c4), b_hi);
    }
    if (!(mbar_wait(bar, phase) && v_ok)) kda_set_status(KDA_ERR_TIMEOUT);   // as after the first product
    phase ^= 1;
    tc_fence_after();
    if (wq == 0) {   // warps 0 and 4: row lane of X, columns 16 wh .. 16 wh + 15, into Abar's row 32 + lane
        float d[16], e[16];
        tmem_ld16(tl + 96 + 16 * wh, d);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) e[u] = -d[u] * sBeta[16 * wh + u];
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2)
            *reinterpret_cast<uint4*>(sm + S::ABAR + sw128_off(32 + lane, 2 * wh + j2)) = pack_bf16x8(&e[8 * j2]);
    }
    KDA_TRACE_POINT(ptr_, 8192 + 19);
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    KDA_TRACE_POINT(ptr_, 8192 + 4);

    // ---- (4) [W | U] = Abar [K_dec | V] -> TMEM [0, 256) (lanes 0-63 meaningful) ----
    // Only the issuing thread waits for v; a failure is carried into the check after the
    // product (which then read whatever v's buffer held: nothing is kept).
    if (tid == 0) {
        v_ok = mbar_wait(barv, 0);
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 256, false, true);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem, smem_desc(sb + S::ABAR + ks * 32, 16, 1024, kSwizzle128),
                      smem_desc(sb + S::KD0 + ks * 2048, S::BLK, 1024, kSwizzle128), id, ks > 0);
        umma_commit(bar);
    }
    if (!(mbar_wait(bar, phase) && v_ok)) kda_set_status(KDA_ERR_TIMEOUT);   // as after the first product
    phase ^= 1;
    tc_fence_after();
    if (wq < 2) {
        // rows r of W (column half 0) -> bf16 B image in place of K_dec (two 64-column blocks,
        // 128-byte swizzle); rows r of U (column half 1) -> four 32-column slices with a
        // 64-byte swizzle, slices 0, 1 in place of V's first block and 2, 3 of its second
        const int r = 32 * wq + lane;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float d[32];
            const int col = 128 * wh + 32 * cb;
            tmem_ld32(tl + col, d);
            tmem_wait_ld();
            if (wh == 0) {
                const uint32_t blk = S::KD0 + (col >> 6) * S::BLK;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    *reinterpret_cast<uint4*>(sm + blk + sw128_off(r, ((col & 63) >> 3) + qq)) =
                        pack_bf16x8(&d[8 * qq]);
            } else {
                const uint32_t slice = (cb < 2 ? S::V0 : S::V1) + (cb & 1) * 4096;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    *reinterpret_cast<uint4*>(sm + slice + sw64_off(r, qq)) = pack_bf16x8(&d[8 * qq]);
            }
        }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    KDA_TRACE_POINT(ptr_, 8192 + 5);

    // ---- (5) -M = K_res^T W -> TMEM [0, 128) and Aqk W -> TMEM [128, 256) (lanes 0-63), issued
    // back to back: the second product runs while the first is drained ----
    if (tid == 0) {
        tc_fence_after();
        // U is final: its image (four value slices) goes to the record as it is
        bulk_s2g(rec + kRecU, sb + S::V0, 8192);
        bulk_s2g(rec + kRecU + 8192, sb + S::V1, 8192);
        constexpr uint32_t idM = idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem, smem_desc(sb + S::KI0 + ks * 2048, S::BLK, 1024, kSwizzle128),
                      smem_desc(sb + S::KD0 + ks * 2048, S::BLK, 1024, kSwizzle128), idM, ks > 0);
        umma_commit(bar);
        constexpr uint32_t idP = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
            umma_bf16(tmem + 128, smem_desc(sb + S::AQK + ks * 32, 16, 1024, kSwizzle128),
                      smem_desc(sb + S::KD0 + ks * 2048, S::BLK, 1024, kSwizzle128), idP, ks > 0);
        umma_commit(bar + 8);
        bulk_wait_read<2>();   // the K_res / Aqk copies have read their sources
    }
    ok = mbar_wait(bar, phase);
    phase ^= 1;
    tc_fence_after();
    if (!prep_sync_ok(ok, tid)) goto done;
    {
        // Drain of M: warp (wq, wh) turns its 32 TMEM lanes x 64 columns (K block wh of M, rows
        // i = 32 wq ..) into a 4 KB piece of the record (32 complete swizzled rows) staged in a
        // private, now unused 4 KB slot, and copies it out with one bulk copy.
        uint8_t* slot = sm + stage_slot(warp);
        float d[64];
        tmem_ld32(tl + 64 * wh, *reinterpret_cast<float(*)[32]>(&d[0]));
        tmem_ld32(tl + 64 * wh + 32, *reinterpret_cast<float(*)[32]>(&d[32]));
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 64; ++u) d[u] = -d[u];
#pragma unroll
        for (int cb = 0; cb < 8; ++cb)
            *reinterpret_cast<uint4*>(slot + sw128_off(lane, cb)) = pack_bf16x8(&d[8 * cb]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) bulk_s2g(rec + kRecSB + wh * kRecSBHalf + wq * 4096, smem_u32(slot), 4096);
    }
    KDA_TRACE_POINT(ptr_, 8192 + 6);
    if (wq < 2) {
        // Drain of P = Q_dec - Aqk W: rows r = 32 wq .., K block wh.  Both products have read W
        // by now, so its space holds the staging slots.
        ok = __all_sync(0xffffffffu, mbar_wait(bar + 8, 1));   // its second phase
        if (!ok) {
            if (lane == 0) kda_set_status(KDA_ERR_TIMEOUT);
        } else {
            tc_fence_after();
            const int r = 32 * wq + lane;
            uint8_t* slot = sm + (wh ? S::KD1 : S::KD0) + wq * 4096;
            float d[64];
            tmem_ld32(tl + 128 + 64 * wh, *reinterpret_cast<float(*)[32]>(&d[0]));
            tmem_ld32(tl + 128 + 64 * wh + 32, *reinterpret_cast<float(*)[32]>(&d[32]));
            tmem_wait_ld();
#pragma unroll
            for (int cb = 0; cb < 8; ++cb) {
                float qv[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + S::QD0 + wh * S::BLK + sw128_off(r, cb)), qv);
#pragma unroll
                for (int u = 0; u < 8; ++u) d[8 * cb + u] = qv[u] - d[8 * cb + u];
            }
#pragma unroll
            for (int cb = 0; cb < 8; ++cb)
                *reinterpret_cast<uint4*>(slot + sw128_off(lane, cb)) = pack_bf16x8(&d[8 * cb]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) bulk_s2g(rec + kRecSB + wh * kRecSBHalf + kRecP + wq * 4096, smem_u32(slot), 4096);
        }
    }
done:
    // no copy may still read shared memory at exit; their global writes may still be in
    // flight (they complete before the grid does).  After a failed wait the input copies may
    // still be landing: give them their bounded waits (immediate once complete).
    if (lane == 0) bulk_wait_read<0>();
    if (tid == 0) {
        (void)mbar_wait(barqk, 0);
        (void)mbar_wait(barv, 0);
    }
    tc_fence_before();
    __syncthreads();
    KDA_TRACE_POINT(ptr_, 8192 + 7);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrepTmemCols);
    }
}

}  // namespace tc
}  // namespace kda

#include "kda_prep_strong.cuh"

namespace kda {
namespace tc {

// ------------------------------------------------------------------ chunk recurrence + outputs
// One CTA per (sequence, head, NV = 32 or 64 value channels).  Per chunk, two tensor-core
// product streams read the same bf16 image of S_in's slice and the slice of U:
//   D_S = K_res^T U + M S_in     (128 x NV, K = 64 + 128)  -> S_out = gamma S_in + D_S
//   D_O = Aqk U + P S_in         ( 64 x NV, K = 64 + 128)  -> O = D_O
// The U terms do not depend on S_in: they are issued into the (double-buffered) accumulators
// before the state of the chunk is ready, so the serial chain is S image -> M S_in (8 MMAs)
// -> drain and update -> next image.  Narrow slices (small N) keep each instruction of the
// chain cheap; the launch takes NV = 32 while four CTAs per (sequence, head) fit on the SMs
// at once, else 64.
//   warps 0-7: state (warp w: key rows 32 (w % 4) .. +31 = its TMEM lanes, columns NV/2 (w / 4)
//   .. of the slice), then this chunk's output rows 16 (w % 4) .. +15 (the M = 64 accumulator
//   puts row r in lane 32 (r / 16) + r % 16); warp 8: loader (2 stages); warp 9: issuer of D_S;
//   warp 10: issuer of D_O.  The two issuers are separate threads, so that the output product
//   never holds back the chain's.
constexpr int kRecThreads = 352;
constexpr int kRecStateWarps = 8;
constexpr int kRecLoaderWarp = 8, kIssuerWarp = 9, kIssuerOWarp = 10;
constexpr int kStages = 2, kPrefetchAhead = 4;
constexpr uint32_t kUSlice = 4096;    // one 32-column U slice: 64 token rows of 64 B
constexpr uint32_t kRecHead = kRecU;  // [M ; P], K_res and Aqk: the record's first 72 KB

template <int NV_>
struct RecCfg {
    static constexpr int NV = NV_, NSL = D / NV, NC = NV / 2;   // NC: columns per thread
    // stage: [M ; P], K_res and Aqk as stored, then this CTA's U slice
    static constexpr uint32_t kStU = kRecHead;
    static constexpr uint32_t kUBytes = (NV / 32) * kUSlice;
    static constexpr uint32_t kStageBytes = kStU + kUBytes;
    // S image (MN-major B operand): 128 key rows of 2 NV bytes, 128- or 64-byte swizzle
    static constexpr uint32_t kSRow = 2 * NV, kSImg = 128 * kSRow, kSSbo = 8 * kSRow;
    static constexpr uint32_t kSSwz = NV == 64 ? kSwizzle128 : kSwizzle64;
    static constexpr uint32_t SB = kStages * kStageBytes;   // S images, 2 buffers
    static constexpr uint32_t OST = SB + 2 * kSImg;          // output staging [64 rows][2 NV B]
    // full[2] empty[2] mma_s[2] mma_o[2] ofree[2] sbr[2] sdrain[2] fin[2]
    static constexpr uint32_t BAR = OST + 64 * kSRow;
    static constexpr uint32_t TMEM = BAR + 16 * 8;
    static constexpr uint32_t FLAG = TMEM + 4;
    static constexpr uint32_t BYTES = FLAG + 4 + 1024;
    // D_S buffers [0, NV), [NV, 2 NV); D_O buffers [2 NV, 3 NV), [3 NV, 4 NV)
    static constexpr uint32_t kTmemCols = 4 * NV;
    static_assert(kStageBytes % 1024 == 0, "stage images must stay 1 KB aligned");
    static_assert(BYTES <= 232448, "recurrence shared memory exceeds 227 KB");
    // byte offset of 16-byte chunk `ch` of row `row` in an S image / the output staging
    __device__ static __forceinline__ uint32_t s_off(uint32_t row, uint32_t ch) {
        if constexpr (NV == 64) return sw128_off(row, ch);
        else return sw64_off(row, ch);
    }
};

// Loader of the recurrence kernels (one thread): every chunk's record (the first head_bytes
// as stored, then `tail_bytes` from tail_off) into stage kk % 2 once the products of chunk
// kk - 2 have released it; the records a few chunks ahead go to L2 first.  Never leaves with
// copies in flight.
template <typename RecordAt>
__device__ __forceinline__ void load_record_stages(uint32_t sb, uint32_t stage_bytes, uint32_t full0,
                                                   uint32_t empty0, int nchunks, volatile int* abort_flag,
                                                   RecordAt record, uint32_t head_bytes, uint32_t tail_off,
                                                   uint32_t tail_bytes) {
    auto prefetch = [&](int kk) {
        bulk_prefetch_l2(record(kk), head_bytes);
        if (tail_bytes) bulk_prefetch_l2(record(kk) + tail_off, tail_bytes);
    };
    for (int kk = 0; kk < nchunks && kk < kPrefetchAhead; ++kk) prefetch(kk);
    int issued = 0;
    for (int kk = 0; kk < nchunks && !*abort_flag; ++kk) {
        const int st = kk % kStages, use = kk / kStages;
        if (use > 0 && !mbar_wait(empty0 + 8 * st, (use - 1) & 1)) {
            kda_set_status(KDA_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
        }
        const uint32_t fb = full0 + 8 * st, dst = sb + st * stage_bytes;
        mbar_arrive_expect_tx(fb, head_bytes + tail_bytes);
        bulk_g2s(dst, record(kk), head_bytes, fb);
        if (tail_bytes) bulk_g2s(dst + head_bytes, record(kk) + tail_off, tail_bytes, fb);
        if (kk + kPrefetchAhead < nchunks) prefetch(kk + kPrefetchAhead);
        ++issued;
    }
    for (int kk = max(0, issued - kStages); kk < issued; ++kk)
        mbar_wait(full0 + 8 * (kk % kStages), (kk / kStages) & 1);
}

// Segments of the chunk-parallel scan (seg_tab non-null): CTA (segment s, head h, slice) runs
// the segment's chunks from S_in(s) (the initial state for a sequence's first segment) and
// writes the final state only from the sequence's last segment.
// The window of chunks one recurrence launch covers: chunks [c_lo, c_hi) of the problem,
// whose records start at records[0]; a sequence that began before c_lo starts from
// carry_in, one that continues past c_hi leaves its state in carry_out (both [H][D][D]
// fp32).  One window from 0 to INT32_MAX is the whole problem.
struct RecWindow {
    int c_lo, c_hi;
    int last;   // the last window: it also owns empty sequences that sit at its end
    const float* carry_in;
    float* carry_out;
};
constexpr RecWindow kWholeProblem = {0, INT32_MAX, 1, nullptr, nullptr};

// DIN: channels per head of the caller's outputs and states (128, or 64 with the chunk
// tensors of a 128-channel problem whose channels from 64 on are zero: only the value slices
// of the first 64 columns run, and only the state's first 64 rows are read or written).
// kOrdered: the CTAs take the sequences in the order the chunk-table kernel wrote after the
// chunk offsets (several sequences); otherwise in index order.
template <int NV, int DIN, bool kOrdered>
__global__ void __launch_bounds__(kRecThreads, 1)
rec_kernel(int num_seqs, int H, const int32_t* __restrict__ off, const int2* __restrict__ tab,
           const uint8_t* __restrict__ records, const float* initial_state, float* final_state,
           __nv_bfloat16* __restrict__ out, const int32_t* __restrict__ etab, float* emit_states,
           const int4* __restrict__ seg_tab, const int32_t* __restrict__ seg_count,
           const float* __restrict__ seg_states, RecWindow win) {
    using S = RecCfg<NV>;
    constexpr int NSL = DIN / NV;   // value slices of the caller's columns
    kda_grid_wait();   // the chunk table and the records
    const int sl = blockIdx.x % NSL;
    const int h = (blockIdx.x / NSL) % H;
    const int unit = blockIdx.x / (NSL * H);   // sequence, or scan segment
    int n, c_begin, nchunks;
    bool write_final = final_state != nullptr;
    const float* s_init;
    int s_ld = DIN;             // row length of s_init
    float* s_carry = nullptr;   // where the state goes when the sequence continues past the window
    if (seg_tab) {
        if (unit >= *seg_count) return;   // the whole CTA, before any barrier
        const int4 sg = seg_tab[unit];    // (sequence, first chunk, chunks, index | last << 16)
        n = sg.x;
        c_begin = sg.y;
        nchunks = sg.z;
        write_final = write_final && (sg.w >> 16) != 0;
        const bool first = (sg.w & 0xFFFF) == 0;
        s_init = first ? (initial_state ? initial_state + ((size_t)n * H + h) * DIN * DIN : nullptr)
                       : seg_states + ((size_t)unit * H + h) * (kSegStateBytes / sizeof(float)) + 2 * D * D;
        if (!first) s_ld = D;
    } else {
        // this sequence's chunks inside the window [c_lo, c_hi)
        n = kOrdered ? off[num_seqs + 1 + unit] : unit;
        const int a = off[n], b = off[n + 1];
        c_begin = max(a, win.c_lo);
        nchunks = min(b, win.c_hi) - c_begin;
        if (nchunks <= 0) {
            // an empty sequence belongs to the window at its position (the last window takes
            // those at the very end); a sequence outside the window has nothing to do here
            const bool owner = a == b && a >= win.c_lo && (a < win.c_hi || win.last);
            if (!owner) return;   // the whole CTA, before any barrier
            nchunks = 0;
        }
        const bool starts_here = a >= win.c_lo;
        s_init = starts_here ? (initial_state ? initial_state + ((size_t)n * H + h) * DIN * DIN : nullptr)
                             : win.carry_in + (size_t)h * DIN * DIN;
        if (b > win.c_hi) {
            write_final = false;
            s_carry = win.carry_out + (size_t)h * DIN * DIN;
        }
    }
    auto record = [&](int kk) { return records + ((size_t)(c_begin + kk - win.c_lo) * H + h) * kRecBytes; };

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    const uint32_t sb = smem_u32(sm);
    // Each barrier's waiters can never fall two phases behind: its next phase needs an
    // arrival that every waiter of the current phase precedes.
    const uint32_t full0 = sb + S::BAR, empty0 = full0 + 16, mma_s = full0 + 32, mma_o = full0 + 48;
    const uint32_t ofree = full0 + 64, sbr0 = full0 + 80, sdrain = full0 + 96, fin = full0 + 112;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::FLAG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) tmem_alloc(sb + S::TMEM, S::kTmemCols);
    if (tid == 0) {
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(full0 + 8 * b2, 1);
            mbar_init(empty0 + 8 * b2, 2);    // tcgen05.commit of both products that read it
            mbar_init(mma_s + 8 * b2, 1);
            mbar_init(mma_o + 8 * b2, 1);
            mbar_init(ofree + 8 * b2, kRecStateWarps);
            mbar_init(sbr0 + 8 * b2, kRecStateWarps);
            mbar_init(sdrain + 8 * b2, kRecStateWarps);
            mbar_init(fin + 8 * b2, 1);
        }
        fence_mbar_init();
        *abort_flag = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = *reinterpret_cast<volatile uint32_t*>(sm + S::TMEM);

    if (warp == kRecLoaderWarp) {
        if (lane == 0)
            load_record_stages(sb, S::kStageBytes, full0, empty0, nchunks, abort_flag, record, kRecHead,
                               kRecU + sl * S::kUBytes, S::kUBytes);
    } else if (warp == kIssuerWarp || warp == kIssuerOWarp) {
        // ---------------- issuers: D_S (warp 9) and D_O (warp 10) into buffer kk % 2 ----------
        // The U term first (its buffer drained by chunk kk - 2), then, once the image of S_in is
        // in, the S term.  The image of S_in stays put until both products of the chunk are
        // done: the state warps overwrite it only after they have drained D_O.
        if (lane == 0) {
            const bool is_s = warp == kIssuerWarp;
            constexpr uint32_t idSU = idesc_bf16(128, NV, true, true);     // K_res^T (MN-major) U (MN-major)
            constexpr uint32_t idSS = idesc_bf16(128, NV, false, true);    // M (K-major) S (MN-major)
            constexpr uint32_t idOU = idesc_bf16(64, NV, false, true);     // Aqk (K-major) U
            constexpr uint32_t idOS = idesc_bf16(64, NV, false, true);     // P (K-major) S
            bool ok = true;
            for (int kk = 0; kk < nchunks && !*abort_flag; ++kk) {
                const int st = kk % kStages, b = kk & 1, use = kk >> 1;
                const uint32_t stage = sb + st * S::kStageBytes;
                const uint32_t sbuf = sb + S::SB + b * S::kSImg;
                const uint32_t tD = tS + (is_s ? 0u : 2u * NV) + NV * b;
                if (!mbar_wait(full0 + 8 * st, (kk / kStages) & 1) ||
                    (use > 0 && !mbar_wait((is_s ? sdrain : ofree) + 8 * b, (use - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks) {
                    const uint64_t bu = smem_desc(stage + S::kStU + ks * 1024, kUSlice, 512, kSwizzle64);
                    if (is_s)
                        umma_bf16(tD, smem_desc(stage + kRecUB + ks * 2048, 8192, 1024, kSwizzle128), bu, idSU, ks > 0);
                    else
                        umma_bf16(tD, smem_desc(stage + kRecAQ + ks * 32, 16, 1024, kSwizzle128), bu, idOU, ks > 0);
                }
                if (!mbar_wait(sbr0 + 8 * b, use & 1)) {
                    ok = false;
                    break;
                }
                if (is_s) KDA_TRACE_POINT(blockIdx.x == 0 && kk < 512, 16 * kk + 8);
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t bs = smem_desc(sbuf + ks * 2 * S::kSSbo, 16, S::kSSbo, S::kSSwz);
                    const uint32_t a = stage + kRecSB + (ks >> 2) * kRecSBHalf + (ks & 3) * 32 + (is_s ? 0u : kRecP);
                    umma_bf16(tD, smem_desc(a, 16, 1024, kSwizzle128), bs, is_s ? idSS : idOS, 1);
                }
                umma_commit((is_s ? mma_s : mma_o) + 8 * b);
                umma_commit(empty0 + 8 * st);
                if (is_s) KDA_TRACE_POINT(blockIdx.x == 0 && kk < 512, 16 * kk + 9);
            }
            if (!ok) {
                kda_set_status(KDA_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // nothing may still run on the tensor pipe when Tensor Memory is released
            const uint32_t fb = fin + 8 * (is_s ? 0 : 1);
            umma_commit(fb);
            mbar_wait(fb, 0);
        }
    } else {
        // ---------------- state: row i, columns NC cw .. NC cw + NC - 1 of the slice -------
        constexpr int NC = S::NC;
        const int q4 = warp & 3, i = 32 * q4 + lane, cw = warp >> 2;
        const uint32_t taw = (uint32_t)(32 * q4) << 16;
        const size_t col0 = (size_t)sl * NV + NC * cw;
        const int r_out = 16 * q4 + lane;   // output row of this lane (lanes 0-15)
        float Sr[NC];
        if (s_init && i < DIN) {
#pragma unroll
            for (int j4 = 0; j4 < NC / 4; ++j4) {
                const float4 t = reinterpret_cast<const float4*>(s_init + (size_t)i * s_ld + col0)[j4];
                Sr[4 * j4] = t.x; Sr[4 * j4 + 1] = t.y; Sr[4 * j4 + 2] = t.z; Sr[4 * j4 + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < NC; ++j) Sr[j] = 0.f;
        }
        // bf16 image of the state entering the next chunk (B operand of both products)
        auto put_state = [&](int b) {
#pragma unroll
            for (int cb = 0; cb < NC / 8; ++cb)
                *reinterpret_cast<uint4*>(sm + S::SB + b * S::kSImg + S::s_off(i, (NC / 8) * cw + cb)) =
                    pack_bf16x8(&Sr[8 * cb]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(sbr0 + 8 * b);
        };
        // gamma of row i, the (first token, rows) and the emission slot of a chunk, loaded a
        // chunk ahead so that their global-load latency stays off the chain
        float gam_next = 0.f;
        int2 ce_next = make_int2(0, 0);
        int e_next = -1;
        if (nchunks > 0) {
            gam_next = __ldg(reinterpret_cast<const float*>(record(0) + kRecGamma) + i);
            ce_next = tab[c_begin];
            if (etab) e_next = etab[c_begin];
            put_state(0);
        }
        bool ok = true;
        for (int kk = 0; kk < nchunks; ++kk) {
            const int b = kk & 1, use = kk >> 1;
            const bool more = kk + 1 < nchunks;
            const float gam = gam_next;
            const int2 ce = ce_next;
            const int e_slot = e_next;
            if (more) {
                gam_next = __ldg(reinterpret_cast<const float*>(record(kk + 1) + kRecGamma) + i);
                ce_next = tab[c_begin + kk + 1];
                if (etab) e_next = etab[c_begin + kk + 1];
            }
            const bool tr = blockIdx.x == 0 && tid == 0 && kk < 512;
            (void)tr;
            KDA_TRACE_POINT(tr, 16 * kk + 0);
            ok = __all_sync(0xffffffffu, mbar_wait(mma_s + 8 * b, use & 1));
            if (!ok || *abort_flag) { ok = false; break; }
            KDA_TRACE_POINT(tr, 16 * kk + 1);
            tc_fence_after();
            {
                float dsv[NC];
                tmem_ld_cols(tS + taw + NV * b + NC * cw, dsv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sdrain + 8 * b);
#pragma unroll
                for (int j = 0; j < NC; ++j) Sr[j] = fmaf(gam, Sr[j], dsv[j]);
            }
            KDA_TRACE_POINT(tr, 16 * kk + 2);
            // the image of S_{kk+1} replaces that of S_{kk-1}, whose products (D_S(kk-1), and
            // D_O(kk-1), drained below in the previous pass) are complete
            if (more) put_state((kk + 1) & 1);
            KDA_TRACE_POINT(tr, 16 * kk + 4);
            if (e_slot >= 0 && i < DIN) {   // emission boundary at the end of this chunk: the state as it is
                float* dst = emit_states + ((size_t)e_slot * H + h) * DIN * DIN + (size_t)i * DIN + col0;
#pragma unroll
                for (int j4 = 0; j4 < NC / 4; ++j4)
                    reinterpret_cast<float4*>(dst)[j4] =
                        make_float4(Sr[4 * j4], Sr[4 * j4 + 1], Sr[4 * j4 + 2], Sr[4 * j4 + 3]);
            }
            // output rows 16 q4 .. 16 q4 + 15, columns NC cw .. of the slice
            ok = __all_sync(0xffffffffu, mbar_wait(mma_o + 8 * b, use & 1));
            if (!ok) break;
            tc_fence_after();
            float dov[NC];
            tmem_ld_cols(tS + taw + 2 * NV + NV * b + NC * cw, dov);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree + 8 * b);
            // lane l (< 16) holds row 16 q4 + l: stage the bf16 rows, then re-read them so that
            // NC / 8 lanes store one row's 2 NC contiguous bytes
            uint8_t* os = sm + S::OST;
            if (lane < 16) {
#pragma unroll
                for (int cb = 0; cb < NC / 8; ++cb)
                    *reinterpret_cast<uint4*>(os + S::s_off(r_out, (NC / 8) * cw + cb)) = pack_bf16x8(&dov[8 * cb]);
            }
            __syncwarp();
            {
                constexpr int LPR = NC / 8, RPI = 32 / LPR;   // lanes per row, rows per instruction
                uint4 ov[16 / RPI];
#pragma unroll
                for (int g = 0; g < 16 / RPI; ++g)
                    ov[g] = *reinterpret_cast<const uint4*>(
                        os + S::s_off(16 * q4 + RPI * g + lane / LPR, LPR * cw + lane % LPR));
#pragma unroll
                for (int g = 0; g < 16 / RPI; ++g) {
                    const int rr = 16 * q4 + RPI * g + lane / LPR;
                    if (rr < ce.y)
                        *reinterpret_cast<uint4*>(out + ((size_t)(ce.x + rr) * H + h) * DIN + sl * NV + NC * cw +
                                                  8 * (lane % LPR)) = ov[g];
                }
            }
            __syncwarp();   // the staging rows are rewritten by the next chunk
            KDA_TRACE_POINT(tr, 16 * kk + 7);
        }
        if (!ok) {
            if (lane == 0) kda_set_status(KDA_ERR_TIMEOUT);
            *abort_flag = 1;
        } else if ((write_final || s_carry) && i < DIN) {
            float* dst = (s_carry ? s_carry : final_state + ((size_t)n * H + h) * DIN * DIN) + (size_t)i * DIN + col0;
#pragma unroll
            for (int j4 = 0; j4 < NC / 4; ++j4)
                reinterpret_cast<float4*>(dst)[j4] =
                    make_float4(Sr[4 * j4], Sr[4 * j4 + 1], Sr[4 * j4 + 2], Sr[4 * j4 + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tS, S::kTmemCols);
    }
}

// ------------------------------------------------------------------ chunk-parallel scan
// Scan segments from the chunk offsets: sequence n gets max(1, ceil(chunks_n / seg))
// segments (an empty sequence one segment without chunks, so that its final state is still
// written); seg_tab[s] = (n, first chunk, chunks, index | last << 16), seg_off[n] the first
// segment of sequence n, *seg_count the total.  Single CTA of 1024 threads.
__global__ void __launch_bounds__(1024)
segment_index_kernel(int num_seqs, const int32_t* __restrict__ off, int seg,
                     int32_t* __restrict__ seg_off, int32_t* __restrict__ seg_count,
                     int4* __restrict__ seg_tab) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + tid;
        const int cnt = n < num_seqs ? max(1, (off[n + 1] - off[n] + seg - 1) / seg) : 0;
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        if (n < num_seqs) seg_off[n] = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - cnt;
        __syncthreads();
        if (tid == 0) carry += warp_tot[31];
        __syncthreads();
    }
    if (tid == 0) {
        seg_off[num_seqs] = carry;
        *seg_count = carry;
    }
    __syncthreads();
    for (int sgi = tid; sgi < carry; sgi += 1024) {
        const int n = find_seq(seg_off, num_seqs, sgi);
        const int p = sgi - seg_off[n], last = seg_off[n + 1] - 1 == sgi;
        const int chunks = off[n + 1] - off[n];
        seg_tab[sgi] = make_int4(n, off[n] + p * seg, max(0, min(seg, chunks - p * seg)), p | (last << 16));
    }
}

// Pass 1 of the chunk-parallel scan: CTA (segment s, head h), for every segment but the last
// of its sequence, runs the segment's chunks from a zero state (S_local) and composes the
// segment's transition T = prod (diag(gamma) + M) beside it; both go to the segment states.
// In the transposed form of rec_kernel, X = T^T evolves like S^T without the U term,
//   X <- X diag(gamma) + X M^T  from X = I,
// so the chain step is two products with the same B operand (M, the first 128 rows of the
// record's [M ; P]).  warps 0-7: S^T and X (rows j = 32 (w % 4) + lane, columns 64 (w / 4) ..),
// warp 8: loader, warp 9: issuer.  Tensor Memory: D_S [0, 128), D_X [128, 256), S^T images
// [256, 320) [320, 384), X images [384, 448) [448, 512).
constexpr int kSegThreads = 320, kSegStateWarps = 8, kSegLoaderWarp = 8, kSegIssuerWarp = 9;
struct SegSmem {
    static constexpr uint32_t kStage = (kRecBytes + 1023) / 1024 * 1024;   // one record, as stored
    // full[2] empty[2] mma sready[2] sdrain fin
    static constexpr uint32_t BAR = kStages * kStage;
    static constexpr uint32_t TMEM = BAR + 16 * 8;
    static constexpr uint32_t FLAG = TMEM + 4;
    static constexpr uint32_t BYTES = FLAG + 4 + 1024;
    static_assert(BYTES <= 232448, "scan shared memory exceeds 227 KB");
};
constexpr uint32_t kSegTmemCols = 512;
// operand descriptors of the transposed products, K step ks: [M ; P] (K-major B), K_res
// (MN-major B) and U^T (MN-major A, four 32-column atoms)
__device__ __forceinline__ uint64_t seg_m_desc(uint32_t stage, int ks) {
    return smem_desc(stage + kRecSB + (ks >> 2) * kRecSBHalf + (ks & 3) * 32, 16, 1024, kSwizzle128);
}
__device__ __forceinline__ uint64_t seg_kres_desc(uint32_t stage, int ks) {
    return smem_desc(stage + kRecUB + ks * 2048, 8192, 1024, kSwizzle128);
}
__device__ __forceinline__ uint64_t seg_u_desc(uint32_t stage, int ks) {
    return smem_desc(stage + kRecU + ks * 1024, kUSlice, 512, kSwizzle64);
}
__global__ void __launch_bounds__(kSegThreads, 1)
seg_kernel(int H, const uint8_t* __restrict__ records, const int4* __restrict__ seg_tab,
           const int32_t* __restrict__ seg_count, float* __restrict__ seg_states) {
    using S = SegSmem;
    const int h = blockIdx.x % H, sgi = blockIdx.x / H;
    if (sgi >= *seg_count) return;   // the whole CTA, before any barrier
    const int4 sg = seg_tab[sgi];
    if ((sg.w >> 16) != 0) return;   // a sequence's last segment needs no transition
    const int c_begin = sg.y, nchunks = sg.z;
    auto record = [&](int kk) { return records + ((size_t)(c_begin + kk) * H + h) * kRecBytes; };
    constexpr uint32_t kDX = 128, kSTi = 256, kXTi = 384;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    const uint32_t sb = smem_u32(sm);
    const uint32_t full0 = sb + S::BAR, empty0 = full0 + 16, mmas = full0 + 32, sready0 = full0 + 64;
    const uint32_t sdrain = full0 + 80, finbar = full0 + 112;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::FLAG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0) tmem_alloc(sb + S::TMEM, kSegTmemCols);
    if (tid == 0) {
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(full0 + 8 * b2, 1);
            mbar_init(empty0 + 8 * b2, 1 + kSegStateWarps);
            mbar_init(sready0 + 8 * b2, kSegStateWarps);
        }
        mbar_init(mmas, 1);
        mbar_init(sdrain, kSegStateWarps);
        mbar_init(finbar, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *reinterpret_cast<volatile uint32_t*>(sm + S::TMEM);

    if (warp == kSegLoaderWarp) {
        if (lane == 0)
            load_record_stages(sb, S::kStage, full0, empty0, nchunks, abort_flag, record, kRecU, kRecU,
                               kRecBytes - kRecU);
    } else if (warp == kSegIssuerWarp) {
        if (lane == 0) {
            constexpr uint32_t idSU = idesc_bf16(128, 128, true, true);    // U^T (MN-major) K_res (MN-major)
            constexpr uint32_t idSS = idesc_bf16(128, 128, false, false);  // S^T / X (TMEM) M (K-major)
            bool ok = true;
            for (int kk = 0; kk < nchunks && !*abort_flag; ++kk) {
                const int st = kk % kStages, b = kk & 1;
                const uint32_t stage = sb + st * S::kStage;
                // the record is in; D_S and D_X of chunk kk - 1 have been drained
                if (!mbar_wait(full0 + 8 * st, (kk / kStages) & 1) ||
                    (kk > 0 && !mbar_wait(sdrain, (kk - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks) umma_bf16(tm, seg_u_desc(stage, ks), seg_kres_desc(stage, ks), idSU, ks > 0);
                if (!mbar_wait(sready0 + 8 * b, (kk >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t bm = seg_m_desc(stage, ks);
                    umma_bf16_tmem_a(tm, tm + kSTi + 64 * b + 8 * ks, bm, idSS, 1);
                    umma_bf16_tmem_a(tm + kDX, tm + kXTi + 64 * b + 8 * ks, bm, idSS, ks > 0);
                }
                umma_commit(mmas);
                umma_commit(empty0 + 8 * st);
            }
            if (!ok) {
                kda_set_status(KDA_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(finbar);
            mbar_wait(finbar, 0);
        }
    } else {
        const int q4 = warp & 3, j = 32 * q4 + lane, c = warp >> 2;
        const uint32_t lanes = (uint32_t)(32 * q4) << 16;
        float Sr[64], Xr[64];
#pragma unroll
        for (int u = 0; u < 64; ++u) {
            Sr[u] = 0.f;
            Xr[u] = (64 * c + u == j) ? 1.f : 0.f;
        }
        auto put = [&](int b) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t r[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) r[u] = pack_bf16x2(Sr[32 * hf + 2 * u], Sr[32 * hf + 2 * u + 1]);
                tmem_st16(tm + lanes + kSTi + 64 * b + 32 * c + 16 * hf, r);
#pragma unroll
                for (int u = 0; u < 16; ++u) r[u] = pack_bf16x2(Xr[32 * hf + 2 * u], Xr[32 * hf + 2 * u + 1]);
                tmem_st16(tm + lanes + kXTi + 64 * b + 32 * c + 16 * hf, r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sready0 + 8 * b);
        };
        if (nchunks > 0) put(0);
        bool ok = true;
        for (int kk = 0; kk < nchunks; ++kk) {
            const int st = kk % kStages;
            ok = __all_sync(0xffffffffu, mbar_wait(mmas, kk & 1));
            if (!ok || *abort_flag) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float4* gam = reinterpret_cast<const float4*>(sm + st * S::kStage + kRecGamma) + 16 * c;
            // x[16 q ..] = gamma x + D for one 16-column quarter of D_S (into Sr) or D_X (into Xr);
            // quarters keep the live registers within the 168 a 320-thread CTA may use
            auto update = [&](float(&x)[64], uint32_t dcol, int qt) {
                float d[16];
                tmem_ld16(tm + lanes + dcol + 64 * c + 16 * qt, d);
                tmem_wait_ld();
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    const float4 g4 = gam[4 * qt + u4];
                    x[16 * qt + 4 * u4 + 0] = fmaf(g4.x, x[16 * qt + 4 * u4 + 0], d[4 * u4 + 0]);
                    x[16 * qt + 4 * u4 + 1] = fmaf(g4.y, x[16 * qt + 4 * u4 + 1], d[4 * u4 + 1]);
                    x[16 * qt + 4 * u4 + 2] = fmaf(g4.z, x[16 * qt + 4 * u4 + 2], d[4 * u4 + 2]);
                    x[16 * qt + 4 * u4 + 3] = fmaf(g4.w, x[16 * qt + 4 * u4 + 3], d[4 * u4 + 3]);
                }
            };
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) update(Sr, 0u, qt);
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) update(Xr, kDX, qt);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(sdrain);
                mbar_arrive(empty0 + 8 * st);   // gamma of this stage read
            }
            if (kk + 1 < nchunks) put((kk + 1) & 1);
        }
        if (!ok) {
            if (lane == 0) kda_set_status(KDA_ERR_TIMEOUT);
            *abort_flag = 1;
        } else {
            float* dst = seg_states + ((size_t)sgi * H + h) * (kSegStateBytes / sizeof(float));
#pragma unroll
            for (int u = 0; u < 64; ++u) {
                dst[(size_t)(64 * c + u) * D + j] = Sr[u];            // S_local[i][j]
                dst[D * D + (size_t)(64 * c + u) * D + j] = Xr[u];    // T[i][j] = X[j][i]
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, kSegTmemCols);
    }
}

// The segments' starting states along each sequence, S_in(p+1) = T_p S_in(p) + S_local(p)
// from S_in(0) = the initial state (or 0), in fp32 on CUDA cores; S_in(p) is stored for
// p > 0.  One CTA of 512 threads per (sequence, head), S_in(p) in shared memory (64 KB).
constexpr int kCombineThreads = 512;
constexpr size_t kCombineSmem = sizeof(float) * D * D;
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(int H, const float* __restrict__ initial_state, const int32_t* __restrict__ seg_off,
               float* __restrict__ seg_states, int din) {
    extern __shared__ __align__(16) float sS[];
    const int h = blockIdx.x % H, n = blockIdx.x / H, tid = threadIdx.x;
    const int s0 = seg_off[n], ns = seg_off[n + 1] - s0;
    if (ns <= 1) return;
    constexpr size_t kWords = kSegStateBytes / sizeof(float);
    for (int e = tid; e < D * D; e += kCombineThreads) {   // the caller's din x din state, top left
        const int r = e / D, c = e % D;
        sS[e] = initial_state && r < din && c < din ? initial_state[((size_t)n * H + h) * din * din + r * din + c]
                                                    : 0.f;
    }
    __syncthreads();
    // thread: row i = tid / 4, columns j = tid % 4 + 4 z (z < 32)
    const int i = tid >> 2, j0 = tid & 3;
    for (int p = 0; p + 1 < ns; ++p) {
        const float* seg = seg_states + ((size_t)(s0 + p) * H + h) * kWords;
        const float* Trow = seg + D * D + (size_t)i * D;
        float acc[32];
#pragma unroll
        for (int z = 0; z < 32; ++z) acc[z] = seg[(size_t)i * D + j0 + 4 * z];   // S_local
        for (int kx = 0; kx < D; ++kx) {
            const float t = Trow[kx];
#pragma unroll
            for (int z = 0; z < 32; ++z) acc[z] = fmaf(t, sS[kx * D + j0 + 4 * z], acc[z]);
        }
        __syncthreads();   // every read of S_in(p) done
        float* dst = seg_states + ((size_t)(s0 + p + 1) * H + h) * kWords + 2 * D * D;
#pragma unroll
        for (int z = 0; z < 32; ++z) {
            sS[i * D + j0 + 4 * z] = acc[z];
            dst[(size_t)i * D + j0 + 4 * z] = acc[z];
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ launch
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; a function-local static is initialised exactly once even when several
// host threads make their first call at the same time.
inline EncodeTiledFn encode_tiled() {
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

// Rows = tokens (T), columns = H*D elements; box = 64 tokens x `box_cols` columns.
inline bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, size_t elem,
                      int64_t T, int H, uint32_t box_cols, CUtensorMapSwizzle sw, int din = D) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)H * din, (cuuint64_t)T};
    const cuuint64_t strides[1] = {(cuuint64_t)H * din * elem};
    const cuuint32_t box[2] = {box_cols, (cuuint32_t)C};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Workspace {
    int32_t* off;
    int2* tab;
    int32_t* etab;
    int32_t* strong_count;
    int2* strong_units;
    int seg;                 // chunks per scan segment, 0 without segments
    int64_t max_segs;
    int32_t* seg_off;
    int32_t* seg_count;
    int4* seg_tab;
    float* seg_states;
    uint8_t* records;
};
inline Workspace split_workspace(void* workspace, int64_t total, int num_seqs, int H) {
    uint8_t* base = static_cast<uint8_t*>(workspace);
    uint8_t* strong = base + ws_strong_offset(total, num_seqs);
    Workspace w{reinterpret_cast<int32_t*>(base), reinterpret_cast<int2*>(base + ws_table_offset(num_seqs)),
                reinterpret_cast<int32_t*>(base + ws_emit_offset(total, num_seqs)),
                reinterpret_cast<int32_t*>(strong), reinterpret_cast<int2*>(strong + 16),
                scan_segment_chunks(total, num_seqs, H), 0, nullptr, nullptr, nullptr, nullptr,
                base + ws_records_offset(total, num_seqs, H)};
    if (w.seg > 0) {
        uint8_t* sc = base + ws_scan_offset(total, num_seqs, H);
        w.max_segs = max_segments(total, num_seqs, w.seg);
        w.seg_off = reinterpret_cast<int32_t*>(sc);
        sc += align_up(sizeof(int32_t) * (num_seqs + 1), 16);
        w.seg_count = reinterpret_cast<int32_t*>(sc);
        w.seg_tab = reinterpret_cast<int4*>(sc + 16);
        w.seg_states = reinterpret_cast<float*>(sc + 16 + align_up(sizeof(int4) * w.max_segs, 1024));
    }
    return w;
}

// SMs of the current device (cached per device; 0 when the query fails).  Host threads
// may race on the first query of a device: they store the same value, atomically.
// Launch with programmatic stream serialization: the kernel's blocks may be scheduled while
// the kernel ahead of it in the stream is still running; they wait for it in kda_grid_wait.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline int device_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Chunk table (+ emission slots when emit_pos is given) + chunk-parallel preparation, then
// the CUDA-core preparation of the chunks prep_kernel listed for their strong decay.
// What the preparation of any range of chunks needs: the inputs, their tensor maps and the
// chunk table.
struct PrepInputs {
    CUtensorMap tq, tk, tv, tg;
    const void *q, *k, *v;
    const float *g, *beta;
    int num_seqs, H;
    int64_t total;
    const int32_t* off;
    const int2* tab;
    uint32_t in_flags;
    int din;   // channels per head of q, k, v, g: 128 or 64
};
inline cudaError_t make_prep_inputs(PrepInputs* p, const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, int num_seqs, int64_t total, int H, const Workspace& w,
                                    uint32_t in_flags, int din) {
    const bool g_scalar = (in_flags & kInGScalar) != 0;
    *p = PrepInputs{};
    p->q = q; p->k = k; p->v = v; p->g = g; p->beta = beta;
    p->num_seqs = num_seqs; p->H = H; p->total = total; p->off = w.off; p->tab = w.tab; p->in_flags = in_flags;
    p->din = din;
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_tmap(&p->tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64, sw, din) ||
        !make_tmap(&p->tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64, sw, din) ||
        !make_tmap(&p->tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64, sw, din) ||
        (!g_scalar && !make_tmap(&p->tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, total, H, (uint32_t)din,
                                 CU_TENSOR_MAP_SWIZZLE_NONE, din)))
        return cudaErrorInvalidValue;
    if (g_scalar) p->tg = p->tq;   // a scalar gate is read with plain loads: this map goes unused
    return cudaSuccess;
}
// Prepares chunks c_base .. c_base + nchunks - 1 (those that exist) into records[0 ..]:
// the tensor-core preparation, then the CUDA-core one for the chunks it listed in
// (count, list), which the chunk-table kernel zeroed.
inline cudaError_t launch_prep_chunks(const PrepInputs& p, int64_t c_base, int64_t nchunks, uint8_t* records,
                                      int32_t* count, int2* list, cudaStream_t stream) {
    const bool g_scalar = (p.in_flags & kInGScalar) != 0;
    const bool pro = (p.in_flags & (kInNormQK | kInGLogits | kInBetaLogits)) != 0;
    const bool d64 = p.din == 64;
    auto prep = d64 ? (g_scalar ? (pro ? prep_kernel<true, true, 64> : prep_kernel<true, false, 64>)
                                : (pro ? prep_kernel<false, true, 64> : prep_kernel<false, false, 64>))
                    : (g_scalar ? (pro ? prep_kernel<true, true, 128> : prep_kernel<true, false, 128>)
                                : (pro ? prep_kernel<false, true, 128> : prep_kernel<false, false, 128>));
    auto strong = d64 ? (g_scalar ? prep_strong_kernel<true, 64> : prep_strong_kernel<false, 64>)
                      : (g_scalar ? prep_strong_kernel<true, 128> : prep_strong_kernel<false, 128>);
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PrepSmem::BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(strong, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StrongSmem::BYTES);
    if (e != cudaSuccess) return e;
    e = launch_after(prep, dim3((unsigned)(nchunks * p.H)), dim3(kPrepThreads), PrepSmem::BYTES, stream,
                     p.tq, p.tk, p.tv, p.tg, g_scalar ? p.g : nullptr, p.beta, p.num_seqs, p.H, p.off, p.tab,
                     records, count, list, p.in_flags, p.total, (int)c_base);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    const int64_t sgrid = std::min<int64_t>(nchunks * p.H, sms > 0 ? sms : 148);
    return launch_after(strong, dim3((unsigned)sgrid), dim3(kStrongThreads), StrongSmem::BYTES, stream,
                        static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
                        static_cast<const __nv_bfloat16*>(p.v), p.g, p.beta, p.num_seqs, p.H, p.tab, records,
                        (const int32_t*)count, (const int2*)list, p.in_flags, p.total, (int)c_base);
}

// The recurrence for `chains` (sequence or segment, head) chains of head width din: value
// slices of 32 columns while all their CTAs fit on the SMs at once, else of 64.
struct RecLaunch {
    void (*kernel)(int, int, const int32_t*, const int2*, const uint8_t*, const float*, float*,
                   __nv_bfloat16*, const int32_t*, float*, const int4*, const int32_t*, const float*,
                   RecWindow);
    uint32_t smem;
    int nsl;   // CTAs per chain
};
// ordered: sequences taken longest first (several sequences, no scan segments).
inline RecLaunch pick_rec(int64_t chains, int din, bool ordered) {
    const int sms = device_sm_count();
    const bool narrow = chains * (din / 32) <= (int64_t)(sms > 0 ? sms : 148);
    if (din == 64) {
        if (ordered)
            return narrow ? RecLaunch{rec_kernel<32, 64, true>, RecCfg<32>::BYTES, 2}
                          : RecLaunch{rec_kernel<64, 64, true>, RecCfg<64>::BYTES, 1};
        return narrow ? RecLaunch{rec_kernel<32, 64, false>, RecCfg<32>::BYTES, 2}
                      : RecLaunch{rec_kernel<64, 64, false>, RecCfg<64>::BYTES, 1};
    }
    if (ordered)
        return narrow ? RecLaunch{rec_kernel<32, 128, true>, RecCfg<32>::BYTES, 4}
                      : RecLaunch{rec_kernel<64, 128, true>, RecCfg<64>::BYTES, 2};
    return narrow ? RecLaunch{rec_kernel<32, 128, false>, RecCfg<32>::BYTES, 4}
                  : RecLaunch{rec_kernel<64, 128, false>, RecCfg<64>::BYTES, 2};
}

inline cudaError_t launch_prepare(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu, int num_seqs,
                                  int64_t total, int H, void* workspace, cudaStream_t stream,
                                  const int64_t* emit_pos = nullptr, int num_emit = 0,
                                  uint32_t in_flags = 0, int din = D) {
    const Workspace w = split_workspace(workspace, total, num_seqs, H);
    chunk_index_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total, w.off, w.tab,
                                               num_emit > 0 ? w.etab : nullptr, w.strong_count, 1);
    if (num_seqs > 1) {
        const cudaError_t e0 = launch_after(order_kernel, dim3(1), dim3(1024), (uint32_t)order_smem_bytes(num_seqs),
                                            stream, w.off, num_seqs);
        if (e0 != cudaSuccess) return e0;
    }
    if (num_emit > 0)
        emit_index_kernel<<<(num_emit + 255) / 256, 256, 0, stream>>>(cu, num_seqs, w.off, emit_pos,
                                                                       num_emit, w.etab);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || total == 0) return e;
    PrepInputs p;
    e = make_prep_inputs(&p, q, k, v, g, beta, num_seqs, total, H, w, in_flags, din);
    if (e != cudaSuccess) return e;
    return launch_prep_chunks(p, 0, max_chunks(total, num_seqs), w.records, w.strong_count, w.strong_units, stream);
}

inline cudaError_t launch_scan(const float* s0, float* sf, void* out, int num_seqs, int64_t total,
                               int H, void* workspace, cudaStream_t stream,
                               float* emit_states = nullptr, uint32_t in_flags = 0, int din = D) {
    const Workspace w = split_workspace(workspace, total, num_seqs, H);
    if ((int64_t)num_seqs * H == 0) return cudaSuccess;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    const int32_t* et = emit_states ? w.etab : nullptr;
    const bool scan = w.seg > 0 && !(in_flags & kInSerialChains);
    const int64_t units = scan ? w.max_segs : num_seqs;   // chains: sequences, or scan segments
    const RecLaunch rl = pick_rec(units * H, din, !scan && num_seqs > 1);
    auto rec = rl.kernel;
    const uint32_t rec_smem = rl.smem;
    const int nsl = rl.nsl;
    cudaError_t e = cudaFuncSetAttribute(rec, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rec_smem);
    if (e != cudaSuccess) return e;
    if (!scan)
        return launch_after(rec, dim3((unsigned)(num_seqs * H * nsl)), dim3(kRecThreads), rec_smem, stream,
                            num_seqs, H, (const int32_t*)w.off, (const int2*)w.tab, (const uint8_t*)w.records, s0,
                            sf, o, et, emit_states, (const int4*)nullptr, (const int32_t*)nullptr,
                            (const float*)nullptr, kWholeProblem);
    e = cudaFuncSetAttribute(seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SegSmem::BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCombineSmem);
    if (e != cudaSuccess) return e;
    segment_index_kernel<<<1, 1024, 0, stream>>>(num_seqs, w.off, w.seg, w.seg_off, w.seg_count, w.seg_tab);
    seg_kernel<<<(unsigned)(w.max_segs * H), kSegThreads, SegSmem::BYTES, stream>>>(H, w.records, w.seg_tab,
                                                                                    w.seg_count, w.seg_states);
    combine_kernel<<<(unsigned)num_seqs * H, kCombineThreads, kCombineSmem, stream>>>(H, s0, w.seg_off, w.seg_states,
                                                                                   din);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_after(rec, dim3((unsigned)(w.max_segs * H * nsl)), dim3(kRecThreads), rec_smem, stream,
                        num_seqs, H, (const int32_t*)w.off, (const int2*)w.tab, (const uint8_t*)w.records, s0, sf,
                        o, et, emit_states, (const int4*)w.seg_tab, (const int32_t*)w.seg_count,
                        (const float*)w.seg_states, kWholeProblem);
}

// The whole prefill.  window: chunks per window when the workspace holds fewer records than
// the problem has chunks (window_chunks); the chunk-parallel scan runs only in one window.
inline cudaError_t launch_prefill(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const float* s0, const int32_t* cu,
                                  int num_seqs, int64_t total, int H, void* out, float* sf,
                                  void* workspace, cudaStream_t stream,
                                  const int64_t* emit_pos = nullptr, int num_emit = 0,
                                  float* emit_states = nullptr, uint32_t in_flags = 0,
                                  int64_t window = INT64_MAX, int din = D) {
    const int64_t mc = max_chunks(total, num_seqs);
    if (window >= mc) {
        cudaError_t e = launch_prepare(q, k, v, g, beta, cu, num_seqs, total, H, workspace, stream,
                                       emit_pos, num_emit, in_flags, din);
        if (e == cudaSuccess)
            e = launch_scan(s0, sf, out, num_seqs, total, H, workspace, stream,
                            num_emit > 0 ? emit_states : nullptr, in_flags, din);
        return e;
    }
    if (window <= 0 || num_seqs == 0) return cudaErrorInvalidValue;
    const Workspace w = split_workspace(workspace, total, num_seqs, H);   // chunk offsets, table, slots
    const WindowLayout l = window_layout(total, num_seqs, H, window);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int32_t* counts = reinterpret_cast<int32_t*>(base + l.counts);
    int2* list = reinterpret_cast<int2*>(base + l.list);
    float* carry = reinterpret_cast<float*>(base + l.carry);
    uint8_t* records = base + l.records;
    const int64_t nw = (mc + window - 1) / window;
    chunk_index_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total, w.off, w.tab,
                                               num_emit > 0 ? w.etab : nullptr, counts, (int)nw);
    if (num_seqs > 1) {
        const cudaError_t e0 = launch_after(order_kernel, dim3(1), dim3(1024), (uint32_t)order_smem_bytes(num_seqs),
                                            stream, w.off, num_seqs);
        if (e0 != cudaSuccess) return e0;
    }
    if (num_emit > 0)
        emit_index_kernel<<<(num_emit + 255) / 256, 256, 0, stream>>>(cu, num_seqs, w.off, emit_pos,
                                                                       num_emit, w.etab);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    PrepInputs p;
    if (total > 0 && (e = make_prep_inputs(&p, q, k, v, g, beta, num_seqs, total, H, w, in_flags, din)) != cudaSuccess)
        return e;
    const RecLaunch rl = pick_rec((int64_t)num_seqs * H, din, num_seqs > 1);
    auto rec = rl.kernel;
    const uint32_t rec_smem = rl.smem;
    const int nsl = rl.nsl;
    if ((e = cudaFuncSetAttribute(rec, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rec_smem)) != cudaSuccess)
        return e;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    const size_t slot = (size_t)H * din * din;   // one carried state per head
    for (int64_t wi = 0; wi < nw; ++wi) {
        const int64_t c_lo = wi * window;
        if (total > 0 && (e = launch_prep_chunks(p, c_lo, window, records, counts + wi, list, stream)) != cudaSuccess)
            return e;
        const RecWindow rw = {(int)c_lo, (int)std::min<int64_t>(c_lo + window, INT32_MAX), wi == nw - 1 ? 1 : 0,
                              carry + (size_t)(wi & 1) * slot, carry + (size_t)((wi + 1) & 1) * slot};
        e = launch_after(rec, dim3((unsigned)(num_seqs * H * nsl)), dim3(kRecThreads), rec_smem, stream, num_seqs,
                         H, (const int32_t*)w.off, (const int2*)w.tab, (const uint8_t*)records, s0, sf, o,
                         (const int32_t*)(num_emit > 0 ? w.etab : nullptr), num_emit > 0 ? emit_states : nullptr,
                         (const int4*)nullptr, (const int32_t*)nullptr, (const float*)nullptr, rw);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// One thread waits (bounded) on a barrier nothing arrives on and reports the expiry.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar_storage;
    if (threadIdx.x == 0) {
        const uint32_t bar = smem_u32(&bar_storage);
        mbar_init(bar, 1);
        fence_mbar_init();
        if (!mbar_wait(bar, 0, limit_ns)) kda_set_status(KDA_ERR_TIMEOUT);
    }
}

}  // namespace tc
}  // namespace kda
