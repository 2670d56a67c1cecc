// fa_internal.h -- declarations shared by the host ABI (fa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/fa.h"

namespace fa {

// Device error-flag codes mirror fa_status.
constexpr int kErrInvalidArg = FA_ERR_INVALID_ARG;
constexpr int kErrTimeout = FA_ERR_TIMEOUT;

// Element counts of the buffers a call's kernels touch with plain loads and stores (TMA
// accesses are bounded by their tensor maps).  Filled by the host on every call; only builds
// with FA_DEBUG defined read them: there every such access checks its index first (in_bounds).
struct Extents {
    size_t q;          // q, o, dO, dq
    size_t kv;         // k, v, dk, dv
    size_t lse;        // lse
    size_t vec;        // the backward's per-row workspace vectors D and |dO|
    size_t acc;        // fixed-point dQ accumulator
    size_t hmax;       // per-chunk bound maxima
    size_t part;       // decode partial outputs (fp32 rows of d); partial lse: part / d
    int nseq;          // entries of seqlens / cache_lens (B) or of cu_seqlens (B + 1)
    int heads_q;       // entries of the FP8 q descale array (B * H)
    int heads_kv;      // entries of the FP8 k, v descale arrays (B * H_kv)
};

// Extents of the attention buffers (head-major [B, H, N, d] or packed [T, H, d]) and of the
// backward workspace carved for them.
inline Extents extents(int B, int H, int H_kv, int N, int d, int T, bool packed) {
    Extents e{};
    const size_t Np = ((size_t)N + 127) / 128 * 128;
    e.q = packed ? (size_t)T * H * d : (size_t)B * H * N * d;
    e.kv = packed ? (size_t)T * H_kv * d : (size_t)B * H_kv * N * d;
    e.lse = packed ? (size_t)H * T : (size_t)B * H * N;
    e.vec = (size_t)B * H * N;  // [B, H, N] in both layouts (N = the longest sequence)
    e.acc = (size_t)B * H * Np * d;
    e.hmax = (size_t)B * H * (Np / 128) * 2;
    e.part = 0;
    e.nseq = packed ? B + 1 : B;
    e.heads_q = B * H;
    e.heads_kv = B * H_kv;
    return e;
}

// Two layouts of the user tensors.
//   head-major: q, o, dO, dq [B, H, N, d]; k, v, dk, dv [B, H_kv, N, d]; lse [B, H, N].
//   packed (cu_seqlens != nullptr): sequence b is rows [cu[b], cu[b+1]) of q, o, dO, dq
//     [T, H, d] and of k, v, dk, dv [T, H_kv, d]; lse is [H, T]; N is the longest sequence.
struct FwdParams {
    void* o;               // bf16 [B, H, N, d] or packed [T, H, d]
    float* lse;            // fp32 [B, H, N] or packed [H, T]
    const int* seqlens;    // device int32 [B] key lengths (head-major only) or nullptr
    const int* cu_seqlens; // device int32 [B + 1] packed sequence offsets or nullptr
    int T;                 // packed: rows of the packed tensors
    int* err;              // device error flag
    int B, H, N;
    int H_kv;              // key/value heads; query head h reads K/V head h / (H / H_kv)
    float scale_log2;      // scale * log2(e)
    int causal;
    uint64_t timeout_ns;
    Extents dbg;
};

struct BwdParams {
    const void* o;         // bf16 [B, H, N, d]
    const void* dO;        // bf16 [B, H, N, d]
    const float* lse;      // fp32 [B, H, N]
    const void* k;         // bf16 [B, H, N, d] (read by the preprocess kernel for its bound)
    const void* v;         // bf16 [B, H, N, d]
    void* dq;              // bf16 out
    void* dk;              // bf16 out
    void* dv;              // bf16 out
    float* Dvec;           // fp32 [B, H, N]            workspace: rowsum(dO * O)
    float* dOnorm;         // fp32 [B, H, N]            workspace: |dO_i|_2
    float* headmax;        // fp32 [B, H, N_pad/128, 2] workspace: per-chunk max |v_j|_2, max |k_jl|
    int* dq_acc;           // int32 [B, H, N_pad, d]    workspace: fixed-point dQ accumulator
    const int* seqlens;
    const int* cu_seqlens; // packed layout (see FwdParams); the workspace stays [B, H, N_pad]
    int T;
    int* err;
    int B, H, N, N_pad;
    int H_kv;              // key/value heads (H % H_kv == 0); dK, dV are [B, H_kv, N, d]
    float scale;
    float scale_log2;
    int causal;
    uint64_t timeout_ns;
    int num_sms;           // SMs of the device (the persistent grid); 0: one CTA per key block
    Extents dbg;
};

#ifdef __CUDACC__
#ifdef FA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Debug builds (FA_DEBUG): true when elements [i, i + width) lie inside a buffer of n
// elements; otherwise FA_ERR_INVALID_ARG is recorded in `err` and the caller skips the access
// (nothing traps).  Release builds: always true, and the check compiles away.
__device__ __forceinline__ bool in_bounds(int* err, size_t i, size_t width, size_t n) {
    if constexpr (!kDebugChecks) {
        return true;
    } else {
        if (i + width <= n) return true;
        if (err) atomicCAS(err, 0, kErrInvalidArg);
        return false;
    }
}

// Where sequence b lives.  Head-major: rows [0, N) of its heads, keys valid below L (the key
// length, N without seqlens).  Packed: rows [t0, t0 + L) and queries and keys both end at L;
// offsets that do not describe rows inside [0, T) with L <= N are reported through the error
// flag and the sequence is treated as empty (nothing read, nothing written).
struct SeqExtent {
    int t0;   // first packed row (0 head-major)
    int L;    // valid keys
    int Lq;   // query rows that exist (N head-major, L packed)
};

// `packed` must equal (p.cu_seqlens != nullptr); kernels compiled for one layout pass it as a
// constant so that the other layout's state drops out.
template <class P>
__device__ __forceinline__ SeqExtent sequence_extent(const P& p, int b, bool report,
                                                     bool packed) {
    SeqExtent e{0, p.N, p.N};
    if (packed) {
        if (!in_bounds(p.err, (size_t)b, 2, (size_t)p.dbg.nseq)) {
            e.L = e.Lq = 0;
            return e;
        }
        const int t0 = p.cu_seqlens[b], t1 = p.cu_seqlens[b + 1];
        if (t0 < 0 || t1 < t0 || t1 - t0 > p.N || t1 > p.T) {
            if (report) atomicCAS(p.err, 0, kErrInvalidArg);
            e.t0 = 0;
            e.L = e.Lq = 0;
        } else {
            e.t0 = t0;
            e.L = e.Lq = t1 - t0;
        }
    } else if (p.seqlens != nullptr) {
        if (!in_bounds(p.err, (size_t)b, 1, (size_t)p.dbg.nseq)) return e;
        int L = p.seqlens[b];
        if (L < 1 || L > p.N) {
            if (report) atomicCAS(p.err, 0, kErrInvalidArg);
            L = L < 1 ? 1 : p.N;
        }
        e.L = L;
    }
    return e;
}

// Row (in units of d elements) of position n of head hx (of Hx heads) of sequence b.
__device__ __forceinline__ size_t row_of(bool packed, int b, int hx, int Hx, int N, int t0,
                                         int n) {
    return packed ? (size_t)(t0 + n) * Hx + hx : ((size_t)b * Hx + hx) * N + n;
}
// Index of the lse entry of query position n of head h (of H heads) of sequence b.
__device__ __forceinline__ size_t lse_of(bool packed, int b, int h, int H, int N, int T, int t0,
                                         int n) {
    return packed ? (size_t)h * T + t0 + n : ((size_t)b * H + h) * N + n;
}
#endif

// Current bound on device-side waits (fa_set_wait_timeout_ns).
uint64_t wait_timeout_ns();

// Raises the dynamic shared-memory limit of each of `kernels` to `bytes` on the current
// device, once per device: the attribute belongs to the device's context, so a process that
// uses several GPUs sets it on each.  `done` keeps one bit per device (devices 0-63).  Several
// host threads may race here harmlessly: setting the attribute twice is idempotent.
template <class... Kernel>
cudaError_t set_smem_limit_once(std::atomic<uint64_t>& done, int bytes, Kernel... kernels) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    for (const void* k : {reinterpret_cast<const void*>(kernels)...}) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
    }
    done.fetch_or(bit, std::memory_order_acq_rel);
    return cudaSuccess;
}

// Tensor maps: a bf16 [B*H, N, d] tensor seen as 3-D (d, N, B*H), 128-byte swizzle,
// box = 64 columns x `box_rows` rows; rows past N read as zeros.
bool make_bf16_map(CUtensorMap* map, const void* base, int d, int N, int BH, int box_rows);
// A packed bf16 [T, Hx, d] tensor seen as 3-D (d, Hx, T), box = 64 columns x 1 head x
// `box_rows` rows (the same 128-byte-swizzled shared tile); rows past T read as zeros.
// Coordinates are (column, head, row).
bool make_bf16_map_packed(CUtensorMap* map, const void* base, int d, int Hx, int T, int box_rows);

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int B, int num_sms, cudaStream_t stream);

// ev_start / ev_stop (optional) are recorded on `stream` right before and after the fused
// backward kernel (between the preprocess and the dQ convert kernels).
cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream,
                       cudaEvent_t ev_start = nullptr, cudaEvent_t ev_stop = nullptr);

}  // namespace fa
