// fa_api.cu -- host side of the C ABI declared in include/fa.h: argument validation, tensor
// maps, the per-device error flag and kernel launches.  No compute happens here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "fa_decode.h"
#include "fa_fwd_fp8.h"
#include "fa_internal.h"

namespace fa {

// fa_fwd_d256.cu: head dimension 256 (forward only).
cudaError_t launch_fwd_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int B, cudaStream_t stream);

namespace {

constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_timeout_ns{4000000000ull};

// fa_set_kernel_timing_events: consumed by the next entry point called on this host thread.
thread_local cudaEvent_t t_ev_start = nullptr;
thread_local cudaEvent_t t_ev_stop = nullptr;

void take_timing_events(cudaEvent_t* start, cudaEvent_t* stop) {
    *start = t_ev_start;
    *stop = t_ev_stop;
    t_ev_start = t_ev_stop = nullptr;
}

struct DeviceState {
    bool probed = false;
    bool supported = false;
    int num_sms = 0;
    int* err_flag = nullptr;  // 4-byte device buffer
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return g_encode;
}

// Returns the current device's state, probing it (and allocating its error flag) once.
DeviceState* current_device(fa_status* st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = FA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& s = g_dev[dev];
    if (!s.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            *st = FA_ERR_CUDA;
            return nullptr;
        }
        s.supported = (major == 10 && minor == 0);
        s.num_sms = sms;
        if (s.supported) {
            if (cudaMalloc(&s.err_flag, sizeof(int)) != cudaSuccess ||
                cudaMemset(s.err_flag, 0, sizeof(int)) != cudaSuccess) {
                *st = FA_ERR_CUDA;
                return nullptr;
            }
        }
        s.probed = true;
    }
    if (!s.supported) {
        *st = FA_ERR_UNSUPPORTED;
        return nullptr;
    }
    *st = FA_OK;
    return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int H, int N, int d, float scale) {
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return FA_ERR_INVALID_ARG;
    const long long elems = (long long)B * H * N * d;
    if (elems >= (1ll << 31)) return FA_ERR_INVALID_ARG;
    return FA_OK;
}

int pad128(int N) { return (N + 127) / 128 * 128; }

}  // namespace

uint64_t wait_timeout_ns() { return g_timeout_ns.load(); }

bool make_bf16_map(CUtensorMap* map, const void* base, int d, int N, int BH, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_map_packed(CUtensorMap* map, const void* base, int d, int Hx, int T, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)Hx, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)Hx * d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_fp8_map(CUtensorMap* map, const void* base, int N, int BHx) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)N, (cuuint64_t)BHx};
    cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// Tensor map of a user tensor with Hx heads: head-major [B, Hx, N, d] or packed [T, Hx, d];
// boxes of 64 columns x `rows` rows.
bool user_map(CUtensorMap* map, const void* base, int d, int B, int Hx, int N, int T,
              bool packed, int rows = 128) {
    return packed ? make_bf16_map_packed(map, base, d, Hx, T, rows)
                  : make_bf16_map(map, base, d, N, B * Hx, rows);
}

// Checks shared by the head-major and packed entry points; T = 0 for head-major.
fa_status check_layout(int B, int H, int H_kv, int N, int d, float scale, const int* seqlens,
                       const int* cu_seqlens, int T, bool fwd) {
    (void)fwd;  // every head dim has both passes in both layouts
    fa_status st = check_common(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (H_kv < 1 || H_kv > H || H % H_kv != 0) return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return FA_ERR_INVALID_ARG;
        if (T < 1 || (long long)T * H * d >= (1ll << 31)) return FA_ERR_INVALID_ARG;
    }
    return FA_OK;
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int H_kv, int N, int d, float scale, int causal, const int* seqlens,
                   const int* cu_seqlens, int T, cudaStream_t stream) {
    fa_status st = check_layout(B, H, H_kv, N, d, scale, seqlens, cu_seqlens, T, true);
    if (st != FA_OK) return st;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;

    const bool packed = cu_seqlens != nullptr;
    CUtensorMap tq, tk, tv;
    if (!user_map(&tq, q, d, B, H, N, T, packed) || !user_map(&tk, k, d, B, H_kv, N, T, packed) ||
        !user_map(&tv, v, d, B, H_kv, N, T, packed))
        return FA_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.seqlens = seqlens;
    p.cu_seqlens = cu_seqlens;
    p.T = T;
    p.err = dev->err_flag;
    p.B = B;
    p.H = H;
    p.N = N;
    p.H_kv = H_kv;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.timeout_ns = g_timeout_ns.load();
    p.dbg = extents(B, H, H_kv, N, d, T, packed);
    cudaEvent_t ev0, ev1;
    take_timing_events(&ev0, &ev1);
    if (ev0) cudaEventRecord(ev0, stream);
    const cudaError_t e = d == 256 ? launch_fwd_d256(tq, tk, tv, p, B, stream)
                                   : launch_fwd(d, tq, tk, tv, p, B, dev->num_sms, stream);
    if (ev1) cudaEventRecord(ev1, stream);
    if (e != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

// Split-KV decode: the number of key ranges that minimises (waves of CTAs) x (key blocks per
// CTA + 3 for its fixed cost: start-up, the first loads' latency, the epilogue), preferring
// fewer ranges on ties.  `bk` keys per block, `slots` CTAs resident per wave.  The constant is
// measured: over split counts of 1 to 64 on five cache shapes it picks the fastest one each
// time (one block of fixed cost picked up to 9 % slower counts).
// With per-sequence lengths (`ragged`, known only on the device) the waves model overrates a
// few long ranges, because the short sequences' CTAs finish early; there the count is at least
// ceil(4 slots / pairs), which keeps the longest range near half of one slot's share of the
// work when lengths average N / 2 (on four ragged batches this lands on or next to the fastest
// count; the waves model alone was up to 1.6x slower).
int decode_splits(int B, int H_kv, int n_mt, int N, int bk, int slots, bool ragged) {
    const int nblk = (N + bk - 1) / bk;
    const long long base = (long long)B * H_kv * n_mt;
    int best = 1;
    long long best_cost = -1;
    for (int s = 1; s <= nblk && s <= 256; ++s) {
        const int bps = (nblk + s - 1) / s;
        if ((nblk + bps - 1) / bps != s) continue;  // same ranges as a smaller s
        const long long waves = (base * s + slots - 1) / slots;
        const long long cost = waves * (bps + 3);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    if (ragged) {
        const long long floor_s = (4LL * slots + base - 1) / base;
        if (best < floor_s) best = (int)(floor_s < nblk ? floor_s : nblk);
    }
    return best;
}

fa_status check_decode(int B, int H, int H_kv, int Nq, int N, int d, float scale, int splits) {
    if (B < 1 || H < 1 || H_kv < 1 || Nq < 1 || N < 1 || splits < 0) return FA_ERR_INVALID_ARG;
    if (H % H_kv != 0 || B > 65535 || H > 65535) return FA_ERR_INVALID_ARG;
    if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if ((long long)B * H * Nq * d >= (1ll << 31) || (long long)B * H_kv * N * d >= (1ll << 31))
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}

}  // namespace
}  // namespace fa

using namespace fa;

namespace fa {
// fa_selftest.cu
cudaError_t launch_wait_selftest(int* err, uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_bounds_selftest(int* buf, int n, int value, int* err, cudaStream_t stream);
}  // namespace fa

extern "C" {

const char* fa_status_string(fa_status s) {
    switch (s) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim or device";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call failed";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait timed out";
        case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    }
    return "unknown fa_status";
}

void fa_set_kernel_timing_events(void* start_event, void* stop_event) {
    t_ev_start = static_cast<cudaEvent_t>(start_event);
    t_ev_stop = static_cast<cudaEvent_t>(stop_event);
}

void fa_set_wait_timeout_ns(uint64_t ns) {
    g_timeout_ns.store(ns < 1000000ull ? 1000000ull : ns);
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int H_kv, int N, int d, float scale, int causal, const int* seqlens,
                     fa_stream_t stream) {
    return fwd_impl(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, seqlens, nullptr, 0,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int H, int H_kv,
                        int d, float scale, int causal, fa_stream_t stream) {
    if (!cu_seqlens) return FA_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, o, lse, B, H, H_kv, max_seqlen, d, scale, causal, nullptr,
                    cu_seqlens, total, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, const int* seqlens, fa_stream_t stream) {
    return fa_fwd_gqa(q, k, v, o, lse, B, H, H, N, d, scale, causal, seqlens, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
    if (check_common(B, H, N, d, 1.0f) != FA_OK) return 0;
    const size_t BH = (size_t)B * H;
    const size_t Np = (size_t)pad128(N);
    size_t bytes = 0;
    auto add = [&](size_t n) { bytes += (n + 255) / 256 * 256; };
    add(BH * N * sizeof(float));             // D
    add(BH * N * sizeof(float));             // |dO_i|
    add(BH * (Np / 128) * 2 * sizeof(float)); // per-chunk maxima of |v_j| and |k_jl|
    add(BH * Np * d * sizeof(int));          // fixed-point dQ accumulator
    return bytes;
}

static fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o,
                          const void* dO, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int H_kv, int N, int d, float scale, int causal,
                          const int* seqlens, const int* cu_seqlens, int T, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    fa_status st = check_layout(B, H, H_kv, N, d, scale, seqlens, cu_seqlens, T, false);
    if (st != FA_OK) return st;
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, N, d))
        return FA_ERR_WORKSPACE;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;

    const int BH = B * H;
    const int Np = pad128(N);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    size_t off = 0;
    auto take = [&](size_t n) {
        void* p = ws + off;
        off += (n + 255) / 256 * 256;
        return p;
    };
    BwdParams p{};
    p.o = o;
    p.dO = dO;
    p.lse = lse;
    p.k = k;
    p.v = v;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.Dvec = static_cast<float*>(take((size_t)BH * N * sizeof(float)));
    p.dOnorm = static_cast<float*>(take((size_t)BH * N * sizeof(float)));
    p.headmax = static_cast<float*>(take((size_t)BH * (Np / 128) * 2 * sizeof(float)));
    p.dq_acc = static_cast<int*>(take((size_t)BH * Np * d * sizeof(int)));
    p.seqlens = seqlens;
    p.cu_seqlens = cu_seqlens;
    p.T = T;
    p.err = dev->err_flag;
    p.B = B;
    p.H = H;
    p.N = N;
    p.N_pad = Np;
    p.H_kv = H_kv;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.timeout_ns = g_timeout_ns.load();
    const bool packed = cu_seqlens != nullptr;
    p.num_sms = dev->num_sms;
    p.dbg = extents(B, H, H_kv, N, d, T, packed);

    CUtensorMap tq, tk, tv, tdo;
    const int q_rows = d == 256 ? 64 : 128;  // query rows per backward step
    if (!user_map(&tq, q, d, B, H, N, T, packed, q_rows) ||
        !user_map(&tk, k, d, B, H_kv, N, T, packed) ||
        !user_map(&tv, v, d, B, H_kv, N, T, packed) ||
        !user_map(&tdo, dO, d, B, H, N, T, packed, q_rows))
        return FA_ERR_CUDA;
    cudaEvent_t ev0, ev1;
    take_timing_events(&ev0, &ev1);
    if (launch_bwd(d, tq, tk, tv, tdo, p, stream, ev0, ev1) != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                     const void* dO, const float* lse, void* dq, void* dk, void* dv, int B, int H,
                     int H_kv, int N, int d, float scale, int causal, const int* seqlens,
                     void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, H, H_kv, N, d, scale, causal, seqlens,
                    nullptr, 0, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                        const void* dO, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens, int B, int max_seqlen, int total, int H, int H_kv,
                        int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                        fa_stream_t stream) {
    if (!cu_seqlens) return FA_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, H, H_kv, max_seqlen, d, scale, causal,
                    nullptr, cu_seqlens, total, workspace, workspace_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 float scale, int causal, const int* seqlens, void* workspace,
                 size_t workspace_bytes, fa_stream_t stream) {
    return fa_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, B, H, H, N, d, scale, causal, seqlens,
                      workspace, workspace_bytes, stream);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                     const float* k_descale, const float* v_descale, void* o, float* lse, int B,
                     int H, int H_kv, int N, int d, float scale, int causal, const int* seqlens,
                     fa_stream_t stream) {
    fa_status st = check_common(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (H_kv < 1 || H_kv > H || H % H_kv != 0) return FA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    for (const void* ptr : {(const void*)q_descale, (const void*)k_descale,
                            (const void*)v_descale, (const void*)seqlens})
        if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 3u)) return FA_ERR_INVALID_ARG;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;

    CUtensorMap tq, tk, tv;
    if (!make_fp8_map(&tq, q, N, B * H) || !make_fp8_map(&tk, k, N, B * H_kv) ||
        !make_fp8_map(&tv, v, N, B * H_kv))
        return FA_ERR_CUDA;
    Fp8Params p{};
    p.o = o;
    p.lse = lse;
    p.seqlens = seqlens;
    p.q_descale = q_descale;
    p.k_descale = k_descale;
    p.v_descale = v_descale;
    p.err = dev->err_flag;
    p.H = H;
    p.N = N;
    p.H_kv = H_kv;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.timeout_ns = g_timeout_ns.load();
    p.dbg = extents(B, H, H_kv, N, d, 0, false);
    cudaEvent_t ev0, ev1;
    take_timing_events(&ev0, &ev1);
    const cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
    if (ev0) cudaEventRecord(ev0, st_);
    const cudaError_t e = launch_fwd_fp8(tq, tk, tv, p, B, st_);
    if (ev1) cudaEventRecord(ev1, st_);
    if (e != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

int fa_decode_num_splits(int B, int H, int H_kv, int Nq, int N, int d, int ragged) {
    if (check_decode(B, H, H_kv, Nq, N, d, 1.0f, 0) != FA_OK) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            sms = v;
    }
    const int n_mt = ((H / H_kv) * Nq + 127) / 128;
    return decode_splits(B, H_kv, n_mt, N, decode_block_keys(d), sms * decode_ctas_per_sm(d),
                         ragged != 0);
}

size_t fa_decode_workspace_size(int B, int H, int Nq, int d, int splits) {
    if (B < 1 || H < 1 || Nq < 1 || splits < 1 || (d != 64 && d != 128 && d != 256)) return 0;
    if (splits == 1) return 0;
    const size_t rows = (size_t)B * H * Nq;
    const size_t o_bytes = ((size_t)splits * rows * d * sizeof(float) + 255) / 256 * 256;
    return o_bytes + (size_t)splits * rows * sizeof(float);
}

fa_status fa_fwd_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                        float* lse, const int* cache_lens, int B, int H, int H_kv, int Nq, int N,
                        int d, float scale, int causal, int splits, void* workspace,
                        size_t workspace_bytes, fa_stream_t stream) {
    fa_status st = check_decode(B, H, H_kv, Nq, N, d, scale, splits);
    if (st != FA_OK) return st;
    if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    if (cache_lens && (reinterpret_cast<uintptr_t>(cache_lens) & 3u)) return FA_ERR_INVALID_ARG;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;

    const int G = H / H_kv;
    const int n_mt = (G * Nq + 127) / 128;
    const int bk = decode_block_keys(d);
    const int nblk = (N + bk - 1) / bk;
    if (splits == 0)
        splits = decode_splits(B, H_kv, n_mt, N, bk, dev->num_sms * decode_ctas_per_sm(d),
                               cache_lens != nullptr);
    if (splits > nblk) splits = nblk;
    const int bps = (nblk + splits - 1) / splits;
    splits = (nblk + bps - 1) / bps;  // ranges that actually hold keys
    if ((long long)H_kv * n_mt > 65535) return FA_ERR_INVALID_ARG;  // grid.y

    DecodeParams p{};
    p.o = o;
    p.lse = lse;
    if (splits > 1) {
        const size_t need = fa_decode_workspace_size(B, H, Nq, d, splits);
        if (!workspace || !aligned16(workspace) || workspace_bytes < need)
            return FA_ERR_WORKSPACE;
        const size_t rows = (size_t)B * H * Nq;
        p.o_part = static_cast<float*>(workspace);
        p.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                              ((size_t)splits * rows * d * sizeof(float) + 255) /
                                                  256 * 256);
    }
    p.cache_lens = cache_lens;
    p.err = dev->err_flag;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.G = G;
    p.Nq = Nq;
    p.N = N;
    p.n_mtiles = n_mt;
    p.splits = splits;
    p.blocks_per_split = bps;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.timeout_ns = g_timeout_ns.load();
    p.dbg = Extents{};
    p.dbg.q = (size_t)B * H * Nq * d;
    p.dbg.kv = (size_t)B * H_kv * N * d;
    p.dbg.lse = (size_t)B * H * Nq;
    p.dbg.part = splits > 1 ? (size_t)splits * B * H * Nq * d : 0;
    p.dbg.nseq = B;

    CUtensorMap tq, tk, tv;
    if (!make_bf16_map(&tq, q, d, G * Nq, B * H_kv, 128) ||
        !make_bf16_map(&tk, k_cache, d, N, B * H_kv, bk) ||
        !make_bf16_map(&tv, v_cache, d, N, B * H_kv, bk))
        return FA_ERR_CUDA;
    cudaEvent_t ev0, ev1;
    take_timing_events(&ev0, &ev1);
    if (launch_decode(d, tq, tk, tv, p, reinterpret_cast<cudaStream_t>(stream), ev0, ev1) !=
        cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

fa_status fa_selftest_bounds(int* buf, int n, int value, fa_stream_t stream) {
    if (!kDebugChecks) return FA_ERR_UNSUPPORTED;  // checks compiled out: nothing to exercise
    if (!buf || n < 1 || (reinterpret_cast<uintptr_t>(buf) & 3u)) return FA_ERR_INVALID_ARG;
    fa_status st;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;
    if (fa::launch_bounds_selftest(buf, n, value, dev->err_flag,
                                   reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

int fa_debug_checks(void) { return kDebugChecks ? 1 : 0; }

fa_status fa_selftest_wait_timeout(fa_stream_t stream) {
    fa_status st;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;
    if (fa::launch_wait_selftest(dev->err_flag, g_timeout_ns.load(),
                                 reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

fa_status fa_check_device_error(fa_stream_t stream) {
    fa_status st;
    DeviceState* dev = current_device(&st);
    if (!dev) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    int flag = 0;
    if (cudaMemcpy(&flag, dev->err_flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FA_ERR_CUDA;
    if (flag != 0 && cudaMemset(dev->err_flag, 0, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return static_cast<fa_status>(flag);
}

}  // extern "C"
