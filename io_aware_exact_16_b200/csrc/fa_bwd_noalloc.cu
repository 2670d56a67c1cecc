// fa_bwd_noalloc.cu -- the backward pass for callers that must not allocate device memory.
//
// fa_bwd needs a workspace that the caller allocates.  Some callers cannot do that: a serving
// process that reserves (almost) all device memory for its own pool at start-up, where a later
// cudaMalloc would fail or fragment that pool, or a latency-critical loop where cudaMalloc /
// cudaFree are off limits because they can block and synchronise the whole device.  For them
// fa_bwd_noalloc runs the same three backward kernels on a fixed scratch area that is part of
// this library's device image: a file-scope __device__ array, created when the library's code
// is loaded onto a GPU and kept by every GPU that loads it until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it only names a
// stand-in object), so the device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, and handed to the kernels.  Under lazy
// module loading that first lookup is also when the array is placed in device memory.
#include <cuda_runtime.h>

#include <mutex>

#include "fa_internal.h"

namespace {

constexpr size_t kScratchBytes = FA_BWD_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The shared scratch of every fa_bwd_noalloc call on a device (see the header).
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

struct ScratchDevice {
    bool ready = false;      // set-up done for this device
    bool supported = false;  // compute capability 10.0
    int num_sms = 0;         // multiprocessors (the backward's persistent grid)
    void* scratch = nullptr; // device address of g_bwd_scratch on this device
};
ScratchDevice g_scratch_dev[kMaxDevices];
std::mutex g_scratch_mutex;

// One-time set-up for the current device: check it is a B200-class GPU and look up the
// device address of the scratch array.  Allocates nothing.
fa_status scratch_for_current_device(void** out, int* num_sms) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchDevice& s = g_scratch_dev[dev];
    if (!s.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        s.supported = (major == 10 && minor == 0);
        if (s.supported) {
            // With lazy module loading (the CUDA default since 12.2) this lookup is what loads
            // this file's device image, and with it commits the scratch array: it can fail for
            // lack of device memory, which is reported as FA_ERR_WORKSPACE.
            void* ptr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
            if (e == cudaErrorMemoryAllocation) {
                cudaGetLastError();  // not sticky: clear it so later calls start clean
                return FA_ERR_WORKSPACE;
            }
            if (e != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
            s.scratch = ptr;
        }
        s.ready = true;
    }
    if (!s.supported) return FA_ERR_UNSUPPORTED;
    *out = s.scratch;
    *num_sms = s.num_sms;
    return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v,
                                           const void* o, const void* dO, const float* lse,
                                           void* dq, void* dk, void* dv, int B, int H, int N,
                                           int d, float scale, int causal, const int* seqlens,
                                           int* error_flag, fa_stream_t stream) {
    // Same argument rules as fa_bwd (fa_bwd_workspace_size returns 0 for invalid sizes).
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const size_t need = fa_bwd_workspace_size(B, H, N, d);
    if (need == 0) return FA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale <= 3.4e38f)) return FA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    if (error_flag && (reinterpret_cast<uintptr_t>(error_flag) & 3u)) return FA_ERR_INVALID_ARG;
    // Larger problems than the fixed scratch holds are refused, never truncated.
    if (need > kScratchBytes) return FA_ERR_WORKSPACE;
    void* scratch = nullptr;
    int num_sms = 0;
    fa_status st = scratch_for_current_device(&scratch, &num_sms);
    if (st != FA_OK) return st;

    // Carve the scratch exactly as fa_bwd carves its workspace.  Nothing in it has to start
    // at zero: the first backward kernel writes D, the norms and the bound maxima and clears
    // the dQ accumulator on every call, so the previous call's leftovers never matter.
    const int BH = B * H;
    const int Np = (N + 127) / 128 * 128;
    uint8_t* ws = static_cast<uint8_t*>(scratch);
    size_t off = 0;
    auto take = [&](size_t n) {
        void* p = ws + off;
        off += (n + 255) / 256 * 256;
        return p;
    };
    fa::BwdParams p{};
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
    p.err = error_flag;  // caller-owned; NULL = device-side errors are not reported
    p.B = B;
    p.H = H;
    p.N = N;
    p.N_pad = Np;
    p.H_kv = H;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.timeout_ns = fa::wait_timeout_ns();
    p.num_sms = num_sms;
    p.dbg = fa::extents(B, H, H, N, d, 0, false);

    CUtensorMap tq, tk, tv, tdo;
    if (!fa::make_bf16_map(&tq, q, d, N, BH, 128) || !fa::make_bf16_map(&tk, k, d, N, BH, 128) ||
        !fa::make_bf16_map(&tv, v, d, N, BH, 128) || !fa::make_bf16_map(&tdo, dO, d, N, BH, 128))
        return FA_ERR_CUDA;
    if (fa::launch_bwd(d, tq, tk, tv, tdo, p, reinterpret_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}
