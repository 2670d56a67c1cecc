// fa_internal.h -- declarations shared by the host ABI (fa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fa.h"

namespace fa {

// Device error-flag codes mirror fa_status.
constexpr int kErrInvalidArg = FA_ERR_INVALID_ARG;
constexpr int kErrTimeout = FA_ERR_TIMEOUT;

struct FwdParams {
    void* o;               // bf16 [B, H, N, d]
    float* lse;            // fp32 [B, H, N]
    const int* seqlens;    // device int32 [B] or nullptr
    int* err;              // device error flag
    int H, N;
    int H_kv;              // key/value heads; query head h reads K/V head h / (H / H_kv)
    float scale_log2;      // scale * log2(e)
    int causal;
    uint64_t timeout_ns;
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
    int* err;
    int B, H, N, N_pad;
    int H_kv;              // key/value heads (H % H_kv == 0); dK, dV are [B, H_kv, N, d]
    float scale;
    float scale_log2;
    int causal;
    uint64_t timeout_ns;
};

// Current bound on device-side waits (fa_set_wait_timeout_ns).
uint64_t wait_timeout_ns();

// Tensor maps: a bf16 [B*H, N, d] tensor seen as 3-D (d, N, B*H), 128-byte swizzle,
// box = 64 columns x `box_rows` rows; rows past N read as zeros.
bool make_bf16_map(CUtensorMap* map, const void* base, int d, int N, int BH, int box_rows);

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int B, int num_sms, cudaStream_t stream);

cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream);

}  // namespace fa
