// fa_fwd_fp8.h -- parameters of the FP8 (e4m3) forward kernel (fa_fwd_fp8.cu), shared with the
// host ABI (fa_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {

struct Fp8Params {
    void* o;                 // bf16 [B, H, N, d]
    float* lse;              // fp32 [B, H, N]
    const int* seqlens;      // device int32 [B] key lengths, or nullptr
    const float* q_descale;  // device fp32 [B, H]    (value = code * descale), nullptr = 1
    const float* k_descale;  // device fp32 [B, H_kv]
    const float* v_descale;  // device fp32 [B, H_kv]
    int* err;                // device error flag
    int H, N, H_kv;
    float scale_log2;        // scale * log2(e)
    int causal;
    uint64_t timeout_ns;
    Extents dbg;            // buffer sizes for the FA_DEBUG index checks
};

// Tensor maps: e4m3 [B*Hx, N, 128] as bytes, box 128 x 128 rows, 128-byte swizzle.
bool make_fp8_map(CUtensorMap* map, const void* base, int N, int BHx);

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const Fp8Params& p, int B, cudaStream_t stream);

}  // namespace fa
