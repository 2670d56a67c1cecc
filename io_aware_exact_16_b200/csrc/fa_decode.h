// fa_decode.h -- parameters of the split-KV decode kernels (fa_decode.cu), shared with the
// host ABI (fa_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {

struct DecodeParams {
    void* o;                // bf16 [B, H, Nq, d]
    float* lse;             // fp32 [B, H, Nq]
    float* o_part;          // fp32 [splits, B*H*Nq, d] workspace (splits > 1)
    float* lse_part;        // fp32 [splits, B*H*Nq]    workspace (splits > 1)
    const int* cache_lens;  // device int32 [B] valid cache rows, or nullptr (= N)
    int* err;               // device error flag
    int B, H, H_kv, G, Nq;  // G = H / H_kv query heads per cache head
    int N;                  // cache rows per head (capacity)
    int n_mtiles;           // ceil(G * Nq / 128)
    int splits;             // key ranges per (b, cache head)
    int blocks_per_split;   // key blocks (decode_block_keys(d) keys each) per range
    float scale_log2;       // scale * log2(e)
    int causal;
    uint64_t timeout_ns;
    Extents dbg;            // buffer sizes for the FA_DEBUG index checks
};

// Query tile map: q [B, H, Nq, d] seen as (d, G*Nq, B*H_kv); cache maps as make_bf16_map.
// Keys per block of the decode kernel for head dim d (the unit of blocks_per_split and of the
// K/V tensor maps' box rows) and how many of its CTAs share one SM.
int decode_block_keys(int d);
int decode_ctas_per_sm(int d);

// ev_start / ev_stop (optional) bracket the split kernel on `stream` (not the combine).
cudaError_t launch_decode(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream,
                          cudaEvent_t ev_start = nullptr, cudaEvent_t ev_stop = nullptr);

}  // namespace fa
