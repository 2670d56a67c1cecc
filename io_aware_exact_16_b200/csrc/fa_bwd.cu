// fa_bwd.cu -- exact-attention backward pass for sm_100a.
//
// The forward pass keeps only the per-row log-sum-exp; the backward pass recomputes the
// probabilities block by block from it (flash-attention glossary page, "Hoe werkt het?", item
// "Herberekening") and forms the ordinary derivative of softmax(scale Q K^T) V:
//
//   P  = exp(scale Q K^T - lse)       dV = P^T dO          dP = dO V^T
//   D  = rowsum(dO * O)               dS = P * (dP - D)
//   dK = scale dS^T Q                 dQ = scale dS K
//
// Three kernels run in order on one stream:
//   fa_bwd_pre_kernel   D = rowsum(dO * O) in fp32; clears the ordering counters
//   fa_bwd_kernel       one CTA per 128-key block: recomputes S^T, P^T, dP^T, dS^T per
//                       128-query block with tcgen05 MMAs, accumulates dK, dV in tensor memory
//                       and adds its dQ block contribution into an fp32 accumulator in a fixed
//                       key-block order (deterministic)
//   fa_bwd_dq_kernel    dQ = scale * accumulator -> bf16
//
// Main-kernel warp roles (320 threads):
//   warps 0-3  S/dP -> P, dS (thread r owns key row r = TMEM lane r)
//   warps 4-7  dQ drain (thread r owns query row r) + dK/dV epilogue
//   warp  8    MMA issue (one thread) + TMEM allocation
//   warp  9    TMA producer (one thread)
// Tensor memory (512 columns): A [0,128) S^T -> P^T (bf16) -> dQ block (fp32, d columns)
//                              B [128,256) dP^T -> dS^T (bf16)
//                              dV [256, 256+d)   dK [256+d, 256+2d)
// Shared memory: K_j, V_j (once), a 2-stage ring of Q_i / dO_i, dS^T (bf16, 128-byte
// swizzled, written by warps 0-3 for the dQ MMA), lse*log2(e) and D of the query block.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
    static constexpr int BM = 128;  // query rows per block
    static constexpr int BN = 128;  // key rows per CTA
    static constexpr int KCH = D / 64;
    static constexpr int QST = 2;   // Q / dO stages
    static constexpr int KV_TILE_BYTES = BN * D * 2;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int CHUNK_BYTES = 128 * 128;
    static constexpr int DS_BYTES = BN * BM * 2;
    static constexpr int SMEM_K = 0;
    static constexpr int SMEM_V = SMEM_K + KV_TILE_BYTES;
    static constexpr int SMEM_Q = SMEM_V + KV_TILE_BYTES;
    static constexpr int SMEM_DO = SMEM_Q + QST * Q_TILE_BYTES;
    static constexpr int SMEM_DS = SMEM_DO + QST * Q_TILE_BYTES;
    static constexpr int SMEM_VEC = SMEM_DS + DS_BYTES;       // [2][128] lse2, [2][128] D
    static constexpr int SMEM_BAR = SMEM_VEC + 4 * BM * 4;
    static constexpr int NUM_BARS = 1 + 2 * QST + 5;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16;
    static constexpr int THREADS = 320;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
};

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ int seq_len(const BwdParams& p, int b, bool report) {
    int L = p.N;
    if (p.seqlens != nullptr) {
        L = p.seqlens[b];
        if (L < 1 || L > p.N) {
            if (report) record_error(p.err, kErrInvalidArg);
            L = L < 1 ? 1 : p.N;
        }
    }
    return L;
}

// ---------------------------------------------------------------------------- preprocess
// D[row] = sum_k dO[row, k] * O[row, k] in fp32.  16 threads per row for d = 128 (8 for d = 64),
// each reading 16 bytes of dO and O.  Also clears the ordering counters and the tile counter.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p, int rows, int n_sem) {
    constexpr int TPR = D / 8;  // threads per row
    const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
    const int row = gtid / TPR;
    const int part = gtid % TPR;
    float acc = 0.f;
    if (row < rows) {
        const uint4 a = reinterpret_cast<const uint4*>(p.dO)[(size_t)row * TPR + part];
        const uint4 o = reinterpret_cast<const uint4*>(p.o)[(size_t)row * TPR + part];
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 fa = __bfloat1622float2(a2[i]);
            const float2 fo = __bfloat1622float2(o2[i]);
            acc = fmaf(fa.x, fo.x, acc);
            acc = fmaf(fa.y, fo.y, acc);
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && part == 0) p.Dvec[row] = acc;
    for (int i = gtid; i < n_sem; i += gridDim.x * blockDim.x) p.sem[i] = 0;
    if (gtid == 0) *p.tile_counter = 0;
}

// ---------------------------------------------------------------------------- dQ convert
// dq = bf16(scale * dq_acc) for the N real rows of every head; 8 elements per thread.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p, long long total8) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total8) return;
    const long long e = i * 8;               // element index in [BH, N, D]
    const long long row = e / D;             // bh * N + n
    const int col = (int)(e % D);
    const long long bh = row / p.N;
    const long long n = row % p.N;
    const float4* src =
        reinterpret_cast<const float4*>(p.dq_acc + ((bh * p.N_pad + n) * D + col));
    const float4 x = src[0], y = src[1];
    uint4 out;
    out.x = pack_bf16x2(x.x * p.scale, x.y * p.scale);
    out.y = pack_bf16x2(x.z * p.scale, x.w * p.scale);
    out.z = pack_bf16x2(y.x * p.scale, y.y * p.scale);
    out.w = pack_bf16x2(y.z * p.scale, y.w * p.scale);
    reinterpret_cast<uint4*>(p.dq)[i] = out;
}

// ---------------------------------------------------------------------------- main kernel
template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int n_q = (p.N + C::BM - 1) / C::BM;  // query blocks per head
    const int n_kv = (p.N + C::BN - 1) / C::BN;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_kv = bars;
    uint64_t* bar_qfull = bars + 1;
    uint64_t* bar_qempty = bar_qfull + C::QST;
    uint64_t* bar_sfull = bar_qempty + C::QST;
    uint64_t* bar_pfull = bar_sfull + 1;
    uint64_t* bar_dqfull = bar_pfull + 1;
    uint64_t* bar_dqempty = bar_dqfull + 1;
    uint64_t* bar_dkvfull = bar_dqempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
    int* tile_slot = reinterpret_cast<int*>(smem + C::SMEM_MISC + 8);
    float* s_lse2 = reinterpret_cast<float*>(smem + C::SMEM_VEC);       // [2][BM]
    float* s_D = s_lse2 + 2 * C::BM;                                      // [2][BM]

    // Tiles are claimed in launch order with an atomic ticket, so a CTA only ever waits (in the
    // ordered dQ reduction) for tiles that running CTAs claimed earlier: no deadlock.
    if (threadIdx.x == 0) {
        *tile_slot = atomicAdd(p.tile_counter, 1);
        if (smem_u32(smem) & 1023u) record_error(p.err, kErrInvalidArg);
    }
    __syncthreads();
    const int tile = *tile_slot;
    const int bh = tile / n_kv;
    // Key block of this tile.  Causal heads run their key blocks from last to first: block j
    // then reaches query block i after i - j steps, so the order in which blocks arrive at a
    // query block is j = i, i-1, ..., 0 -- the order the dQ reduction below adds them in.
    const int j = p.causal ? (n_kv - 1 - tile % n_kv) : (tile % n_kv);
    const int b = bh / p.H;
    const int L = seq_len(p, b, threadIdx.x == 0 && j == 0);
    const int k0 = j * C::BN;

    if (k0 >= L) {
        // Every key of this block is padding: dK = dV = 0 and no dQ contribution.
        const int rows = min(C::BN, p.N - k0);
        uint4* dk = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dk) + ((size_t)bh * p.N + k0) * D);
        uint4* dv = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dv) + ((size_t)bh * p.N + k0) * D);
        for (int i = threadIdx.x; i < rows * D / 8; i += blockDim.x) {
            dk[i] = make_uint4(0, 0, 0, 0);
            dv[i] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int i_start = p.causal ? j : 0;  // causal: query blocks before the diagonal see none
    const int n_kv_valid = (L + C::BN - 1) / C::BN;
    const int n_it = n_q - i_start;

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < C::QST; ++s) {
            mbar_init(&bar_qfull[s], 1);
            mbar_init(&bar_qempty[s], 1);
        }
        mbar_init(bar_sfull, 1);
        mbar_init(bar_pfull, C::BN);
        mbar_init(bar_dqfull, 1);
        mbar_init(bar_dqempty, C::BM);
        mbar_init(bar_dkvfull, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&]() {
        record_error(p.err, kErrTimeout);
        *abort_flag = 1;
    };

    if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            prefetch_tensormap(&tmDO);
            mbar_arrive_expect_tx(bar_kv, 2 * C::KV_TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(smem + C::SMEM_K + c * C::CHUNK_BYTES, &tmK, bar_kv, c * 64, k0, bh);
                tma_load_3d(smem + C::SMEM_V + c * C::CHUNK_BYTES, &tmV, bar_kv, c * 64, k0, bh);
            }
            int it = 0;
            for (; it < n_it; ++it) {
                const int s = it % C::QST;
                const uint32_t ph = (it / C::QST) & 1;
                const int q0 = (i_start + it) * C::BM;
                if (!mbar_wait(&bar_qempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&bar_qfull[s], 2 * C::Q_TILE_BYTES);
                for (int c = 0; c < C::KCH; ++c) {
                    tma_load_3d(smem + C::SMEM_Q + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES, &tmQ,
                                &bar_qfull[s], c * 64, q0, bh);
                    tma_load_3d(smem + C::SMEM_DO + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES,
                                &tmDO, &bar_qfull[s], c * 64, q0, bh);
                }
            }
            // Do not leave while our copies may still be landing in shared memory.
            for (int t = max(0, it - C::QST); t < it; ++t)
                mbar_wait(&bar_qfull[t % C::QST], (t / C::QST) & 1, p.timeout_ns, abort_flag);
            mbar_wait(bar_kv, 0, p.timeout_ns, abort_flag);
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, false, false);  // S^T, dP^T
            constexpr uint32_t idKV = idesc_bf16(128, D, false, true);    // dV, dK (A in TMEM)
            constexpr uint32_t idQ = idesc_bf16(128, D, true, true);      // dQ = dS K
            const uint32_t sK = smem_u32(smem + C::SMEM_K);
            const uint32_t sV = smem_u32(smem + C::SMEM_V);
            const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
            const uint32_t sDO = smem_u32(smem + C::SMEM_DO);
            const uint32_t sDS = smem_u32(smem + C::SMEM_DS);
            bool ok = mbar_wait(bar_kv, 0, p.timeout_ns, abort_flag);
            for (int it = 0; ok && it < n_it; ++it) {
                const int s = it % C::QST;
                const uint32_t ph = (it / C::QST) & 1;
                const uint32_t qa = sQ + s * C::Q_TILE_BYTES;
                const uint32_t da = sDO + s * C::Q_TILE_BYTES;
                if (!(ok = mbar_wait(&bar_qfull[s], ph, p.timeout_ns, abort_flag))) break;
                if (it > 0 && !(ok = mbar_wait(bar_dqempty, (it - 1) & 1, p.timeout_ns, abort_flag)))
                    break;
                tc_fence_after();
                // S^T = K Q^T and dP^T = V dO^T: K-major operands, 16-column K steps.
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32;
                    mma_ss(tmem + C::TM_A, sdesc_sw128(sK + off, 16, 1024),
                           sdesc_sw128(qa + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32;
                    mma_ss(tmem + C::TM_B, sdesc_sw128(sV + off, 16, 1024),
                           sdesc_sw128(da + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar_sfull);
                if (!(ok = mbar_wait(bar_pfull, it & 1, p.timeout_ns, abort_flag))) break;
                tc_fence_after();
                // dV += P^T dO and dK += dS^T Q: A from tensor memory (16 queries = 8 columns per
                // K step), B MN-major in shared memory (16 query rows = 2048 bytes per K step).
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; ++kk)
                    mma_ts(tmem + C::TM_DV, tmem + C::TM_A + kk * 8,
                           sdesc_sw128(da + kk * 2048, C::CHUNK_BYTES, 1024), idKV,
                           (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; ++kk)
                    mma_ts(tmem + C::TM_DK, tmem + C::TM_B + kk * 8,
                           sdesc_sw128(qa + kk * 2048, C::CHUNK_BYTES, 1024), idKV,
                           (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&bar_qempty[s]);
                // dQ block = dS K: A = dS (queries x keys) read MN-major from the dS^T tile,
                // B = K MN-major (16 key rows = 2048 bytes per K step).
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ss(tmem + C::TM_A, sdesc_sw128(sDS + kk * 2048, C::CHUNK_BYTES, 1024),
                           sdesc_sw128(sK + kk * 2048, C::CHUNK_BYTES, 1024), idQ,
                           kk > 0 ? 1u : 0u);
                tc_commit(bar_dqfull);
            }
            if (!ok) fail();
            // Always signal the end, then wait for every MMA this thread issued to finish, so
            // tensor memory is never released under a running MMA (also on the abort path).
            tc_commit(bar_dkvfull);
            mbar_wait(bar_dkvfull, 0, p.timeout_ns, abort_flag);
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ P^T and dS^T
        const int r = threadIdx.x;  // key row in the block == TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int kidx = k0 + r;
        const bool key_padded = kidx >= L;
        uint8_t* ds_row = smem + C::SMEM_DS + r * 128;
        const int sw = r & 7;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = i_start + it;
            const int q0 = i * C::BM;
            const int buf = it & 1;
            {
                const int q = q0 + r;
                s_lse2[buf * C::BM + r] =
                    q < p.N ? p.lse[(size_t)bh * p.N + q] * kLog2e : INFINITY;
                s_D[buf * C::BM + r] = q < p.N ? p.Dvec[(size_t)bh * p.N + q] : 0.f;
            }
            named_barrier(1, 128);
            ok = mbar_wait(bar_sfull, it & 1, p.timeout_ns, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const bool diag = p.causal && (i == j);
            const float* lse2 = s_lse2 + buf * C::BM;
            const float* Dv = s_D + buf * C::BM;
#pragma unroll 1
            for (int c = 0; c < C::BM / 32; ++c) {
                uint32_t sv[32], dp[32];
                tmem_ld32(tmem + lane_base + C::TM_A + c * 32, sv);
                tmem_ld32(tmem + lane_base + C::TM_B + c * 32, dp);
                tmem_ld_wait();
                reg_fence32(sv);
                reg_fence32(dp);
                uint32_t pw[16], dw[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int col = c * 32 + e;
                    float p0 = ex2(fmaf(__uint_as_float(sv[e]), p.scale_log2, -lse2[col]));
                    float p1 = ex2(fmaf(__uint_as_float(sv[e + 1]), p.scale_log2, -lse2[col + 1]));
                    if (key_padded || (diag && r > col)) p0 = 0.f;
                    if (key_padded || (diag && r > col + 1)) p1 = 0.f;
                    const float d0 = p0 * (__uint_as_float(dp[e]) - Dv[col]);
                    const float d1 = p1 * (__uint_as_float(dp[e + 1]) - Dv[col + 1]);
                    pw[e / 2] = pack_bf16x2(p0, p1);
                    dw[e / 2] = pack_bf16x2(d0, d1);
                }
                // P^T and dS^T as bf16 into tensor memory over the columns already read.
                tmem_st16(tmem + lane_base + C::TM_A + c * 16, pw);
                tmem_st16(tmem + lane_base + C::TM_B + c * 16, dw);
                // dS^T row r into the 128-byte-swizzled shared tile: query chunk c/2, 16-byte
                // units (c%2)*4 .. +3, unit u stored at position u ^ (r % 8).
                uint8_t* base = ds_row + (c / 2) * C::CHUNK_BYTES;
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    const int u = (c % 2) * 4 + u4;
                    *reinterpret_cast<uint4*>(base + ((u ^ sw) << 4)) =
                        make_uint4(dw[4 * u4], dw[4 * u4 + 1], dw[4 * u4 + 2], dw[4 * u4 + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_pfull);
        }
        if (!ok) fail();
    } else {
        // ------------------------------------------------------------ dQ drain, dK/dV epilogue
        const int r = threadIdx.x - 128;  // query row in the block == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = i_start + it;
            ok = mbar_wait(bar_dqfull, it & 1, p.timeout_ns, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t v[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_base + C::TM_A + c * 32, v + c * 32);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) reg_fence32(v + c * 32);
            tc_fence_before();
            mbar_arrive(bar_dqempty);

            // Ordered reduction into the fp32 accumulator of query block i.  Non-causal: key
            // blocks add in ascending order (position j).  Causal: descending from the last key
            // block that sees block i (position jmax - j).  The counter holds the number of
            // blocks already added; a tile only waits for tiles claimed before it.
            const int jmax = min(i, n_kv_valid - 1);
            const int pos = p.causal ? (jmax - j) : j;
            int* sem = p.sem + (size_t)bh * n_q + i;
            if (r == 0 && pos > 0) {
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(sem) != pos) {
                    if (*abort_flag || globaltimer_ns() - t0 > p.timeout_ns) { ok = false; break; }
                }
                if (!ok) fail();
            }
            named_barrier(2, 128);
            if (*abort_flag) { ok = false; break; }
            float* dst = p.dq_acc + ((size_t)bh * p.N_pad + (size_t)i * C::BM + r) * D;
            if (pos == 0) {
#pragma unroll
                for (int c = 0; c < D; c += 4)
                    *reinterpret_cast<float4*>(dst + c) =
                        make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                    __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
            } else {
#pragma unroll
                for (int c = 0; c < D; c += 4)
                    red_add_v4(dst + c, __uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                               __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
            }
            __threadfence();
            named_barrier(2, 128);
            if (r == 0) st_release_gpu(sem, pos + 1);
        }
        if (ok) ok = mbar_wait(bar_dkvfull, 0, p.timeout_ns, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const int kidx = k0 + r;
            const bool in_range = kidx < p.N;
            const size_t off = ((size_t)bh * p.N + (in_range ? kidx : 0)) * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col0 = which ? C::TM_DK : C::TM_DV;
                const float mul = which ? p.scale : 1.0f;
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(which ? p.dk : p.dv) + off;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_base + col0 + c * 32, x);
                    tmem_ld_wait();
                    reg_fence32(x);
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(x[2 * e]) * mul,
                                           __uint_as_float(x[2 * e + 1]) * mul);
                    if (in_range) {
                        uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    }
                }
            }
        } else {
            fail();
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_bwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    using C = BwdCfg<D>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(fa_bwd_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int BH = p.B * p.H;
    const int n_q = (p.N + C::BM - 1) / C::BM;
    const int n_kv = (p.N + C::BN - 1) / C::BN;
    const int rows = BH * p.N;
    const int n_sem = BH * n_q;
    {
        constexpr int TPR = D / 8;
        const long long threads = (long long)rows * TPR;
        const int blocks = (int)((threads + 255) / 256);
        fa_bwd_pre_kernel<D><<<blocks, 256, 0, stream>>>(p, rows, n_sem);
    }
    fa_bwd_kernel<D><<<BH * n_kv, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    {
        const long long total8 = (long long)rows * D / 8;
        const int blocks = (int)((total8 + 255) / 256);
        fa_bwd_dq_kernel<D><<<blocks, 256, 0, stream>>>(p, total8);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq_acc, const BwdParams& p,
                       int num_sms, cudaStream_t stream) {
    (void)tdq_acc;
    (void)num_sms;
    if (d == 64) return launch_bwd_d<64>(tq, tk, tv, tdo, p, stream);
    return launch_bwd_d<128>(tq, tk, tv, tdo, p, stream);
}

}  // namespace fa
