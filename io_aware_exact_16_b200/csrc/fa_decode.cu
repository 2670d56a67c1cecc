// fa_decode.cu -- split-KV attention of a few new queries against a long key/value cache
// (sm_100a), for token-by-token generation: the regime of FlashInfer's KV-cache processing in
// streaming generation and of FlashDecoding (FlashAttention (DE), "Spezialisierte Lösungen";
// FlashDecoding++ in its literature list).
//
// Per (batch b, key/value head hk) the query tile is the G * Nq rows of the G query heads that
// share hk (G = H / H_kv), Nq new queries each: in [B, H, Nq, d] these rows are contiguous, so
// one TMA box of 128 rows loads them (rows past G * Nq read as zeros).  The cache's key axis is
// cut into `splits` ranges of whole 128-key blocks; CTA (s, tile, b) runs the forward pass of
// the method (tiled Q K^T, online softmax, P V; FlashAttention (DE), "Online-Softmax-
// Berechnung") over range s only and, with more than one range, writes its partial result as
// (O_s normalised by its own sum, lse_s).  The combine kernel then forms
//   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s,
// the same rescaling the online softmax applies between blocks, so the result is exact.
//
// Decode is bound by reading the cache (each key/value row is read once, used by G * Nq query
// rows), so the CTA keeps a deep ring of 16 KB K/V chunks in flight and double-buffers the
// score block in tensor memory (S(j+1) is computed while the softmax works on S(j)).
//   tensor memory:  S_a [0,BN)  S_b [BN,2BN)  O [2BN, 2BN + d)   (BN keys per block)
//   MMA order:      S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...
// Warp roles (192 threads): warps 0-3 softmax (thread r owns tile row r = TMEM lane r), warp 4
// MMA issue + TMEM allocation, warp 5 TMA.
//
// Causal masking is aligned to the end of the cache: query i of Nq is position L - Nq + i of
// its sequence and sees keys j <= L - Nq + i.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"
#include "fa_decode.h"

namespace fa {
namespace {

using namespace sm100;

// BN = 64 (d <= 128): 256 tensor-memory columns and ~105 KB of shared memory per CTA, so two
// CTAs share an SM and their serial per-block chains (S -> softmax -> P V) overlap;
// BN = 128 (d = 256): O alone needs 256 columns, one CTA per SM.
template <int D>
struct DecCfg {
    static constexpr int BM = 128;                   // query rows per tile
    static constexpr int BN = (D == 256) ? 128 : 64; // keys per block
    static constexpr int CTAS_PER_SM = (D == 256) ? 1 : 2;
    static constexpr int KCH = D / 64;               // 64-column chunks per row
    static constexpr int Q_CHUNK_BYTES = BM * 128;   // a Q chunk: 128 rows x 128 bytes
    static constexpr int CHUNK_BYTES = BN * 128;     // a K/V chunk: BN rows x 128 bytes
    static constexpr int NSLOT = (D == 256) ? 10 : 9;
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_RING = SMEM_Q + KCH * Q_CHUNK_BYTES;
    static constexpr int SMEM_BAR = SMEM_RING + NSLOT * CHUNK_BYTES;
    // q, full[NSLOT], empty[NSLOT], sfull[2], pfull[2], ofull, done
    static constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 1 + 1;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + alignment slack
    static constexpr int THREADS = 192;
    static constexpr uint32_t TM_O = 2 * BN;         // after the two score buffers
    static constexpr uint32_t TMEM_COLS = (TM_O + D <= 256) ? 256 : 512;
    __device__ static constexpr uint32_t tm_s(int buf) { return buf ? (uint32_t)BN : 0u; }
    static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-CTA limit");
    static_assert(CTAS_PER_SM == 1 || (SMEM_BYTES + 1024) * 2 <= 233472,
                  "two CTAs must fit in one SM's shared memory");
    static_assert(TM_O + D <= TMEM_COLS && TMEM_COLS * CTAS_PER_SM <= 512, "tensor memory");
};

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

template <int D>
__global__ void __launch_bounds__(192, DecCfg<D>::CTAS_PER_SM)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
    using C = DecCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int split = blockIdx.x;
    const int hk = blockIdx.y / p.n_mtiles;          // key/value head
    const int mt = blockIdx.y % p.n_mtiles;          // 128-row tile of the group's query rows
    const int b = blockIdx.z;
    const int bhk = b * p.H_kv + hk;
    const int GNq = p.G * p.Nq;                      // query rows sharing this cache head

    int L = p.N;
    if (p.cache_lens != nullptr && in_bounds(p.err, b, 1, p.dbg.nseq)) {
        L = p.cache_lens[b];
        if (L < 1 || L > p.N) {
            if (threadIdx.x == 0 && split == 0 && blockIdx.y == 0) record_error(p.err, kErrInvalidArg);
            L = L < 1 ? 1 : p.N;
        }
    }
    // This CTA's keys: whole 128-key blocks [blk0, blk1) of the cache, cut at L.
    const int nblk_all = (L + C::BN - 1) / C::BN;
    const int blk0 = min(split * p.blocks_per_split, nblk_all);
    const int blk1 = min(blk0 + p.blocks_per_split, nblk_all);
    const int nblk = blk1 - blk0;  // may be 0 for a short sequence: partial (0, -inf)

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_full = bars + 1;                  // [NSLOT]
    uint64_t* bar_empty = bar_full + C::NSLOT;      // [NSLOT]
    uint64_t* bar_sfull = bar_empty + C::NSLOT;     // [2]
    uint64_t* bar_pfull = bar_sfull + 2;            // [2]
    uint64_t* bar_ofull = bar_pfull + 2;
    uint64_t* bar_done = bar_ofull + 1;             // every MMA of this CTA finished
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bar_sfull[t], 1);
            mbar_init(&bar_pfull[t], C::BM);
        }
        mbar_init(bar_ofull, 1);
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
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

    if (warp == 5) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nblk > 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(bar_q, C::KCH * C::Q_CHUNK_BYTES);
            for (int c = 0; c < C::KCH; ++c)
                tma_load_3d(smem + C::SMEM_Q + c * C::Q_CHUNK_BYTES, &tmQ, bar_q, c * 64,
                            mt * C::BM, bhk);
            int u = 0;  // chunks issued into the ring
            bool ok = true;
            auto load_block = [&](const CUtensorMap* map, int j) {
                for (int c = 0; ok && c < C::KCH; ++c) {
                    const int s = u % C::NSLOT;
                    const uint32_t ph = (u / C::NSLOT) & 1;
                    if (!mbar_wait(&bar_empty[s], ph ^ 1, p.timeout_ns, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar_full[s], C::CHUNK_BYTES);
                    tma_load_3d(smem + C::SMEM_RING + s * C::CHUNK_BYTES, map, &bar_full[s],
                                c * 64, (blk0 + j) * C::BN, bhk);
                    ++u;
                }
            };
            // The MMA thread's consumption order: S(0), S(1), then PV(j), S(j+2) for each j.
            load_block(&tmK, 0);
            if (nblk > 1) load_block(&tmK, 1);
            for (int j = 0; ok && j < nblk; ++j) {
                load_block(&tmV, j);
                if (j + 2 < nblk) load_block(&tmK, j + 2);
            }
            if (!ok) fail();
            // Do not leave the CTA while our copies may still be landing in shared memory.
            for (int t = max(0, u - C::NSLOT); t < u; ++t)
                mbar_wait_drain(&bar_full[t % C::NSLOT], (t / C::NSLOT) & 1, p.timeout_ns);
            if (!mbar_wait_drain(bar_q, 0, p.timeout_ns)) fail();
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(C::BM, C::BN, false, false);
            constexpr uint32_t idPV = idesc_bf16(C::BM, 64, false, true);
            const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
            const uint32_t sR = smem_u32(smem + C::SMEM_RING);
            int u = 0;  // ring chunks consumed, in the producer's order

            // S(buf) = Q K_blk^T over the d/64 chunks (16-column steps 32 bytes apart).
            auto issue_S = [&](int buf) {
                for (int c = 0; c < C::KCH; ++c) {
                    const int s = u % C::NSLOT;
                    if (!mbar_wait(&bar_full[s], (u / C::NSLOT) & 1, p.timeout_ns, abort_flag))
                        return false;
                    tc_fence_after();
                    const uint32_t ka = sR + s * C::CHUNK_BYTES;
                    const uint32_t qa = sQ + c * C::Q_CHUNK_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tmem + C::tm_s(buf), sdesc_sw128(qa + kk * 32, 16, 1024),
                               sdesc_sw128(ka + kk * 32, 16, 1024), idS,
                               (c > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_empty[s]);
                    ++u;
                }
                tc_commit(&bar_sfull[buf]);
                return true;
            };
            // O[:, 64c:64c+64] += P V_c per 64-column chunk c of V (P from tensor memory).
            auto issue_PV = [&](int buf, bool accumulate) {
                for (int c = 0; c < C::KCH; ++c) {
                    const int s = u % C::NSLOT;
                    if (!mbar_wait(&bar_full[s], (u / C::NSLOT) & 1, p.timeout_ns, abort_flag))
                        return false;
                    tc_fence_after();
                    const uint32_t va = sR + s * C::CHUNK_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_ts(tmem + C::TM_O + 64 * c, tmem + C::tm_s(buf) + kk * 8,
                               sdesc_sw128(va + kk * 2048, C::CHUNK_BYTES, 1024), idPV,
                               (accumulate || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_empty[s]);
                    ++u;
                }
                tc_commit(bar_ofull);
                return true;
            };

            if (nblk > 0) {
                bool ok = mbar_wait(bar_q, 0, p.timeout_ns, abort_flag);
                if (ok) ok = issue_S(0);
                if (ok && nblk > 1) ok = issue_S(1);
                for (int j = 0; ok && j < nblk; ++j) {
                    const int buf = j & 1;
                    if (!(ok = mbar_wait(&bar_pfull[buf], (j >> 1) & 1, p.timeout_ns,
                                         abort_flag)))
                        break;
                    tc_fence_after();
                    if (!(ok = issue_PV(buf, j > 0))) break;
                    if (j + 2 < nblk && !(ok = issue_S(buf))) break;
                }
                if (!ok) fail();
            }
            // Wait for every MMA issued here before tensor memory can be released.
            tc_commit(bar_done);
            mbar_wait_drain(bar_done, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroup
        const int r = threadIdx.x;                  // tile row = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t tO = tmem + lane_base + C::TM_O;
        const int gr = mt * C::BM + r;              // row within the group: (g, i) = (gr / Nq, gr % Nq)
        const bool valid = gr < GNq;
        // A warp whose 32 rows are all padding keeps the barrier rhythm but skips the work.
        const bool warp_valid = __any_sync(0xffffffffu, valid);
        const int qi = valid ? gr % p.Nq : 0;
        // visible keys j < lim (absolute cache positions); causal: aligned to the cache's end
        const int lim = p.causal ? min(L, L - p.Nq + qi + 1) : L;
        const float c = p.scale_log2;
        float m = -INFINITY;  // running max of S * c (log2 units), possibly stale by <= 8
        float l = 0.f;        // running sum of exp2(S * c - m)
        bool ok = true;

        for (int j = 0; j < nblk; ++j) {
            const int buf = j & 1;
            const uint32_t tS = tmem + lane_base + C::tm_s(buf);
            ok = mbar_wait(&bar_sfull[buf], (j >> 1) & 1, p.timeout_ns, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            if (warp_valid) {
                tc_fence_after();
                uint32_t s[C::BN];
#pragma unroll
                for (int q = 0; q < C::BN / 32; ++q) tmem_ld32(tS + q * 32, s + q * 32);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < C::BN / 32; ++q) reg_fence32(s + q * 32);
                const int k0 = (blk0 + j) * C::BN;
                if (k0 + C::BN > lim) {
#pragma unroll
                    for (int i = 0; i < C::BN; ++i)
                        if (k0 + i >= lim) s[i] = __float_as_uint(-INFINITY);
                }
                float mx8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx8[k] = __uint_as_float(s[k]);
#pragma unroll
                for (int i = 8; i < C::BN; i += 8)
#pragma unroll
                    for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(s[i + k]));
#pragma unroll
                for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                    for (int k = 0; k < w; ++k) mx8[k] = fmaxf(mx8[k], mx8[k + w]);
                const float m_new = fmaxf(m, mx8[0] * c);
                const bool grow = m_new > m + 8.0f;  // false while both are -inf
                const float alpha = (grow && m != -INFINITY) ? ex2(m - m_new) : 1.0f;
                if (grow) {
                    l *= alpha;
                    m = m_new;
                }
                const float mb = (m == -INFINITY) ? 0.f : m;
                const float2 c2 = make_float2(c, c);
                const float2 nm2 = make_float2(-mb, -mb);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int hh = 0; hh < C::BN / 64; ++hh) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e0 = hh * 64 + 2 * i;
                        const float2 x = ffma2(make_float2(__uint_as_float(s[e0]),
                                                           __uint_as_float(s[e0 + 1])), c2, nm2);
                        const float2 e = make_float2(ex2(x.x), ex2(x.y));
                        acc[i % 4] = fadd2(acc[i % 4], e);
                        pk[i] = pack_bf16x2(e.x, e.y);
                    }
                    tmem_st32(tS + hh * 32, pk);  // P over S columns already read
                }
                l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                     ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
                if (__any_sync(0xffffffffu, grow && j > 0)) {
                    // Rescale O once PV(j-1) has landed (S(j) done implies PV(j-2) done, so
                    // the parity wait cannot be a phase behind).
                    ok = mbar_wait(bar_ofull, (j - 1) & 1, p.timeout_ns, abort_flag);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    tc_fence_after();
                    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(tO + q * 32, o);
                        tmem_ld_wait();
                        reg_fence32(o);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float2 y = fmul2(make_float2(__uint_as_float(o[i]),
                                                               __uint_as_float(o[i + 1])), a2);
                            o[i] = __float_as_uint(y.x);
                            o[i + 1] = __float_as_uint(y.y);
                        }
                        tmem_st32(tO + q * 32, o);
                    }
                }
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&bar_pfull[buf]);
        }

        // ------------------------------------------------------------ epilogue
        // every MMA done (bar_done, not the last bar_ofull phase: see the rescale note)
        if (ok) ok = mbar_wait(bar_done, 0, p.timeout_ns, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const size_t rows_total = (size_t)p.B * p.H * p.Nq;
            const size_t R = (size_t)bhk * GNq + (valid ? gr : 0);  // = (b*H + h)*Nq + i
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
            const float lse_v = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (p.splits == 1) {
                const bool o_ok = valid && in_bounds(p.err, R * D, D, p.dbg.q);
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + R * D;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    if (warp_valid) {
                        tmem_ld32(tO + q * 32, o);
                        tmem_ld_wait();
                        reg_fence32(o);
                    }
                    if (o_ok) {
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                               __uint_as_float(o[2 * i + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                    }
                }
                if (valid && in_bounds(p.err, R, 1, p.dbg.lse)) p.lse[R] = lse_v;
            } else {
                // partial of this split: O_s normalised by its own sum (0 if it saw no key)
                const bool o_ok = valid && in_bounds(p.err, ((size_t)split * rows_total + R) * D, D, p.dbg.part);
                float* orow = p.o_part + ((size_t)split * rows_total + R) * D;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    if (warp_valid && nblk > 0) {
                        tmem_ld32(tO + q * 32, o);
                        tmem_ld_wait();
                        reg_fence32(o);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = 0u;
                    }
                    if (o_ok) {
                        float4* dst = reinterpret_cast<float4*>(orow + q * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l,
                                                 __uint_as_float(o[4 * i + 1]) * inv_l,
                                                 __uint_as_float(o[4 * i + 2]) * inv_l,
                                                 __uint_as_float(o[4 * i + 3]) * inv_l);
                    }
                }
                if (valid && in_bounds(p.err, (size_t)split * rows_total + R, 1, p.dbg.part / D))
                    p.lse_part[(size_t)split * rows_total + R] = lse_v;
            }
        } else {
            fail();
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------- combine
// One warp per output row R = (b*H + h)*Nq + i: lse = log sum_s exp(lse_s) and
// O = sum_s exp(lse_s - lse) O_s over the splits, then O -> bf16.  A row that saw no key in
// any split gets O = 0 and lse = -inf.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecodeParams p) {
    constexpr int PER = D / 32;  // columns per lane, contiguous
    constexpr float kLog2e = 1.4426950408889634f;
    const int lane = threadIdx.x % 32;
    const size_t rows_total = (size_t)p.B * p.H * p.Nq;
    const size_t R = (size_t)blockIdx.x * 8 + threadIdx.x / 32;
    if (R >= rows_total) return;
    // every split's partial of this row, and the row of O and lse
    if (!in_bounds(p.err, ((size_t)(p.splits - 1) * rows_total + R) * D, D, p.dbg.part) ||
        !in_bounds(p.err, R * D, D, p.dbg.q) || !in_bounds(p.err, R, 1, p.dbg.lse))
        return;
    float mx = -INFINITY;
    for (int s = lane; s < p.splits; s += 32) mx = fmaxf(mx, p.lse_part[s * rows_total + R]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
    if (mx != -INFINITY)
        for (int s = lane; s < p.splits; s += 32)
            sum += exp2f((p.lse_part[s * rows_total + R] - mx) * kLog2e);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float lse = sum > 0.f ? mx + logf(sum) : -INFINITY;

    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    if (sum > 0.f) {
        for (int s = 0; s < p.splits; ++s) {
            const float ls = p.lse_part[s * rows_total + R];
            if (ls == -INFINITY) continue;  // the split saw no key of this row
            const float w = exp2f((ls - lse) * kLog2e);
            const float* src = p.o_part + (s * rows_total + R) * D + lane * PER;
#pragma unroll
            for (int e = 0; e < PER; e += 2) {
                const float2 v = *reinterpret_cast<const float2*>(src + e);
                acc[e] = fmaf(w, v.x, acc[e]);
                acc[e + 1] = fmaf(w, v.y, acc[e + 1]);
            }
        }
    }
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + R * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
    if (lane == 0) p.lse[R] = lse;
}

template <int D>
cudaError_t launch_decode_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const DecodeParams& p, cudaStream_t stream, cudaEvent_t ev_start,
                            cudaEvent_t ev_stop) {
    using C = DecCfg<D>;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_decode_kernel<D>);
        e != cudaSuccess)
        return e;
    const dim3 grid(p.splits, p.H_kv * p.n_mtiles, p.B);  // splits in units of C::BN blocks
    if (ev_start) cudaEventRecord(ev_start, stream);
    fa_decode_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    if (ev_stop) cudaEventRecord(ev_stop, stream);
    if (p.splits > 1) {
        const size_t rows = (size_t)p.B * p.H * p.Nq;
        fa_decode_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

int decode_block_keys(int d) { return d == 64 ? DecCfg<64>::BN : d == 256 ? DecCfg<256>::BN : DecCfg<128>::BN; }
int decode_ctas_per_sm(int d) {
    return d == 64 ? DecCfg<64>::CTAS_PER_SM : d == 256 ? DecCfg<256>::CTAS_PER_SM : DecCfg<128>::CTAS_PER_SM;
}

cudaError_t launch_decode(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream,
                          cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    if (d == 64) return launch_decode_d<64>(tq, tk, tv, p, stream, ev_start, ev_stop);
    if (d == 256) return launch_decode_d<256>(tq, tk, tv, p, stream, ev_start, ev_stop);
    return launch_decode_d<128>(tq, tk, tv, p, stream, ev_start, ev_stop);
}

}  // namespace fa
