// fa_fwd_d256.cu -- fused exact-attention forward kernel for head dimension 256 (sm_100a).
//
// Same computation as fa_fwd.cu (tiled Q K^T, online softmax, P V, one pass, only O and lse
// written; FlashAttention (DE), "Tiling und blockweise Verarbeitung",
// "Online-Softmax-Berechnung"), for the 256-wide heads that FlashAttention (DE),
// "FlashAttention-2 (2023)" adds support for.  At d = 256 the accumulator O of one 128-row
// query tile alone fills 256 of the 512 tensor-memory columns, so a CTA holds ONE query tile
// and double-buffers the score block instead of ping-ponging two query tiles:
//
//   tensor memory:  S_a [0,128)  S_b [128,256)  O [256,512)
//   MMA order:      S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...
//
// S(j+1) is computed while the softmax works on S(j); P(j) is written as bf16 over the first
// 64 columns of its S buffer and read from there by PV(j); S(j+2) reuses the buffer after
// PV(j) (tcgen05 MMAs of one thread execute in issue order).  Per 128-key block the tensor
// pipe does 2 x 128 x 128 x 256 x 2 flop (~2048 cycles) against one softmax of 128 scores per
// row (~1900 cycles), so the kernel is bound by the tensor pipe and the K/V traffic, not by
// the exponentials.
//
// Shared memory: Q (4 chunks of 64 columns x 128 rows, 64 KB) and a ring of NSLOT 16 KB chunks
// that the TMA thread fills with K and V chunks in exactly the order the MMA thread consumes
// them (K0, K1, V0, K2, V1, K3, ...).  P V runs as four N = 64 MMAs per 16-key step, one per V
// chunk, so each V chunk is released as soon as its MMAs finish.
//
// Warp roles (192 threads): warps 0-3 softmax (thread r owns row r = TMEM lane r), warp 4 MMA
// issue (one thread) + TMEM allocation, warp 5 TMA (one thread).
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

struct Fwd256Cfg {
    static constexpr int D = 256;
    static constexpr int BM = 128;                   // query rows per CTA
    static constexpr int BN = 128;                   // keys per block
    static constexpr int KCH = D / 64;               // 64-column chunks per row
    static constexpr int CHUNK_BYTES = 128 * 128;    // one chunk: 128 rows x 128 bytes
    static constexpr int NSLOT = 10;                 // K/V chunk ring
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_RING = SMEM_Q + KCH * CHUNK_BYTES;
    static constexpr int SMEM_BAR = SMEM_RING + NSLOT * CHUNK_BYTES;
    // q, full[NSLOT], empty[NSLOT], sfull[2], pfull[2], ofull, done
    static constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 1 + 1;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + alignment slack
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_O = 256;
    __device__ static constexpr uint32_t tm_s(int buf) { return buf ? 128u : 0u; }
};
static_assert(Fwd256Cfg::SMEM_BYTES <= 232448, "shared memory over the sm_100 per-CTA limit");

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

template <bool PACKED>
__global__ void __launch_bounds__(192, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = Fwd256Cfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int cta_x = gridDim.x - 1 - blockIdx.x;  // heaviest (causal) query tiles first
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int bh = b * p.H + h;
    const int h_kv = h / (p.H / p.H_kv);            // grouped-query attention
    const int q0 = cta_x * C::BM;

    constexpr bool packed = PACKED;
    const SeqExtent ext = sequence_extent(p, b, threadIdx.x == 0 && h == 0 && cta_x == 0, packed);
    const int L = ext.L;
    if (q0 >= ext.Lq) return;
    // TMA coordinates (y, z) of row n: head-major (n, b*H + h); packed (h, t0 + n).
    auto q_y = [&](int n) { return packed ? h : n; };
    auto q_z = [&](int n) { return packed ? ext.t0 + n : bh; };
    auto kv_y = [&](int n) { return packed ? h_kv : n; };
    auto kv_z = [&](int n) { return packed ? ext.t0 + n : b * p.H_kv + h_kv; };
    // Key blocks this tile needs: keys j < lim, lim = min(L, last row + 1) if causal.
    const int lim_tile = p.causal ? min(L, q0 + C::BM) : L;
    const int nblk = (lim_tile + C::BN - 1) / C::BN;

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
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(bar_q, C::KCH * C::CHUNK_BYTES);
            for (int c = 0; c < C::KCH; ++c)
                tma_load_3d(smem + C::SMEM_Q + c * C::CHUNK_BYTES, &tmQ, bar_q, c * 64, q_y(q0),
                            q_z(q0));
            int u = 0;  // chunks issued into the ring
            bool ok = true;
            // One K or V block = KCH chunks, each into the next ring slot once it is free.
            auto load_block = [&](const CUtensorMap* map, int blk) {
                for (int c = 0; ok && c < C::KCH; ++c) {
                    const int s = u % C::NSLOT;
                    const uint32_t ph = (u / C::NSLOT) & 1;
                    if (!mbar_wait(&bar_empty[s], ph ^ 1, p.timeout_ns, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar_full[s], C::CHUNK_BYTES);
                    tma_load_3d(smem + C::SMEM_RING + s * C::CHUNK_BYTES, map, &bar_full[s],
                                c * 64, kv_y(blk * C::BN), kv_z(blk * C::BN));
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

            // S(buf) = Q K_blk^T: chunk c of K holds d columns [64c, 64c+64); both operands
            // K-major, 16-column steps are 32 bytes apart inside a swizzled 128-byte row.
            auto issue_S = [&](int buf) {
                for (int c = 0; c < C::KCH; ++c) {
                    const int s = u % C::NSLOT;
                    if (!mbar_wait(&bar_full[s], (u / C::NSLOT) & 1, p.timeout_ns, abort_flag))
                        return false;
                    tc_fence_after();
                    const uint32_t ka = sR + s * C::CHUNK_BYTES;
                    const uint32_t qa = sQ + c * C::CHUNK_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tmem + C::tm_s(buf), sdesc_sw128(qa + kk * 32, 16, 1024),
                               sdesc_sw128(ka + kk * 32, 16, 1024), idS,
                               (c > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_empty[s]);  // slot free once these MMAs have read it
                    ++u;
                }
                tc_commit(&bar_sfull[buf]);
                return true;
            };
            // O[:, 64c:64c+64] += P V_c for each chunk c of V: P (bf16, 2 per column, 8
            // columns per 16-key step) from tensor memory, V_c MN-major (16 key rows = 2048
            // bytes per step).
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

            bool ok = mbar_wait(bar_q, 0, p.timeout_ns, abort_flag);
            if (ok) ok = issue_S(0);
            if (ok && nblk > 1) ok = issue_S(1);
            for (int j = 0; ok && j < nblk; ++j) {
                const int buf = j & 1;
                if (!(ok = mbar_wait(&bar_pfull[buf], (j >> 1) & 1, p.timeout_ns, abort_flag)))
                    break;
                tc_fence_after();
                if (!(ok = issue_PV(buf, j > 0))) break;
                if (j + 2 < nblk && !(ok = issue_S(buf))) break;
            }
            if (!ok) fail();
            // Wait for every MMA issued here before tensor memory can be released.
            tc_commit(bar_done);
            mbar_wait_drain(bar_done, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroup
        const int r = threadIdx.x;  // row of the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t tO = tmem + lane_base + C::TM_O;
        const int row = q0 + r;
        const int lim = p.causal ? min(L, row + 1) : L;  // visible keys: j < lim
        const float c = p.scale_log2;
        float m = -INFINITY;  // running max of S * c (log2 units), possibly stale by <= 8
        float l = 0.f;        // running sum of exp2(S * c - m)
        bool ok = true;

        for (int j = 0; j < nblk; ++j) {
            const int buf = j & 1;
            const uint32_t tS = tmem + lane_base + C::tm_s(buf);
            ok = mbar_wait(&bar_sfull[buf], (j >> 1) & 1, p.timeout_ns, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[C::BN];
#pragma unroll
            for (int q = 0; q < C::BN / 32; ++q) tmem_ld32(tS + q * 32, s + q * 32);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < C::BN / 32; ++q) reg_fence32(s + q * 32);

            const int k0 = j * C::BN;
            if (k0 + C::BN > lim) {
#pragma unroll
                for (int i = 0; i < C::BN; ++i)
                    if (k0 + i >= lim) s[i] = __float_as_uint(-INFINITY);
            }
            // Row maximum as 8 independent chains, then a small tree.
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
            // alpha rescales what was accumulated under the old maximum (1 when it is kept).
            const float alpha = (grow && m != -INFINITY) ? ex2(m - m_new) : 1.0f;
            if (grow) {
                l *= alpha;
                m = m_new;
            }
            const float mb = (m == -INFINITY) ? 0.f : m;
            const float2 c2 = make_float2(c, c);
            const float2 nm2 = make_float2(-mb, -mb);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
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
                // Rescale this warp's rows of O once the previous P V has landed (PV(j) cannot
                // start before this thread's P(j) is published below).
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
            tc_fence_before();
            mbar_arrive(&bar_pfull[buf]);
        }

        // ------------------------------------------------------------ epilogue
        // Wait for every MMA (bar_done), not for the last phase of bar_ofull: with the score
        // block double-buffered this thread only knows that PV(nblk-3) has finished, so
        // bar_ofull may be two phases behind and a parity wait could not tell them apart.
        // (The rescale above is safe: S(j) completing implies PV(j-2) completed.)
        if (ok) ok = mbar_wait(bar_done, 0, p.timeout_ns, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
            const size_t o_off = row_of(packed, b, h, p.H, p.N, ext.t0, row < ext.Lq ? row : 0) * D;
            const bool in_range = row < ext.Lq && in_bounds(p.err, o_off, D, p.dbg.q);
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + o_off;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + q * 32, o);
                tmem_ld_wait();
                reg_fence32(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                       __uint_as_float(o[2 * i + 1]) * inv_l);
                if (in_range) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            const size_t l_off = lse_of(packed, b, h, p.H, p.N, p.T, ext.t0, row);
            if (in_range && in_bounds(p.err, l_off, 1, p.dbg.lse)) {
                // lse in natural-log units: (m + log2 l) * ln 2
                p.lse[l_off] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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

template <bool PACKED>
cudaError_t launch_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const FwdParams& p, int B, cudaStream_t stream) {
    using C = Fwd256Cfg;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_fwd_d256_kernel<PACKED>);
        e != cudaSuccess)
        return e;
    dim3 grid((p.N + C::BM - 1) / C::BM, p.H, B);
    fa_fwd_d256_kernel<PACKED><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int B, cudaStream_t stream) {
    return p.cu_seqlens != nullptr ? launch_d256<true>(tq, tk, tv, p, B, stream)
                                   : launch_d256<false>(tq, tk, tv, p, B, stream);
}

}  // namespace fa
