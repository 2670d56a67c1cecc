// fa_fwd_fp8.cu -- fused exact-attention forward kernel on FP8 (e4m3) inputs, head dim 128
// (sm_100a).  FlashAttention-3 added an FP8 mode (Russian article, "FlashAttention-3 (2024)":
// close to 1.2 PFLOP/s in FP8); here both products run as tcgen05 kind::f8f6f4 MMAs (e4m3
// operands, fp32 accumulators), at twice the bf16 tensor rate.
//
// Inputs are e4m3 codes with per-(batch, head) descale factors: q = code * q_descale, etc.
// The two score descales fold into the softmax constant c = scale * log2(e) * qd * kd, the
// value descale into the epilogue.  The structure is that of fa_fwd.cu (two 128-row query
// tiles per CTA in ping-pong, online softmax with P kept in tensor memory); what changes:
//   * a 128-wide e4m3 row is exactly one 128-byte swizzle row, so every tile is one TMA box
//     and one MMA K step covers 32 elements (still 32 bytes of the row);
//   * P is written to tensor memory as e4m3, four per 32-bit column (128 keys = 32 columns),
//     and read from there as the A operand of O += P V; V is the MN-major B operand (legal
//     for 8-bit types), straight from its TMA tile;
//   * P is scaled by 2^4 before rounding (p' = exp2(s c - m + 4)) under a rescale threshold of
//     4 (the running maximum may be stale by at most 4), so p' <= 2^8 stays inside e4m3's
//     range (448) while small probabilities keep 4 more binades above e4m3's underflow; the
//     row sum l' is accumulated from the unrounded fp32 p', and O = acc * v_descale / l'.
#include <cuda_bf16.h>

#include "fa_fwd_fp8.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

struct Fp8Cfg {
    static constexpr int D = 128;
    static constexpr int BM = 128;
    static constexpr int BN = 128;
    static constexpr int TILES = 2;
    static constexpr int ROWS_PER_CTA = BM * TILES;
    static constexpr int TILE_BYTES = 128 * 128;   // 128 rows x 128 one-byte elements
    static constexpr int STAGES = 4;
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_K = SMEM_Q + TILES * TILE_BYTES;
    static constexpr int SMEM_V = SMEM_K + STAGES * TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_V + STAGES * TILE_BYTES;
    static constexpr int NUM_BARS = 1 + 4 * STAGES + 2 + 2 + 2 + 2 + 1;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_SOFTMAX = 224, REGS_OTHER = 56;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr float THRESH = 4.0f;          // rescale when the maximum grew by more
    static constexpr float P_OFFSET = 4.0f;        // p' = p * 2^P_OFFSET
    __device__ static constexpr uint32_t tm_s(int t) { return t ? 128u : 0u; }
    __device__ static constexpr uint32_t tm_o(int t) { return t ? 384u : 256u; }
};
static_assert(Fp8Cfg::SMEM_BYTES <= 232448, "shared memory over the sm_100 per-CTA limit");

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B and an fp32 accumulator
// (format code 0 = E4M3; b_mn selects the MN-major B layout).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool b_mn) {
    return (1u << 4)                        // D format: f32
           | (0u << 7) | (0u << 10)         // A, B format: e4m3
           | ((b_mn ? 1u : 0u) << 16)       // B major
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// D(tmem) = A(smem) * B(smem) (+ D), kind::f8f6f4.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D(tmem) = A(tmem) * B(smem) (+ D), kind::f8f6f4 (A K-major in tensor memory).
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four floats -> four e4m3 bytes (round to nearest even, saturating), x0 in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float x0, float x1, float x2, float x3) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
    return r;
}

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__global__ void __launch_bounds__(384, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Fp8Params p) {
    using C = Fp8Cfg;
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
    const int bh_kv = b * p.H_kv + h / (p.H / p.H_kv);
    const int q_base = cta_x * C::ROWS_PER_CTA;

    int L = p.N;
    if (p.seqlens != nullptr && in_bounds(p.err, b, 1, p.dbg.nseq)) {
        L = p.seqlens[b];
        if (L < 1 || L > p.N) {
            if (threadIdx.x == 0 && h == 0 && cta_x == 0) record_error(p.err, kErrInvalidArg);
            L = L < 1 ? 1 : p.N;
        }
    }
    auto blocks_for = [&](int row_end) {
        const int lim = p.causal ? min(L, row_end) : L;
        return (lim + C::BN - 1) / C::BN;
    };
    const int nblk0 = blocks_for(q_base + C::BM);
    const int nblk1 = blocks_for(q_base + 2 * C::BM);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_kfull = bars + 1;
    uint64_t* bar_kempty = bar_kfull + C::STAGES;
    uint64_t* bar_vfull = bar_kempty + C::STAGES;
    uint64_t* bar_vempty = bar_vfull + C::STAGES;
    uint64_t* bar_sfull = bar_vempty + C::STAGES;  // [2]
    uint64_t* bar_pfull = bar_sfull + 2;            // [2]
    uint64_t* bar_ofull = bar_pfull + 2;            // [2]
    uint64_t* bar_phalf = bar_ofull + 2;            // [2] P of the block's first 64 keys
    uint64_t* bar_done = bar_phalf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
            mbar_init(&bar_vfull[s], 1);
            mbar_init(&bar_vempty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bar_sfull[t], 1);
            mbar_init(&bar_pfull[t], C::BM);
            mbar_init(&bar_phalf[t], C::BM);
            mbar_init(&bar_ofull[t], 1);
        }
        mbar_init(bar_done, 1);
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

    if (warp >= 8) {
      regs_decrease<C::REGS_OTHER>();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(bar_q, C::TILES * C::TILE_BYTES);
            for (int t = 0; t < C::TILES; ++t)
                tma_load_3d(smem + C::SMEM_Q + t * C::TILE_BYTES, &tmQ, bar_q, 0,
                            q_base + t * C::BM, bh);
            const int n = nblk1;
            for (int j = 0; j < n; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                if (!mbar_wait(&bar_kempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&bar_kfull[s], C::TILE_BYTES);
                tma_load_3d(smem + C::SMEM_K + s * C::TILE_BYTES, &tmK, &bar_kfull[s], 0,
                            j * C::BN, bh_kv);
                if (!mbar_wait(&bar_vempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&bar_vfull[s], C::TILE_BYTES);
                tma_load_3d(smem + C::SMEM_V + s * C::TILE_BYTES, &tmV, &bar_vfull[s], 0,
                            j * C::BN, bh_kv);
            }
            for (int j = max(0, n - C::STAGES); j < n; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                mbar_wait_drain(&bar_kfull[s], ph, p.timeout_ns);
                mbar_wait_drain(&bar_vfull[s], ph, p.timeout_ns);
            }
            if (!mbar_wait_drain(bar_q, 0, p.timeout_ns)) fail();
        }
      } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_e4m3(C::BM, C::BN, false);
            constexpr uint32_t idPV = idesc_e4m3(C::BM, D, true);
            const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
            const uint32_t sK = smem_u32(smem + C::SMEM_K);
            const uint32_t sV = smem_u32(smem + C::SMEM_V);
            const int n0 = nblk0, n1 = nblk1;

            // S_t = Q_t K^T: both operands K-major; one K step = 32 e4m3 = 32 bytes.
            auto issue_S = [&](int t, int s) {
                const uint32_t qa = sQ + t * C::TILE_BYTES;
                const uint32_t ka = sK + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    mma_ss_f8(tmem + C::tm_s(t), sdesc_sw128(qa + kk * 32, 16, 1024),
                              sdesc_sw128(ka + kk * 32, 16, 1024), idS, kk > 0 ? 1u : 0u);
            };
            // O_t += P_t V over the keys of one half of the block: P (e4m3, 4 per column, 8
            // columns per 32-key step) from tensor memory, V MN-major (32 key rows = 4096 bytes
            // per step).  The softmax releases P in two halves, so the first half's MMAs run
            // while it computes the second half's exponentials.
            auto issue_PV = [&](int t, int s, bool accumulate, int half) {
                const uint32_t va = sV + s * C::TILE_BYTES;
#pragma unroll
                for (int kk = half * C::BN / 64; kk < (half + 1) * C::BN / 64; ++kk)
                    mma_ts_f8(tmem + C::tm_o(t), tmem + C::tm_s(t) + kk * 8,
                              sdesc_sw128(va + kk * 4096, C::TILE_BYTES, 1024), idPV,
                              (accumulate || kk > 0) ? 1u : 0u);
            };

            auto wait_issue_PV = [&](int t, int s, int j) {
                if (!mbar_wait(&bar_phalf[t], j & 1, p.timeout_ns, abort_flag)) return false;
                tc_fence_after();
                issue_PV(t, s, j > 0, 0);
                if (!mbar_wait(&bar_pfull[t], j & 1, p.timeout_ns, abort_flag)) return false;
                tc_fence_after();
                issue_PV(t, s, true, 1);
                return true;
            };

            bool ok = mbar_wait(bar_q, 0, p.timeout_ns, abort_flag);
            if (ok) ok = mbar_wait(&bar_kfull[0], 0, p.timeout_ns, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_S(0, 0);
                tc_commit(&bar_sfull[0]);
                issue_S(1, 0);
                tc_commit(&bar_sfull[1]);
                tc_commit(&bar_kempty[0]);
            }
            for (int j = 0; ok && j < n1; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                const int jn = j + 1;
                const int sn = jn % C::STAGES;
                const uint32_t phn = (jn / C::STAGES) & 1;
                if (!(ok = mbar_wait(&bar_vfull[s], ph, p.timeout_ns, abort_flag))) break;
                if (j < n0) {
                    if (!(ok = wait_issue_PV(0, s, j))) break;
                    tc_commit(&bar_ofull[0]);
                }
                if (jn < n1) {
                    if (!(ok = mbar_wait(&bar_kfull[sn], phn, p.timeout_ns, abort_flag))) break;
                    tc_fence_after();
                    if (jn < n0) {
                        issue_S(0, sn);
                        tc_commit(&bar_sfull[0]);
                    }
                }
                if (!(ok = wait_issue_PV(1, s, j))) break;
                tc_commit(&bar_ofull[1]);
                tc_commit(&bar_vempty[s]);
                if (jn < n1) {
                    issue_S(1, sn);
                    tc_commit(&bar_sfull[1]);
                    tc_commit(&bar_kempty[sn]);
                }
            }
            if (!ok) fail();
            tc_commit(bar_done);
            mbar_wait_drain(bar_done, 0, p.timeout_ns);
        }
      }
    } else {
        regs_increase<C::REGS_SOFTMAX>();
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp / 4;
        const int r = threadIdx.x % C::BM;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::tm_s(t);
        const uint32_t tO = tmem + lane_base + C::tm_o(t);
        const int nt = t ? nblk1 : nblk0;
        const int row = q_base + t * C::BM + r;
        const int lim = p.causal ? min(L, row + 1) : L;
        const float qd = p.q_descale && in_bounds(p.err, bh, 1, p.dbg.heads_q) ? p.q_descale[bh] : 1.0f;
        const float kd = p.k_descale && in_bounds(p.err, bh_kv, 1, p.dbg.heads_kv)
                             ? p.k_descale[bh_kv] : 1.0f;
        const float c = p.scale_log2 * qd * kd;  // scores of the codes -> log2 units
        float m = -INFINITY;  // running max of S * c, possibly stale by <= THRESH
        float l = 0.f;        // running sum of p' = exp2(S * c - m + P_OFFSET)
        bool ok = true;

        for (int j = 0; j < nt; ++j) {
            ok = mbar_wait(&bar_sfull[t], j & 1, p.timeout_ns, abort_flag);
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
            const bool grow = m_new > m + C::THRESH;  // false while both are -inf
            const float alpha = (grow && m != -INFINITY) ? ex2(m - m_new) : 1.0f;
            if (grow) {
                l *= alpha;
                m = m_new;
            }
            if (__any_sync(0xffffffffu, grow && j > 0)) {
                // Rescale this warp's rows of O before any of P(j) is released (S(j) done
                // implies the previous P V of this tile is done: the MMAs run in issue order).
                ok = mbar_wait(&bar_ofull[t], (j - 1) & 1, p.timeout_ns, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
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
            const float mb = (m == -INFINITY) ? 0.f : m - C::P_OFFSET;
            const float2 c2 = make_float2(c, c);
            const float2 nm2 = make_float2(-mb, -mb);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            // P' (e4m3) over the first 32 columns of S, already read, in two halves of 64 keys,
            // each released to the MMA thread as soon as it is stored.
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e0 = 64 * hh + 4 * i;
                    const float2 xa = ffma2(make_float2(__uint_as_float(s[e0]),
                                                        __uint_as_float(s[e0 + 1])), c2, nm2);
                    const float2 xb = ffma2(make_float2(__uint_as_float(s[e0 + 2]),
                                                        __uint_as_float(s[e0 + 3])), c2, nm2);
                    const float2 ea = make_float2(ex2(xa.x), ex2(xa.y));
                    const float2 eb = make_float2(ex2(xb.x), ex2(xb.y));
                    acc[(2 * i) % 4] = fadd2(acc[(2 * i) % 4], ea);
                    acc[(2 * i + 1) % 4] = fadd2(acc[(2 * i + 1) % 4], eb);
                    pk[i] = pack_e4m3x4(ea.x, ea.y, eb.x, eb.y);
                }
                tmem_st16(tS + 16 * hh, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(hh == 0 ? &bar_phalf[t] : &bar_pfull[t]);
            }
            l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                 ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        }

        // ------------------------------------------------------------ epilogue
        if (ok) ok = mbar_wait(&bar_ofull[t], (nt - 1) & 1, p.timeout_ns, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const float vd = p.v_descale && in_bounds(p.err, bh_kv, 1, p.dbg.heads_kv)
                                 ? p.v_descale[bh_kv] : 1.0f;
            const float mul = l > 0.f ? vd / l : 0.f;
            const size_t o_off = ((size_t)bh * p.N + (row < p.N ? row : 0)) * D;
            const bool in_range = row < p.N && in_bounds(p.err, o_off, D, p.dbg.q);
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + o_off;
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + q * 32, o);
                tmem_ld_wait();
                reg_fence32(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * mul,
                                       __uint_as_float(o[2 * i + 1]) * mul);
                if (in_range) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            if (in_range && in_bounds(p.err, (size_t)bh * p.N + row, 1, p.dbg.lse)) {
                // l' carries the 2^P_OFFSET of p': lse = (m + log2 l' - P_OFFSET) * ln 2
                p.lse[(size_t)bh * p.N + row] =
                    l > 0.f ? (m + __log2f(l) - C::P_OFFSET) * 0.69314718055994531f : -INFINITY;
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

}  // namespace

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const Fp8Params& p, int B, cudaStream_t stream) {
    using C = Fp8Cfg;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_fwd_fp8_kernel);
        e != cudaSuccess)
        return e;
    dim3 grid((p.N + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA, p.H, B);
    fa_fwd_fp8_kernel<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace fa
