// fa_fwd.cu -- fused exact-attention forward kernel for sm_100a.
//
// One CTA owns two 128-row query tiles of one (batch, head) and streams that head's keys and
// values through shared memory in 128-row blocks, never writing the score matrix to device
// memory (FlashAttention (DE), "Tiling und blockweise Verarbeitung"; "Zusammenfassen von
// Operationen in einem CUDA-Kernel").  Per key block j and query tile t:
//
//   S_t   = Q_t K_j^T                       tcgen05 MMA, fp32 accumulator in tensor memory
//   m'    = max(m, rowmax(S_t) * c)         c = scale * log2(e)
//   P_t   = exp2(S_t * c - m')              bf16, written back over S_t in tensor memory
//   l     = alpha * l + rowsum(P_t)         alpha = exp2(m - m')
//   O_t   = alpha * O_t + P_t V_j           tcgen05 MMA with A read from tensor memory
//
// which is the online softmax of FlashAttention (DE), "Online-Softmax-Berechnung": a running
// maximum and a running sum of exponentials, rescaled block by block, so that the final
// O_t / l equals the two-pass softmax exactly (up to rounding).  The rescale of O is skipped
// while the running maximum has grown by at most 8 (in log2 units): the stale maximum is then
// used for both l and O, which stays exact because both share it, and keeps every
// exponential below 2^8.
//
// Warp roles (384 threads = 3 warpgroups):
//   warps 0-3  softmax for query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax for query tile 1
//   warp  8    MMA issue (one thread) + TMEM allocation
//   warp  9    TMA producer (one thread)
//   warps 10-11 idle
// The third warpgroup hands most of its registers to the two softmax warpgroups
// (setmaxnreg: 56 + 2 x 224 per thread slot = 3 x 168 launched; 72 + 2 x 216 in the packed-sequence
// kernel, whose MMA thread spilled at 56).
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d).
// Shared memory: Q0, Q1, and a ring of K and V blocks, all 128-byte swizzled by TMA.
#include "fa_internal.h"
#include "sm100.cuh"

// The softmax releases each block's P to the MMA thread in this many parts of BN / parts keys,
// so that the P V MMAs of the first parts run while it computes the later ones.
#ifndef FA_FWD_P_PARTS
#define FA_FWD_P_PARTS 2
#endif

namespace fa {
namespace {

using namespace sm100;

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                 // query rows per tile
    static constexpr int BN = 128;                 // keys per block
    static constexpr int TILES = 2;                // query tiles per CTA
    static constexpr int ROWS_PER_CTA = BM * TILES;
    static constexpr int KCH = D / 64;             // 64-column (128-byte) chunks per row
    static constexpr int STAGES = (D == 128) ? 2 : 3;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int KV_TILE_BYTES = BN * D * 2;
    static constexpr int CHUNK_BYTES = 128 * 128;  // one 64-column chunk of a 128-row tile
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_K = SMEM_Q + TILES * Q_TILE_BYTES;
    static constexpr int SMEM_V = SMEM_K + STAGES * KV_TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_V + STAGES * KV_TILE_BYTES;
    static constexpr int P_PARTS = FA_FWD_P_PARTS;  // P released in parts of BN / P_PARTS keys
    static_assert(P_PARTS == 2 || P_PARTS == 4, "P is released in halves or quarters");
    // q, k/v full and empty per stage, s/p/o full per tile, P parts, done, and the persistent
    // kernel's Q-empty barrier
    static constexpr int NUM_BARS = 1 + 4 * STAGES + 2 + 2 + 2 + 2 * (P_PARTS - 1) + 1 + 1;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + alignment slack
    static constexpr int THREADS = 384;
    static constexpr uint32_t REGS_SOFTMAX = 224, REGS_OTHER = 56;
    // packed sequences: 56 registers spilled the MMA thread's loop state (72 measured +6 %; the
    // head-major kernels measured 2 % slower with it)
    static constexpr uint32_t REGS_SOFTMAX_PACKED = 216, REGS_OTHER_PACKED = 72;
    // The persistent kernel's MMA and TMA threads carry loop state across units and spill at
    // 56 registers; there the split is 2 x 208 + 88 (the same 3 x 168 launched).
#ifndef FA_FWD_PERSIST_REGS_SOFTMAX
#define FA_FWD_PERSIST_REGS_SOFTMAX 208
#endif
    static constexpr uint32_t REGS_SOFTMAX_PERSIST = FA_FWD_PERSIST_REGS_SOFTMAX;
    static constexpr uint32_t REGS_OTHER_PERSIST = 504 - 2 * REGS_SOFTMAX_PERSIST;
    static constexpr uint32_t REGS_LAUNCH = 168;  // per thread at launch (65536 / 384, rounded to 8)
    static_assert(2 * REGS_SOFTMAX + REGS_OTHER == 3 * REGS_LAUNCH, "register split");
    static_assert(2 * REGS_SOFTMAX_PACKED + REGS_OTHER_PACKED == 3 * REGS_LAUNCH, "register split");
    static_assert(2 * REGS_SOFTMAX_PERSIST + REGS_OTHER_PERSIST == 3 * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;
    // tensor-memory column of S_t / O_t for query tile t
    __device__ static constexpr uint32_t tm_s(int t) { return t ? 128u : 0u; }
    __device__ static constexpr uint32_t tm_o(int t) { return t ? 256u + D : 256u; }
};

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// Query tile pair cta_x of head (b, h), heaviest causal tiles first.  Causal head-major: the
// launch order walks groups of up to 16 heads and, within a group, all heads' tiles from the
// heaviest to the lightest, so the last wave holds light tiles only while one group's K and V
// (2 N d bf16 per head) stay in L2.  The CTA indices are read with volatile moves so that the
// epilogue recomputes (b, h) instead of keeping them live through the softmax loop.
struct CtaCoords {
    int cta_x, h, b;
};
__device__ __forceinline__ CtaCoords cta_coords(bool grouped) {
    uint32_t bx, by, bz, nx, ny, nz;
    asm volatile("mov.u32 %0, %%ctaid.x;" : "=r"(bx));
    asm volatile("mov.u32 %0, %%ctaid.y;" : "=r"(by));
    asm volatile("mov.u32 %0, %%ctaid.z;" : "=r"(bz));
    asm volatile("mov.u32 %0, %%nctaid.x;" : "=r"(nx));
    asm volatile("mov.u32 %0, %%nctaid.y;" : "=r"(ny));
    asm volatile("mov.u32 %0, %%nctaid.z;" : "=r"(nz));
    CtaCoords c;
    if (grouped) {
        constexpr int GH = 16;
        const int BH = (int)(ny * nz);
        const int lin = (int)(bx + nx * (by + ny * bz));
        const int g0 = lin / ((int)nx * GH) * GH;
        const int gh = min(GH, BH - g0);     // heads in this group
        const int r = lin - g0 * (int)nx;    // rank-major position inside the group
        const int flat = g0 + r % gh;
        c.cta_x = (int)nx - 1 - r / gh;
        c.h = flat % (int)ny;
        c.b = flat / (int)ny;
    } else {
        c.cta_x = (int)(nx - 1 - bx);
        c.h = (int)by;
        c.b = (int)bz;
    }
    return c;
}

// An opaque copy of v: values derived from it are recomputed where they are used instead of
// being kept live across the loop in between.
__device__ __forceinline__ int opaque(int v) {
    int r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

template <int D, bool PACKED, bool GROUPED>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // GROUPED (head-major causal launches): the grouped heaviest-first order; otherwise tile
    // pair gridDim.x - 1 - blockIdx.x (heaviest first) of head (blockIdx.z, blockIdx.y).
    const CtaCoords cc = GROUPED ? cta_coords(true)
                                 : CtaCoords{(int)(gridDim.x - 1 - blockIdx.x), (int)blockIdx.y,
                                             (int)blockIdx.z};
    const int cta_x = cc.cta_x;
    const int h = cc.h;
    const int b = cc.b;
    const int bh = b * p.H + h;
    // Grouped-query attention: consecutive query heads share one key/value head.
    const int h_kv = h / (p.H / p.H_kv);
    const int q_base = cta_x * C::ROWS_PER_CTA;

    constexpr bool packed = PACKED;
    const SeqExtent ext = sequence_extent(p, b, threadIdx.x == 0 && h == 0 && cta_x == 0, packed);
    const int L = ext.L;
    // Packed sequences shorter than the longest one leave whole CTAs without query rows.
    if (q_base >= ext.Lq) return;
    // TMA coordinates (y, z) of row n: head-major (n, b*H + h); packed (h, t0 + n).
    auto q_y = [&](int n) { return packed ? h : n; };
    auto q_z = [&](int n) { return packed ? ext.t0 + n : bh; };
    auto kv_y = [&](int n) { return packed ? h_kv : n; };
    auto kv_z = [&](int n) { return packed ? ext.t0 + n : b * p.H_kv + h_kv; };
    // Key blocks each query tile needs: keys j < lim, lim = min(L, last row + 1) if causal.
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
    uint64_t* bar_ppart = bar_ofull + 2;            // [2][P_PARTS-1] P of all but the last part
    uint64_t* bar_done = bar_ppart + 2 * (C::P_PARTS - 1);  // every MMA of this CTA finished
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
            mbar_init(&bar_ofull[t], 1);
            for (int q = 0; q + 1 < C::P_PARTS; ++q) mbar_init(&bar_ppart[t * (C::P_PARTS - 1) + q], C::BM);
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
      regs_set<PACKED ? C::REGS_OTHER_PACKED : C::REGS_OTHER, C::REGS_LAUNCH>();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(bar_q, C::TILES * C::Q_TILE_BYTES);
            for (int t = 0; t < C::TILES; ++t)
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(smem + C::SMEM_Q + t * C::Q_TILE_BYTES + c * C::CHUNK_BYTES, &tmQ,
                                bar_q, c * 64, q_y(q_base + t * C::BM), q_z(q_base + t * C::BM));
            const int n = nblk1;
            for (int j = 0; j < n; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                if (!mbar_wait(&bar_kempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&bar_kfull[s], C::KV_TILE_BYTES);
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(smem + C::SMEM_K + s * C::KV_TILE_BYTES + c * C::CHUNK_BYTES, &tmK,
                                &bar_kfull[s], c * 64, kv_y(j * C::BN), kv_z(j * C::BN));
                if (!mbar_wait(&bar_vempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&bar_vfull[s], C::KV_TILE_BYTES);
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(smem + C::SMEM_V + s * C::KV_TILE_BYTES + c * C::CHUNK_BYTES, &tmV,
                                &bar_vfull[s], c * 64, kv_y(j * C::BN), kv_z(j * C::BN));
            }
            // Do not leave the CTA while our copies may still be landing in shared memory.
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
            constexpr uint32_t idS = idesc_bf16(C::BM, C::BN, false, false);
            constexpr uint32_t idPV = idesc_bf16(C::BM, D, false, true);
            const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
            const uint32_t sK = smem_u32(smem + C::SMEM_K);
            const uint32_t sV = smem_u32(smem + C::SMEM_V);
            const int n0 = nblk0, n1 = nblk1;

            // S_t = Q_t K^T: both operands K-major; 16-column K steps walk the swizzled rows
            // (32 bytes per step) and then the next 64-column chunk.
            auto issue_S = [&](int t, int s) {
                const uint32_t qa = sQ + t * C::Q_TILE_BYTES;
                const uint32_t ka = sK + s * C::KV_TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32;
                    mma_ss(tmem + C::tm_s(t), sdesc_sw128(qa + off, 16, 1024),
                           sdesc_sw128(ka + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
            };
            // O_t += P_t V over the keys of part `part` (BN / P_PARTS keys): P from tensor memory
            // (2 bf16 per column, 8 columns per K step of 16 keys), V MN-major in shared memory
            // (16 key rows = 2048 bytes per K step; the two 64-column chunks of d are
            // CHUNK_BYTES apart).  The softmax releases P part by part, so the first parts'
            // MMAs run while it computes the later parts' exponentials.
            constexpr int KK_PART = C::BN / 16 / C::P_PARTS;  // K steps per part
            auto issue_PV = [&](int t, int s, bool accumulate, int part) {
                const uint32_t va = sV + s * C::KV_TILE_BYTES;
#pragma unroll
                for (int kk = part * KK_PART; kk < (part + 1) * KK_PART; ++kk) {
                    mma_ts(tmem + C::tm_o(t), tmem + C::tm_s(t) + kk * 8,
                           sdesc_sw128(va + kk * 2048, C::CHUNK_BYTES, 1024), idPV,
                           (accumulate || kk > 0) ? 1u : 0u);
                }
            };
            auto wait_issue_PV = [&](int t, int s, int j) {
#pragma unroll
                for (int part = 0; part < C::P_PARTS; ++part) {
                    uint64_t* bar = part + 1 < C::P_PARTS
                                        ? &bar_ppart[t * (C::P_PARTS - 1) + part]
                                        : &bar_pfull[t];
                    if (!mbar_wait(bar, j & 1, p.timeout_ns, abort_flag)) return false;
                    tc_fence_after();
                    issue_PV(t, s, j > 0 || part > 0, part);
                }
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
            // Wait for every MMA issued here before tensor memory can be released.
            tc_commit(bar_done);
            mbar_wait_drain(bar_done, 0, p.timeout_ns);
        }
      }
    } else {
        regs_set<PACKED ? C::REGS_SOFTMAX_PACKED : C::REGS_SOFTMAX, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp / 4;
        const int r = threadIdx.x % C::BM;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::tm_s(t);
        const uint32_t tO = tmem + lane_base + C::tm_o(t);
        const int nt = t ? nblk1 : nblk0;
        const int row = q_base + t * C::BM + r;
        const int lim = p.causal ? min(L, row + 1) : L;  // visible keys: j < lim
        const float c = p.scale_log2;
        float m = -INFINITY;  // running max of S * c (log2 units), possibly stale by <= 8
        float l = 0.f;        // running sum of exp2(S * c - m)
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
            const float mx = mx8[0];
            const float m_new = fmaxf(m, mx * c);
            const bool grow = m_new > m + 8.0f;  // false while both are -inf
            // alpha rescales what was accumulated under the old maximum (1 when it is kept).
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
            const float mb = (m == -INFINITY) ? 0.f : m;
            // p = exp2(S * c - m): the argument as packed two-wide FMAs, the exponential on the
            // MUFU unit, the row sum in 4 packed accumulators (8 independent chains).  P goes to
            // tensor memory in P_PARTS parts, over S columns already read; each part is
            // released to the MMA thread as soon as it is stored.
            const float2 c2 = make_float2(c, c);
            const float2 nm2 = make_float2(-mb, -mb);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            constexpr int WP = C::BN / 2 / C::P_PARTS;  // packed P words per part
#pragma unroll
            for (int part = 0; part < C::P_PARTS; ++part) {
                uint32_t pk[WP];
#pragma unroll
                for (int i = 0; i < WP; ++i) {
                    const int e0 = part * 2 * WP + 2 * i;
                    const float2 x = ffma2(make_float2(__uint_as_float(s[e0]),
                                                       __uint_as_float(s[e0 + 1])), c2, nm2);
                    const float2 e = make_float2(ex2(x.x), ex2(x.y));
                    acc[i % 4] = fadd2(acc[i % 4], e);
                    pk[i] = pack_bf16x2(e.x, e.y);
                }
                if constexpr (WP == 32) tmem_st32(tS + part * WP, pk);
                else tmem_st16(tS + part * WP, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(part + 1 < C::P_PARTS ? &bar_ppart[t * (C::P_PARTS - 1) + part]
                                                  : &bar_pfull[t]);
            }
            l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                 ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        }

        // ------------------------------------------------------------ epilogue
        if (ok) ok = mbar_wait(&bar_ofull[t], (nt - 1) & 1, p.timeout_ns, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const CtaCoords ce = GROUPED ? cta_coords(true) : CtaCoords{cta_x, h, b};  // (b, h) recomputed
            const float inv_l = l > 0.f ? 1.0f / l : 0.f;
            const size_t o_off = row_of(packed, ce.b, ce.h, p.H, p.N, ext.t0, row < ext.Lq ? row : 0) * D;
            const bool in_range = row < ext.Lq && in_bounds(p.err, o_off, D, p.dbg.q);
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
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                       __uint_as_float(o[2 * i + 1]) * inv_l);
                if (in_range) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            const size_t l_off = lse_of(packed, ce.b, ce.h, p.H, p.N, p.T, ext.t0, row);
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
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Persistent forward for head-major launches without per-sequence key lengths.  One CTA per SM
// walks the units blockIdx.x, blockIdx.x + gridDim.x, ...: without a causal mask every unit
// costs the same and they go head by head (tile pair x of head bh, so a few heads' K and V stay
// in L2); with one, tile pair x needs x + 1 key blocks per tile and the units go heaviest
// first across all heads (every head's last pair, then every head's second-to-last, ...), so
// the static round robin ends on the lightest units.  Per key block the arithmetic is fa_fwd_kernel's; across
// units the K/V ring and every barrier phase carry over, the Q tiles are reloaded as soon as the
// previous unit's last score MMA has completed (bar_qempty), and a unit's epilogue overlaps the
// next unit's Q load and first score MMAs.  A unit's first P V of tile t overwrites O_t only
// after the softmax threads of tile t have read O_t in their epilogue: they release P_t(0) of
// the next unit after that.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_persist_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // The mask flag: a template argument at d = 64; read at run time at d = 128, where that
    // build (one kernel for both cases) measured 2-9 % faster without the mask (its register
    // allocation differs) and no slower with it.
    const bool causal = (D == 128) ? p.causal : CAUSAL;
    const int nx = (p.N + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA;  // tile pairs per head
    const int BH = p.B * p.H;
    const int n_units = nx * BH;
    const int nblk = (p.N + C::BN - 1) / C::BN;  // key blocks of an unmasked query tile
    // Unit lin: head bh and first query row; key blocks of tile t (rows up to q_base + 128 t
    // + 127 see keys j < min(N, last row + 1) under the causal mask).
    struct Unit {
        int bh, q_base, n0, n1;
    };
    auto unit = [&](int lin) {
        Unit u;
        int x;
        if (causal) {
            x = nx - 1 - lin / BH;
            u.bh = lin - (lin / BH) * BH;
        } else {
            u.bh = lin / nx;
            x = lin - u.bh * nx;
        }
        u.q_base = x * C::ROWS_PER_CTA;
        u.n0 = causal ? (min(p.N, u.q_base + C::BM) + C::BN - 1) / C::BN : nblk;
        u.n1 = causal ? (min(p.N, u.q_base + 2 * C::BM) + C::BN - 1) / C::BN : nblk;
        return u;
    };

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_kfull = bars + 1;
    uint64_t* bar_kempty = bar_kfull + C::STAGES;
    uint64_t* bar_vfull = bar_kempty + C::STAGES;
    uint64_t* bar_vempty = bar_vfull + C::STAGES;
    uint64_t* bar_sfull = bar_vempty + C::STAGES;  // [2]
    uint64_t* bar_pfull = bar_sfull + 2;            // [2]
    uint64_t* bar_ofull = bar_pfull + 2;            // [2]
    uint64_t* bar_ppart = bar_ofull + 2;            // [2][P_PARTS-1]
    uint64_t* bar_done = bar_ppart + 2 * (C::P_PARTS - 1);
    uint64_t* bar_qempty = bar_done + 1;  // the unit's score MMAs are done: Q may be reloaded
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
            mbar_init(&bar_ofull[t], 1);
            for (int q = 0; q + 1 < C::P_PARTS; ++q) mbar_init(&bar_ppart[t * (C::P_PARTS - 1) + q], C::BM);
        }
        mbar_init(bar_done, 1);
        mbar_init(bar_qempty, 1);
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
      regs_set<C::REGS_OTHER_PERSIST, C::REGS_LAUNCH>();
      if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            int g = 0;   // K/V blocks whose V copy was issued (position in the ring)
            int gk = 0;  // K copies issued
            int uc = 0;  // units started
            bool ok = true;
            for (int lin = blockIdx.x; ok && lin < n_units; lin += gridDim.x, ++uc) {
                const Unit u = unit(lin);
                const int bh = u.bh, q_base = u.q_base;
                const int bkv = (bh / p.H) * p.H_kv + (bh % p.H) / (p.H / p.H_kv);
                if (uc > 0 && !(ok = mbar_wait(bar_qempty, (uc - 1) & 1, p.timeout_ns, abort_flag)))
                    break;
                mbar_arrive_expect_tx(bar_q, C::TILES * C::Q_TILE_BYTES);
                for (int t = 0; t < C::TILES; ++t)
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(smem + C::SMEM_Q + t * C::Q_TILE_BYTES + c * C::CHUNK_BYTES,
                                    &tmQ, bar_q, c * 64, q_base + t * C::BM, bh);
                for (int j = 0; j < u.n1; ++j, ++g) {
                    const int s = g % C::STAGES;
                    const uint32_t ph = (g / C::STAGES) & 1;
                    if (!(ok = mbar_wait(&bar_kempty[s], ph ^ 1, p.timeout_ns, abort_flag))) break;
                    mbar_arrive_expect_tx(&bar_kfull[s], C::KV_TILE_BYTES);
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(smem + C::SMEM_K + s * C::KV_TILE_BYTES + c * C::CHUNK_BYTES,
                                    &tmK, &bar_kfull[s], c * 64, j * C::BN, bkv);
                    ++gk;
                    if (!(ok = mbar_wait(&bar_vempty[s], ph ^ 1, p.timeout_ns, abort_flag))) break;
                    mbar_arrive_expect_tx(&bar_vfull[s], C::KV_TILE_BYTES);
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(smem + C::SMEM_V + s * C::KV_TILE_BYTES + c * C::CHUNK_BYTES,
                                    &tmV, &bar_vfull[s], c * 64, j * C::BN, bkv);
                }
            }
            if (!ok) fail();
            // Do not leave while our copies may still be landing in shared memory: the last
            // STAGES K and V copies issued, and the last Q copy.
            for (int j = max(0, gk - C::STAGES); j < gk; ++j)
                mbar_wait_drain(&bar_kfull[j % C::STAGES], (j / C::STAGES) & 1, p.timeout_ns);
            for (int j = max(0, g - C::STAGES); j < g; ++j)
                mbar_wait_drain(&bar_vfull[j % C::STAGES], (j / C::STAGES) & 1, p.timeout_ns);
            if (uc > 0 && !mbar_wait_drain(bar_q, (uc - 1) & 1, p.timeout_ns)) fail();
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(C::BM, C::BN, false, false);
            constexpr uint32_t idPV = idesc_bf16(C::BM, D, false, true);
            const uint32_t sQ = smem_u32(smem + C::SMEM_Q);
            const uint32_t sK = smem_u32(smem + C::SMEM_K);
            const uint32_t sV = smem_u32(smem + C::SMEM_V);
            auto issue_S = [&](int t, int s) {
                const uint32_t qa = sQ + t * C::Q_TILE_BYTES;
                const uint32_t ka = sK + s * C::KV_TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32;
                    mma_ss(tmem + C::tm_s(t), sdesc_sw128(qa + off, 16, 1024),
                           sdesc_sw128(ka + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
            };
            constexpr int KK_PART = C::BN / 16 / C::P_PARTS;
            auto issue_PV = [&](int t, int s, bool accumulate, int part) {
                const uint32_t va = sV + s * C::KV_TILE_BYTES;
#pragma unroll
                for (int kk = part * KK_PART; kk < (part + 1) * KK_PART; ++kk)
                    mma_ts(tmem + C::tm_o(t), tmem + C::tm_s(t) + kk * 8,
                           sdesc_sw128(va + kk * 2048, C::CHUNK_BYTES, 1024), idPV,
                           (accumulate || kk > 0) ? 1u : 0u);
            };
            // cb = key blocks tile t consumed before this one (the phase of its P barriers);
            // accumulate unless this is a unit's first block.
            auto wait_issue_PV = [&](int t, int s, int cb, bool first) {
#pragma unroll
                for (int part = 0; part < C::P_PARTS; ++part) {
                    uint64_t* bar = part + 1 < C::P_PARTS
                                        ? &bar_ppart[t * (C::P_PARTS - 1) + part]
                                        : &bar_pfull[t];
                    if (!mbar_wait(bar, cb & 1, p.timeout_ns, abort_flag)) return false;
                    tc_fence_after();
                    issue_PV(t, s, !first || part > 0, part);
                }
                return true;
            };
            // Per unit: S_0(0) S_1(0), then per key block j: P V_0(j), S_0(j+1), P V_1(j),
            // S_1(j+1), tile 0's products only for its n0 <= n1 blocks; the commit after the
            // unit's last score MMA (S_1(n1 - 1)) releases the Q tiles.
            bool ok = true;
            int g = 0;   // ring position of the unit's block 0 (= blocks loaded so far)
            int c0 = 0;  // blocks tile 0 consumed in earlier units (its P barriers' phase)
            int uc = 0;  // units started
            for (int lin = blockIdx.x; ok && lin < n_units; lin += gridDim.x, ++uc) {
                const Unit u = unit(lin);
                const int n0 = u.n0, n1 = u.n1;
                if (!(ok = mbar_wait(bar_q, uc & 1, p.timeout_ns, abort_flag))) break;
                if (!(ok = mbar_wait(&bar_kfull[g % C::STAGES], (g / C::STAGES) & 1, p.timeout_ns,
                                     abort_flag)))
                    break;
                tc_fence_after();
                issue_S(0, g % C::STAGES);
                tc_commit(&bar_sfull[0]);
                issue_S(1, g % C::STAGES);
                tc_commit(&bar_sfull[1]);
                tc_commit(&bar_kempty[g % C::STAGES]);
                if (n1 == 1) tc_commit(bar_qempty);
                for (int j = 0; ok && j < n1; ++j) {
                    const int gj = g + j, gn = gj + 1;
                    const int s = gj % C::STAGES, sn = gn % C::STAGES;
                    const uint32_t ph = (gj / C::STAGES) & 1, phn = (gn / C::STAGES) & 1;
                    if (!(ok = mbar_wait(&bar_vfull[s], ph, p.timeout_ns, abort_flag))) break;
                    if (j < n0) {
                        if (!(ok = wait_issue_PV(0, s, c0 + j, j == 0))) break;
                        tc_commit(&bar_ofull[0]);
                    }
                    if (j + 1 < n1) {
                        if (!(ok = mbar_wait(&bar_kfull[sn], phn, p.timeout_ns, abort_flag))) break;
                        tc_fence_after();
                        if (j + 1 < n0) {
                            issue_S(0, sn);
                            tc_commit(&bar_sfull[0]);
                        }
                    }
                    if (!(ok = wait_issue_PV(1, s, gj, j == 0))) break;
                    tc_commit(&bar_ofull[1]);
                    tc_commit(&bar_vempty[s]);
                    if (j + 1 < n1) {
                        issue_S(1, sn);
                        tc_commit(&bar_sfull[1]);
                        tc_commit(&bar_kempty[sn]);
                        if (j + 2 == n1) tc_commit(bar_qempty);
                    }
                }
                g += n1;
                c0 += n0;
            }
            if (!ok) fail();
            tc_commit(bar_done);
            mbar_wait_drain(bar_done, 0, p.timeout_ns);
        }
      }
    } else {
        regs_set<C::REGS_SOFTMAX_PERSIST, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp / 4;
        const int r = threadIdx.x % C::BM;
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::tm_s(t);
        const uint32_t tO = tmem + lane_base + C::tm_o(t);
        const float c = p.scale_log2;
        bool ok = true;
        int cb = 0;  // key blocks processed (the phase of this tile's barriers)
        for (int lin = blockIdx.x; ok && lin < n_units; lin += gridDim.x) {
            const Unit u = unit(lin);
            const int nt = t ? u.n1 : u.n0;
            // visible keys of this thread's row: j < lim (all N without the causal mask)
            const int lim = causal ? min(p.N, u.q_base + t * C::BM + r + 1) : p.N;
            float m = -INFINITY;  // running max of S * c (log2 units), possibly stale by <= 8
            float l = 0.f;        // running sum of exp2(S * c - m)
            for (int j = 0; j < nt; ++j, ++cb) {
                ok = mbar_wait(&bar_sfull[t], cb & 1, p.timeout_ns, abort_flag);
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
                const bool grow = m_new > m + 8.0f;
                const float alpha = (grow && m != -INFINITY) ? ex2(m - m_new) : 1.0f;
                if (grow) {
                    l *= alpha;
                    m = m_new;
                }
                if (__any_sync(0xffffffffu, grow && j > 0)) {
                    ok = mbar_wait(&bar_ofull[t], (cb - 1) & 1, p.timeout_ns, abort_flag);
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
                const float mb = (m == -INFINITY) ? 0.f : m;
                const float2 c2 = make_float2(c, c);
                const float2 nm2 = make_float2(-mb, -mb);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                constexpr int WP = C::BN / 2 / C::P_PARTS;
#pragma unroll
                for (int part = 0; part < C::P_PARTS; ++part) {
                    uint32_t pk[WP];
#pragma unroll
                    for (int i = 0; i < WP; ++i) {
                        const int e0 = part * 2 * WP + 2 * i;
                        const float2 x = ffma2(make_float2(__uint_as_float(s[e0]),
                                                           __uint_as_float(s[e0 + 1])), c2, nm2);
                        const float2 e = make_float2(ex2(x.x), ex2(x.y));
                        acc[i % 4] = fadd2(acc[i % 4], e);
                        pk[i] = pack_bf16x2(e.x, e.y);
                    }
                    if constexpr (WP == 32) tmem_st32(tS + part * WP, pk);
                    else tmem_st16(tS + part * WP, pk);
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(part + 1 < C::P_PARTS ? &bar_ppart[t * (C::P_PARTS - 1) + part]
                                                      : &bar_pfull[t]);
                }
                l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                     ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
            }
            // -------------------------------------------------------- epilogue of the unit
            if (ok) ok = mbar_wait(&bar_ofull[t], (cb - 1) & 1, p.timeout_ns, abort_flag);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const Unit ue = unit(opaque(lin));  // recomputed here, not kept through the loop
                const int bh = ue.bh;
                const int row = ue.q_base + t * C::BM + r;
                const float inv_l = l > 0.f ? 1.0f / l : 0.f;
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
                        w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                           __uint_as_float(o[2 * i + 1]) * inv_l);
                    if (in_range) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                    }
                }
                const size_t l_off = (size_t)bh * p.N + row;
                if (in_range && in_bounds(p.err, l_off, 1, p.dbg.lse))
                    p.lse[l_off] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            } else {
                fail();
                ok = false;
            }
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


template <int D, bool PACKED>
cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdParams& p, int B, int num_sms, cudaStream_t stream) {
    using C = FwdCfg<D>;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_fwd_kernel<D, PACKED, false>,
                                            fa_fwd_kernel<D, PACKED, !PACKED>,
                                            fa_fwd_persist_kernel<D, false>,
                                            fa_fwd_persist_kernel<D, true>);
        e != cudaSuccess)
        return e;
    const int nx = (p.N + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA;
    const long long units = (long long)nx * p.H * B;
    // Head-major launches without key lengths, more units than SMs and at most 32 key blocks
    // per tile (N <= 4096): the persistent kernel, one CTA per SM.  Measured without the causal
    // mask +3 to +30 % up to there and neutral to 2 % slower beyond; with it +34 / +25 / +10 / 0 %
    // at N = 512 / 1024 / 2048 / 4096 (d = 128) and +35 / +23 / +11 / +5 % (d = 64).
    // Otherwise one CTA per unit in the heaviest-first order.
    const int nblk = (p.N + C::BN - 1) / C::BN;
    if (!PACKED && p.seqlens == nullptr && units > num_sms && nblk <= 32) {
        if (p.causal && D != 128)  // (d = 128 reads the flag at run time)
            fa_fwd_persist_kernel<D, true><<<num_sms, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
        else
            fa_fwd_persist_kernel<D, false><<<num_sms, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
        return cudaGetLastError();
    }
    dim3 grid(nx, p.H, B);
    // Head-major causal launches take the grouped heaviest-first order (its own instantiation,
    // so that the other launches keep their code unchanged).
    if (!PACKED && p.causal)
        fa_fwd_kernel<D, PACKED, !PACKED><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    else
        fa_fwd_kernel<D, PACKED, false><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int B, int num_sms, cudaStream_t stream) {
    const bool packed = p.cu_seqlens != nullptr;
    if (d == 64)
        return packed ? launch_fwd_d<64, true>(tq, tk, tv, p, B, num_sms, stream)
                      : launch_fwd_d<64, false>(tq, tk, tv, p, B, num_sms, stream);
    return packed ? launch_fwd_d<128, true>(tq, tk, tv, p, B, num_sms, stream)
                  : launch_fwd_d<128, false>(tq, tk, tv, p, B, num_sms, stream);
}

}  // namespace fa
