// fa_bwd_d256.cu -- exact-attention backward pass for head dim 256 (sm_100a), head-major and
// packed layouts.
//
// The same computation as fa_bwd.cu (recompute P from the forward's log-sum-exp, then
// dV = P^T dO, dS = P * (dP - D), dK = scale dS^T Q, dQ = scale dS K; flash-attention glossary
// page, "Hoe werkt het?", item "Herberekening"), laid out for d = 256.  A 128-key block's dV and
// dK would take 2 x 256 fp32 columns of tensor memory, all of it, and K, V, Q and dO tiles of
// 128 rows would take 256 KB of shared memory.  So:
//   * a CTA owns one 128-key block AND one half of the 256 features (hd = 0 or 1): it keeps
//     dV[:, half] and dK[:, half] in tensor memory and adds dQ[:, half] into the accumulator;
//     the two CTAs of a key block both compute the full S^T = K Q^T and dP^T = V dO^T
//     (contractions over all 256 features), the price of the split (the backward does
//     7 GEMM-halves' worth of work per half instead of 5);
//   * a query step is 64 rows, with a single Q / dO stage: K and V (64 KB each), Q and dO
//     (32 KB each) and the dS^T tile (16 KB) fill 208 KB of shared memory.
// dQ is accumulated in the same order-independent fixed point as fa_bwd.cu (fa_bwd_common.cuh).
//
// Warp roles (512 threads):
//   warps 0-7   compute: warpgroup h owns query columns [32h, 32h+32) of every step; thread
//               (h, r) owns key row r (= TMEM lane r).  Per step a P phase (P^T = exp2(S^T c -
//               lse2) -> tensor memory) and a dS phase (dS^T = P^T (dP^T - D) -> tensor and
//               shared memory); at the end dV[:, half] (warpgroup 0) and dK[:, half] (1).
//   warp  8     MMA issue (one thread) + TMEM allocation
//   warp  9     TMA producer (one thread)
//   warps 10-11 idle
//   warps 12-15 dQ drain: dQ^T[half] (lane = feature, column = query) out of tensor memory,
//               to fixed point, added to the accumulator (one 128-byte line per instruction)
// Tensor memory (512 columns):
//   A  [0,64)     S^T (fp32) -> P^T (bf16, [0,32))
//   B  [64,128)   dP^T (fp32) -> dS^T (bf16, [64,96))
//   DQ [128,192)  dQ^T of the feature half (fp32)
//   DV [256,384)  DK [384,512)
// MMA order per step: S^T, dP^T | dV (after P) | dK (after dS), then Q/dO free | dQ^T.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

#include "fa_bwd_common.cuh"

struct Bwd256 {
    static constexpr int D = 256;
    static constexpr int DH = 128;                 // features per CTA (one half)
    static constexpr int BN = 128;                 // keys per CTA
    static constexpr int BM = 64;                  // queries per step
    static constexpr int KCH = D / 64;             // 64-feature chunks of a row
    static constexpr int KV_CHUNK = BN * 128;      // a 64-feature chunk of K or V (16 KB)
    static constexpr int Q_CHUNK = BM * 128;       // a 64-feature chunk of Q or dO (8 KB)
    static constexpr int SMEM_K = 0;
    static constexpr int SMEM_V = SMEM_K + KCH * KV_CHUNK;
    static constexpr int SMEM_Q = SMEM_V + KCH * KV_CHUNK;
    static constexpr int SMEM_DO = SMEM_Q + KCH * Q_CHUNK;
    static constexpr int SMEM_DS = SMEM_DO + KCH * Q_CHUNK;   // [128 keys][64 queries] bf16
    static constexpr int SMEM_VEC = SMEM_DS + BN * BM * 2;    // [2][64] lse2, [2][64] D
    static constexpr int SMEM_SCALE = SMEM_VEC + 4 * BM * 4;  // [64] fixed-point scales
    static constexpr int SMEM_BAR = SMEM_SCALE + BM * 4;
    // kv, qfull, qempty, sfull, dpfull, pfull, dsfull, dqfull, dqempty, done
    static constexpr int NUM_BARS = 10;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16;  // tmem address, abort flag
    static constexpr int THREADS = 512;
    // 2 x 136 + 104 (MMA / TMA; their threads spilled at 88) + 136 = 4 x 128 launched
    static constexpr uint32_t REGS_COMPUTE = 136, REGS_OTHER = 104, REGS_DRAIN = 136;
    static constexpr uint32_t REGS_LAUNCH = 65536 / THREADS;  // per thread at launch: 128
    static_assert(2 * REGS_COMPUTE + REGS_OTHER + REGS_DRAIN == 4 * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_A = 0, TM_B = 64, TM_DQ = 128, TM_DV = 256, TM_DK = 384;
    // Warpgroup h reads the fp32 S^T / dP^T columns [32h, 32h + 32) and writes the bf16 P^T /
    // dS^T of its 32 queries (16 columns) into the first half of those same columns, so neither
    // warpgroup overwrites columns the other still reads; the MMAs reading P^T / dS^T as A
    // address each 16-query K step where it lies.
    __device__ static constexpr uint32_t a_col(int kk) { return (uint32_t)((kk / 2) * 32 + (kk % 2) * 8); }
    static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-CTA limit");
    static_assert(SMEM_DS % 1024 == 0 && SMEM_Q % 1024 == 0 && SMEM_DO % 1024 == 0,
                  "swizzled tiles must start on 1024-byte boundaries");
};

template <bool PACKED>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDO, const BwdParams p) {
    using C = Bwd256;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int n_kv = (p.N + C::BN - 1) / C::BN;  // key blocks per head

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_kv = bars;
    uint64_t* bar_qfull = bars + 1;
    uint64_t* bar_qempty = bars + 2;
    uint64_t* bar_sfull = bars + 3;
    uint64_t* bar_dpfull = bars + 4;
    uint64_t* bar_pfull = bars + 5;
    uint64_t* bar_dsfull = bars + 6;
    uint64_t* bar_dqfull = bars + 7;
    uint64_t* bar_dqempty = bars + 8;
    uint64_t* bar_done = bars + 9;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
    float* s_lse2 = reinterpret_cast<float*>(smem + C::SMEM_VEC);    // [2][BM]
    float* s_D = s_lse2 + 2 * C::BM;                                   // [2][BM]
    float* s_scale = reinterpret_cast<float*>(smem + C::SMEM_SCALE);  // [BM]

    if (threadIdx.x == 0 && (smem_u32(smem) & 1023u)) record_error(p.err, kErrInvalidArg);
    const int hd = blockIdx.x & 1;          // feature half of this CTA
    const int tile = blockIdx.x >> 1;
    const int bhk = tile / n_kv;            // (batch, key/value head)
    const int j = tile % n_kv;              // key block (causal: the heaviest, j = 0, first)
    const int b = bhk / p.H_kv;
    const int G = p.H / p.H_kv;             // query heads sharing this key/value head
    const int bh_first = b * p.H + (bhk % p.H_kv) * G;
    constexpr bool packed = PACKED;
    const SeqExtent ext = sequence_extent(p, b, threadIdx.x == 0 && j == 0 && hd == 0 &&
                                                    bhk % p.H_kv == 0, packed);
    const int L = ext.L;
    const int n_q = (ext.Lq + C::BM - 1) / C::BM;  // 64-row query blocks
    const int k0 = j * C::BN;

    // TMA coordinates (y, z) of row n of query head qh (= b*H + h) and of this key/value head:
    // head-major (n, head), packed (head within the sequence, t0 + n).
    auto q_y = [&](int qh, int n) { return packed ? qh - b * p.H : n; };
    auto q_z = [&](int qh, int n) { return packed ? ext.t0 + n : qh; };
    const int kv_y = packed ? bhk % p.H_kv : k0;
    const int kv_z = packed ? ext.t0 + k0 : bhk;

    if (k0 >= L) {
        // Packed: these rows belong to no key of this sequence; nothing to write.
        if (packed) return;
        // Every key of this block is padding: dK = dV = 0 (this CTA's feature half).
        const int rows = min(C::BN, p.N - k0);
        if (!in_bounds(p.err, ((size_t)bhk * p.N + k0) * D, (size_t)rows * D, p.dbg.kv)) return;
        __nv_bfloat16* dk = reinterpret_cast<__nv_bfloat16*>(p.dk) + ((size_t)bhk * p.N + k0) * D;
        __nv_bfloat16* dv = reinterpret_cast<__nv_bfloat16*>(p.dv) + ((size_t)bhk * p.N + k0) * D;
        for (int i = threadIdx.x; i < rows * (C::DH / 8); i += blockDim.x) {
            const size_t e = (size_t)(i / (C::DH / 8)) * D + hd * C::DH + (i % (C::DH / 8)) * 8;
            *reinterpret_cast<uint4*>(dk + e) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(dv + e) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    // Causal: only query blocks from the one holding key k0 on see this key block.
    // Non-causal: start there as well and wrap, so the key blocks of a head add into
    // different query blocks at any moment.
    const int i_first = k0 / C::BM;
    const int i_start = p.causal ? i_first : 0;
    const int n_it_head = n_q - i_start;
    const int n_it = G * n_it_head;
    struct Step {
        int g, r;
    };
    auto next_step = [&](Step s) {
        return s.r + 1 == n_it_head ? Step{s.g + 1, 0} : Step{s.g, s.r + 1};
    };
    auto q_head = [&](Step s) { return bh_first + s.g; };
    auto q_block = [&](Step s) {
        const int i = (p.causal ? i_first : min(i_first, n_q - 1)) + s.r;
        if (p.causal) return i;
        return i < n_q ? i : i - n_q;
    };

    if (threadIdx.x == 0) {
        // arrivals per phase: one commit or TMA thread, except P and dS (the 256 compute
        // threads) and dqempty (the 128 drain threads)
        for (int t = 0; t < C::NUM_BARS; ++t) {
            uint64_t* bar = &bars[t];
            mbar_init(bar, (bar == bar_pfull || bar == bar_dsfull) ? 256 : bar == bar_dqempty ? 128 : 1);
        }
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

    if (warp >= 12) {
        regs_set<C::REGS_DRAIN, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ dQ drain
        const int r = threadIdx.x - 384;                // TMEM lane = feature r of the half
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const float factor = head_bound_factor(p, bhk);
        // Named barriers have no timeout: every drain thread executes each of them, also after
        // a failed wait (`ok` then only skips the work).
        bool ok = true;
        Step st{0, 0};
        for (int it = 0; it < n_it; ++it, st = next_step(st)) {
            const int q0 = q_block(st) * C::BM;
            if (r < C::BM) {  // fixed-point scale of query q0 + r (rows past N: 0)
                const int q = q0 + r;
                s_scale[r] = q < ext.Lq && in_bounds(p.err, (size_t)q_head(st) * p.N + q, 1, p.dbg.vec)
                                 ? fmaxf(fixed_point_scale(p.dOnorm[(size_t)q_head(st) * p.N + q], factor), 0.f)
                                 : 0.f;
            }
            named_barrier(2, 128);
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dqfull, it & 1, p.timeout_ns, abort_flag));
            if (ok) {
                tc_fence_after();
                uint32_t v[C::BM];
                tmem_ld32(tmem + lane_base + C::TM_DQ, v);
                tmem_ld32(tmem + lane_base + C::TM_DQ + 32, v + 32);
                tmem_ld_wait();
                reg_fence32(v);
                reg_fence32(v + 32);
                tc_fence_before();
                mbar_arrive(bar_dqempty);  // the next dQ^T may overwrite the columns
                // dQ^T: lane = feature, column = query e: a warp instruction covers 32
                // consecutive features of one query row, one 128-byte line.
                int* acc = p.dq_acc + ((size_t)q_head(st) * p.N_pad + q0) * D + hd * C::DH + r;
                const bool acc_ok = in_bounds(p.err, ((size_t)q_head(st) * p.N_pad + q0) * D,
                                              (size_t)C::BM * D, p.dbg.acc);
                if (acc_ok) {
#pragma unroll
                    for (int e = 0; e < C::BM; e += 2) {
                        const int2 x = to_fixed2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                 s_scale[e], s_scale[e + 1]);
                        red_add_s32(acc + (size_t)e * D, x.x);
                        red_add_s32(acc + (size_t)(e + 1) * D, x.y);
                    }
                }
            }
            named_barrier(2, 128);  // every read of s_scale done before the next step writes
        }
        if (!ok) fail();
    } else if (warp >= 8) {
      regs_set<C::REGS_OTHER, C::REGS_LAUNCH>();
      if (warp == 9 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
        mbar_arrive_expect_tx(bar_kv, 2 * C::KCH * C::KV_CHUNK);
        for (int c = 0; c < C::KCH; ++c) {
            tma_load_3d(smem + C::SMEM_K + c * C::KV_CHUNK, &tmK, bar_kv, c * 64, kv_y, kv_z);
            tma_load_3d(smem + C::SMEM_V + c * C::KV_CHUNK, &tmV, bar_kv, c * 64, kv_y, kv_z);
        }
        int it = 0;
        Step st{0, 0};
        for (; it < n_it; ++it, st = next_step(st)) {
            const int q0 = q_block(st) * C::BM;
            const int qh = q_head(st);
            // one Q / dO stage: wait until the previous step's MMAs have read it
            if (!mbar_wait(bar_qempty, (it & 1) ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
            mbar_arrive_expect_tx(bar_qfull, 2 * C::KCH * C::Q_CHUNK);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(smem + C::SMEM_Q + c * C::Q_CHUNK, &tmQ, bar_qfull, c * 64,
                            q_y(qh, q0), q_z(qh, q0));
                tma_load_3d(smem + C::SMEM_DO + c * C::Q_CHUNK, &tmDO, bar_qfull, c * 64,
                            q_y(qh, q0), q_z(qh, q0));
            }
        }
        // Do not leave while our copies may still be landing in shared memory.
        if (it > 0) mbar_wait_drain(bar_qfull, (it - 1) & 1, p.timeout_ns);
        mbar_wait_drain(bar_kv, 0, p.timeout_ns);
      } else if (warp == 8 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idS = idesc_bf16(128, C::BM, false, false);  // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16(128, C::DH, false, true);  // dV, dK (A in TMEM)
        constexpr uint32_t idQ = idesc_bf16(128, C::BM, true, true);    // dQ^T of the half
        // K-major operands of S^T = K Q^T and dP^T = V dO^T: a 16-feature K step is 32 bytes
        // inside a swizzled row, then the next 64-feature chunk.
        const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::SMEM_K), 16, 1024);
        const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::SMEM_V), 16, 1024);
        const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + C::SMEM_Q), 16, 1024);
        const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + C::SMEM_DO), 16, 1024);
        auto kmaj_kv = [](int kk) { return (uint64_t)(((kk / 4) * C::KV_CHUNK + (kk % 4) * 32) >> 4); };
        auto kmaj_q = [](int kk) { return (uint64_t)(((kk / 4) * C::Q_CHUNK + (kk % 4) * 32) >> 4); };
        // MN-major operands: this CTA's feature half of Q and dO (B of dK, dV: N = 128
        // features = the two 64-feature chunks 2hd, 2hd+1), of K (A of dQ^T: M = 128 features),
        // and the dS^T tile (B of dQ^T: N = 64 queries, one swizzled row per key).  A K step of
        // 16 rows (queries or keys) is 2048 bytes.
        const uint64_t dQh_mn = sdesc_sw128(smem_u32(smem + C::SMEM_Q + 2 * hd * C::Q_CHUNK), C::Q_CHUNK, 1024);
        const uint64_t dDOh_mn = sdesc_sw128(smem_u32(smem + C::SMEM_DO + 2 * hd * C::Q_CHUNK), C::Q_CHUNK, 1024);
        const uint64_t dKh_mn = sdesc_sw128(smem_u32(smem + C::SMEM_K + 2 * hd * C::KV_CHUNK), C::KV_CHUNK, 1024);
        const uint64_t dDS_mn = sdesc_sw128(smem_u32(smem + C::SMEM_DS), C::KV_CHUNK, 1024);
        auto mnmaj = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };

        bool ok = mbar_wait(bar_kv, 0, p.timeout_ns, abort_flag);
        for (int it = 0; ok && it < n_it; ++it) {
            if (!(ok = mbar_wait(bar_qfull, it & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
            // S^T and dP^T over all 256 features (16 K steps).  They overwrite A and B, which
            // the previous step's dV and dK read: the MMAs of this thread run in issue order.
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_A, dK_k + kmaj_kv(kk), dQ_k + kmaj_q(kk), idS, kk > 0 ? 1u : 0u);
            tc_commit(bar_sfull);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_B, dV_k + kmaj_kv(kk), dDO_k + kmaj_q(kk), idS, kk > 0 ? 1u : 0u);
            tc_commit(bar_dpfull);
            // dV[:, half] += P^T dO[:, half]: A = P^T in tensor memory (16 queries = 8 columns).
            if (!(ok = mbar_wait(bar_pfull, it & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BM / 16; ++kk)
                mma_ts(tmem + C::TM_DV, tmem + C::TM_A + C::a_col(kk), dDOh_mn + mnmaj(kk), idKV,
                       (it > 0 || kk > 0) ? 1u : 0u);
            // dK[:, half] += dS^T Q[:, half]; after it nothing reads this step's Q and dO.
            if (!(ok = mbar_wait(bar_dsfull, it & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BM / 16; ++kk)
                mma_ts(tmem + C::TM_DK, tmem + C::TM_B + C::a_col(kk), dQh_mn + mnmaj(kk), idKV,
                       (it > 0 || kk > 0) ? 1u : 0u);
            tc_commit(bar_qempty);
            // dQ^T[half] = K[:, half]^T dS^T (K = 128 keys), once the drain has copied the
            // previous one out of tensor memory.
            if (it > 0 && !(ok = mbar_wait(bar_dqempty, (it - 1) & 1, p.timeout_ns, abort_flag)))
                break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk)
                mma_ss(tmem + C::TM_DQ, dKh_mn + mnmaj(kk), dDS_mn + mnmaj(kk), idQ, kk > 0 ? 1u : 0u);
            tc_commit(bar_dqfull);
        }
        if (!ok) fail();
        // Wait for every MMA issued here before tensor memory can be released.
        tc_commit(bar_done);
        mbar_wait_drain(bar_done, 0, p.timeout_ns);
      }
    } else {
        regs_set<C::REGS_COMPUTE, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ compute warpgroups
        const int h = warp / 4;                          // query-column half of a step
        const int r = threadIdx.x % 128;                 // TMEM lane = key row
        const int ct = threadIdx.x;                      // 0..255
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const int kidx = k0 + r;
        const bool key_padded = kidx >= L;
        uint8_t* ds_row = smem + C::SMEM_DS + r * 128;
        const int sw = r & 7;
        const float c = p.scale_log2;

        // -lse * log2(e) and D of the step's 64 queries into buffer it & 1 (threads 0..63 the
        // lse values, 64..127 the D values); -inf / 0 past N so those queries get P = 0.  The
        // global load is issued one step ahead and stored at the end of the step.
        float staged = 0.f;
        // lse of query head bh_first + g, position q: lse[lse_base + g * lse_hstride + q].
        const size_t lse_hstride = packed ? (size_t)p.T : (size_t)p.N;
        const size_t lse_base = lse_of(packed, b, bh_first - b * p.H, p.H, p.N, p.T, ext.t0, 0);
        auto load_vectors = [&](Step s) {
            const int q = q_block(s) * C::BM + (ct & 63);
            if (ct < 64)
                staged = q < ext.Lq && in_bounds(p.err, lse_base + (size_t)s.g * lse_hstride + q, 1, p.dbg.lse)
                             ? -p.lse[lse_base + (size_t)s.g * lse_hstride + q] * kLog2e
                             : -INFINITY;
            else if (ct < 128)
                staged = q < ext.Lq && in_bounds(p.err, (size_t)q_head(s) * p.N + q, 1, p.dbg.vec)
                             ? p.Dvec[(size_t)q_head(s) * p.N + q] : 0.f;
        };
        auto store_vectors = [&](int it) {
            if (ct < 64) s_lse2[(it & 1) * C::BM + ct] = staged;
            else if (ct < 128) s_D[(it & 1) * C::BM + (ct - 64)] = staged;
        };
        Step st{0, 0};
        load_vectors(st);
        store_vectors(0);
        named_barrier(1, 256);

        // Named barriers have no timeout, so every thread executes every one of them, also
        // after a failed (timed-out or aborted) wait; `ok` then only skips the work.
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int q0 = q_block(st) * C::BM;
            st = next_step(st);                      // the step of it + 1 from here on
            const float* lse2 = s_lse2 + (it & 1) * C::BM + 32 * h;
            const float* Dv = s_D + (it & 1) * C::BM + 32 * h;
            if (it + 1 < n_it) load_vectors(st);   // stored at the end of this step
            // causal: the step's queries [q0, q0 + 64) reach below some key of the block
            const bool diag = p.causal && q0 < k0 + C::BN;

            // ---------------- P phase
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull, it & 1, p.timeout_ns, abort_flag));
            float P[32];
            if (ok) {
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld32(tmem + lane_base + C::TM_A + 32 * h, sv);
                tmem_ld_wait();
                reg_fence32(sv);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 nl = *reinterpret_cast<const float4*>(lse2 + e);  // -lse2
                    const float2 x0 = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                            make_float2(c, c), make_float2(nl.x, nl.y));
                    const float2 x1 = ffma2(make_float2(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])),
                                            make_float2(c, c), make_float2(nl.z, nl.w));
                    P[e] = ex2(x0.x);
                    P[e + 1] = ex2(x0.y);
                    P[e + 2] = ex2(x1.x);
                    P[e + 3] = ex2(x1.y);
                }
                if (key_padded || diag) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (key_padded || kidx > q0 + 32 * h + e) P[e] = 0.f;
                }
            }
            if (ok) {
                uint32_t pw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pw[e] = pack_bf16x2(P[2 * e], P[2 * e + 1]);
                tmem_st16(tmem + lane_base + C::TM_A + 32 * h, pw);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar_pfull);
            }

            // ---------------- dS phase
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dpfull, it & 1, p.timeout_ns, abort_flag));
            uint32_t dw[16];
            if (ok) {
                tc_fence_after();
                uint32_t dp[32];
                tmem_ld32(tmem + lane_base + C::TM_B + 32 * h, dp);
                tmem_ld_wait();
                reg_fence32(dp);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 dv4 = *reinterpret_cast<const float4*>(Dv + e);
                    const float2 a = fmul2(make_float2(P[e], P[e + 1]),
                                           fadd2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                                 make_float2(-dv4.x, -dv4.y)));
                    const float2 bq = fmul2(make_float2(P[e + 2], P[e + 3]),
                                            fadd2(make_float2(__uint_as_float(dp[e + 2]), __uint_as_float(dp[e + 3])),
                                                  make_float2(-dv4.z, -dv4.w)));
                    dw[e / 2] = pack_bf16x2(a.x, a.y);
                    dw[e / 2 + 1] = pack_bf16x2(bq.x, bq.y);
                }
            }
            // Next step's lse / D into the other buffer.  Its last reads were in the previous
            // step, before every thread passed that step's barrier below, and the barrier below
            // orders these stores before the next step's reads.
            if (it + 1 < n_it) store_vectors(it + 1);
            named_barrier(1, 256);  // the next step's lse / D stored
            if (ok) {
                tmem_st16(tmem + lane_base + C::TM_B + 32 * h, dw);  // A of dK
                // dS^T row r, queries [32h, 32h+32): 16-byte units 4h..4h+3 of the row's 128
                // bytes, unit u at position u ^ (r % 8) (the 128-byte swizzle the MMA reads).
                // The dQ^T MMA of the previous step has finished reading the tile: dP^T of
                // this step, issued after it, has completed.
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4*>(ds_row + (((4 * h + u) ^ sw) << 4)) =
                        make_uint4(dw[4 * u], dw[4 * u + 1], dw[4 * u + 2], dw[4 * u + 3]);
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar_dsfull);
            }
        }

        // ---------------- epilogue: dV[:, half] (warpgroup 0) and dK[:, half] * scale (1)
        if (ok) ok = mbar_wait(bar_done, 0, p.timeout_ns, abort_flag);  // every MMA finished
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const bool key_row = kidx < (packed ? L : p.N);
            const size_t off =
                row_of(packed, b, bhk % p.H_kv, p.H_kv, p.N, ext.t0, key_row ? kidx : 0) * D +
                hd * C::DH;
            const uint32_t col0 = h ? C::TM_DK : C::TM_DV;
            const float mul = h ? p.scale : 1.0f;
            const bool in_range = key_row && in_bounds(p.err, off, C::DH, p.dbg.kv);
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(h ? p.dk : p.dv) + off;
#pragma unroll 1
            for (int q = 0; q < C::DH / 32; ++q) {
                uint32_t x[32];
                tmem_ld32(tmem + lane_base + col0 + q * 32, x);
                tmem_ld_wait();
                reg_fence32(x);
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(x[2 * e]) * mul,
                                       __uint_as_float(x[2 * e + 1]) * mul);
                if (in_range) {
                    uint4* dst = reinterpret_cast<uint4*>(out + q * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
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

}  // namespace

cudaError_t launch_bwd_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream,
                            cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    using C = Bwd256;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_bwd_d256_kernel<false>, fa_bwd_d256_kernel<true>);
        e != cudaSuccess)
        return e;
    const dim3 chunks(p.N_pad / 128, p.B * p.H);
    const int n_kv = (p.N + C::BN - 1) / C::BN;
    fa_bwd_pre_kernel<256><<<chunks, 256, 0, stream>>>(p);
    if (ev_start) cudaEventRecord(ev_start, stream);
    const unsigned grid = (unsigned)(p.B * p.H_kv * n_kv * 2);
    if (p.cu_seqlens != nullptr)
        fa_bwd_d256_kernel<true><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    else
        fa_bwd_d256_kernel<false><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    if (ev_stop) cudaEventRecord(ev_stop, stream);
    fa_bwd_dq_kernel<256><<<chunks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
