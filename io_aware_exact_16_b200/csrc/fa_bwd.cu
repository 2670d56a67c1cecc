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
//   fa_bwd_pre_kernel   per row D = rowsum(dO * O) and |dO_i|; per 128-row chunk the largest
//                       |v_j| and |k_jl|; clears the dQ accumulator
//   fa_bwd_kernel       one CTA per 128-key block: recomputes S^T, P^T, dP^T, dS^T per
//                       128-query block with tcgen05 MMAs, accumulates dK, dV in tensor memory
//                       and adds its dQ contribution into the accumulator
//   fa_bwd_dq_kernel    dQ = scale * accumulator -> bf16
//
// Deterministic dQ.  Every key block adds a contribution dS_ib K_b to every query row i it
// sees.  Those contributions are added in integer fixed point, so the sum does not depend on
// the order in which key blocks arrive and repeated runs are bitwise identical, with no
// ordering between CTAs.  Row i uses the scale s_i = 2^floor(log2(2^29 / bound_i)), where
//     bound_i = 2 |dO_i| max_j |v_j| max_{j,l} |k_jl|
// bounds every partial sum: sum_j |dS_ij| = sum_j P_ij |dP_ij - D_i| <= 2 |dO_i| max_j |v_j|
// (|dP_ij| <= |dO_i||v_j|, |D_i| <= |dO_i||O_i| and O_i is a convex combination of the v_j), and
// each feature of sum_j dS_ij k_j is at most that times max |k_jl|.  Every contribution and
// every partial sum therefore stays below 2^29 (+ one rounding per key block), a factor 4
// inside int32.  Each contribution is rounded once, to 2^-29 bound_i, exactly to the nearest
// integer on the FMA and integer pipes (to_fixed).  The bound holds for any inputs, but it is
// loose (random signs cancel in the sum over keys, which no a-priori bound can use): at
// N = 16384 the actual dQ uses about 2^-11 of it, so the resolution has to be this fine for
// the rounding to stay well below the bf16 rounding of dS, also when one value row or one
// key feature is much larger than the rest.
//
// Main-kernel warp roles (512 threads = 4 warpgroups):
//   warps 0-7   compute: warpgroup h owns query columns [64h, 64h+64) of every block; thread
//               (h, r) owns key row r (= TMEM lane r).  Per query block two phases:
//                 P   (needs S^T)  P^T = exp2(S^T c - lse2)   -> tensor memory (bf16)
//                 dS  (needs dP^T) dS^T = P^T (dP^T - D)      -> tensor + shared memory (bf16)
//               The MMA warp issues dV(i), S^T(i+1), dK(i), dQ(i), dP^T(i+1), so the P phase
//               of block i+1 overlaps dK, dQ, the drain and dP^T of block i, and the dS phase
//               overlaps dV and S^T.  At the end they write dV (warpgroup 0) and dK (wg 1).
//   warp  8     MMA issue (one thread) + TMEM allocation
//   warp  9     TMA producer (one thread)
//   warps 10-11 idle
//   warps 12-15 dQ drain: copy the dQ block out of tensor memory, free it, convert it to fixed
//               point and add it to the accumulator with integer atomics.  For d = 128 the
//               block is held transposed (dQ^T = K^T dS^T: lane = feature, column = query) so
//               each warp instruction adds one 128-byte line; for d = 64 it is dQ = dS K (lane =
//               query) and goes through a per-warp shared-memory transpose to the same pattern.
// Registers: warpgroup 2 gives its share to warpgroups 0, 1 and 3 (setmaxnreg).
// Tensor memory (512 columns):
//   A [0,128)   S^T (fp32) -> P^T (bf16, columns [0,64))
//   B [128,256) dP^T (fp32) -> dS^T (bf16, [128,192)) -> the dQ block (fp32)
//   dV [256, 256+d)   dK [256+d, 256+2d)
// Shared memory: K_j, V_j (once), a 2-stage ring of Q_i / dO_i, dS^T (bf16, 128-byte
// swizzled, an operand of the dQ MMA), lse*log2(e), D and the fixed-point scales of the query
// blocks (and for d = 64 the drain's transpose buffers).
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

#include "fa_bwd_common.cuh"

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
    static constexpr int SMEM_VEC = SMEM_DS + DS_BYTES;        // [2][128] lse2, [2][128] D
    static constexpr int SMEM_SCALE = SMEM_VEC + 4 * BM * 4;   // [128] fixed-point scales
    static constexpr int SMEM_XPOSE = SMEM_SCALE + BM * 4;     // d = 64: 4 x [32][33] int32
    static constexpr int XPOSE_BYTES = (D == 64) ? 4 * 32 * 33 * 4 : 0;
    static constexpr int SMEM_BAR = SMEM_XPOSE + XPOSE_BYTES;
    // kv, Q/dO full and empty per stage, s, dp, p, ds, dq full, dq empty, done, and the
    // persistent kernel's unit-done and accumulators-free barriers
    static constexpr int NUM_BARS = 1 + 2 * QST + 7 + 2;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = SMEM_MISC + 16;  // tmem address, abort flag
    static constexpr int THREADS = 512;
    // 2 x compute + MMA / TMA + drain = 4 x 128 launched.  The MMA thread spilled its operand
    // descriptors at 88 registers, so every product it issued waited on local memory: 96 there
    // measured +7 to +11 % (d = 128: 2 x 136 + 96 + 144; d = 64, whose drain holds half as
    // many dQ values: 2 x 152 + 96 + 112).
    static constexpr uint32_t REGS_COMPUTE = (D == 64) ? 152 : 136, REGS_OTHER = 96,
                              REGS_DRAIN = (D == 64) ? 112 : 144;
    // The persistent kernel's MMA and TMA threads carry loop state across units and spill at
    // 88 registers: 2 x 128 + 104 + 152 there.
    static constexpr uint32_t REGS_COMPUTE_PERSIST = 128, REGS_OTHER_PERSIST = 104,
                              REGS_DRAIN_PERSIST = 152;
    static constexpr uint32_t REGS_LAUNCH = 65536 / THREADS;  // per thread at launch: 128
    static_assert(2 * REGS_COMPUTE + REGS_OTHER + REGS_DRAIN == 4 * REGS_LAUNCH, "register split");
    static_assert(2 * REGS_COMPUTE_PERSIST + REGS_OTHER_PERSIST + REGS_DRAIN_PERSIST == 4 * REGS_LAUNCH,
                  "register split");
    static constexpr uint32_t TMEM_COLS = 512;

    static constexpr uint32_t TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
    // Own columns: warpgroup h reads the fp32 S^T / dP^T columns [64h, 64h + 64) of its region
    // and writes the bf16 P^T / dS^T of its 64 queries (32 columns) back into the first half of
    // those same columns, so no warpgroup overwrites columns the other still reads and the P
    // phase needs no barrier; the MMAs that read P^T / dS^T as their A operand address each
    // 16-query K step where it lies.  Otherwise the bf16 halves are packed into columns
    // [32h, 32h + 32) behind a barrier.  The head-major kernels use own columns (+2 to +4 %);
    // the packed-sequence kernel keeps the packed form, where the other addressing cost
    // registers and measured 12 % slower.
    __device__ static constexpr uint32_t bf16_col(bool own, int h) { return own ? 64u * h : 32u * h; }
    __device__ static constexpr uint32_t a_col(bool own, int kk) {
        return own ? (uint32_t)((kk / 4) * 64 + (kk % 4) * 8) : (uint32_t)(kk * 8);
    }
};

// ---------------------------------------------------------------------------- main kernel
template <int D, bool PACKED, bool GROUPED>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr bool OWN = !PACKED;  // own-column P^T / dS^T layout
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int n_kv = (p.N + C::BN - 1) / C::BN;  // key blocks per head (of the longest sequence)

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_kv = bars;
    uint64_t* bar_qfull = bars + 1;
    uint64_t* bar_qempty = bar_qfull + C::QST;
    uint64_t* bar_sfull = bar_qempty + C::QST;
    uint64_t* bar_dpfull = bar_sfull + 1;
    uint64_t* bar_pfull = bar_dpfull + 1;
    uint64_t* bar_dsfull = bar_pfull + 1;
    uint64_t* bar_dqfull = bar_dsfull + 1;
    uint64_t* bar_dqempty = bar_dqfull + 1;
    uint64_t* bar_done = bar_dqempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
    float* s_lse2 = reinterpret_cast<float*>(smem + C::SMEM_VEC);    // [2][BM]
    float* s_D = s_lse2 + 2 * C::BM;                                   // [2][BM]
    float* s_scale = reinterpret_cast<float*>(smem + C::SMEM_SCALE);  // [BM]

    if (threadIdx.x == 0 && (smem_u32(smem) & 1023u)) record_error(p.err, kErrInvalidArg);
    // Key block j of key/value head bhk.  Head-major causal: the launch order walks groups of
    // 16 heads and, inside a group, every head's key blocks from the heaviest (j = 0, the most
    // query blocks) to the lightest, so the last wave holds light blocks only while one
    // group's Q and dO stay in L2; otherwise head by head, j = 0 first.
    // (GROUPED: head-major causal launches, their own instantiation.)
    int bhk, j;
    if constexpr (GROUPED) {
        constexpr int GH = 16;
        const int lin = blockIdx.x;
        const int g0 = lin / (n_kv * GH) * GH;
        const int gh = min(GH, (int)(gridDim.x / n_kv) - g0);  // heads in this group
        const int r = lin - g0 * n_kv;                         // rank-major inside the group
        bhk = g0 + r % gh;
        j = r / gh;
    } else {
        bhk = blockIdx.x / n_kv;
        j = blockIdx.x % n_kv;
    }
    const int b = bhk / p.H_kv;
    const int G = p.H / p.H_kv;   // query heads sharing this key/value head
    const int bh_first = b * p.H + (bhk % p.H_kv) * G;
    constexpr bool packed = PACKED;
    const SeqExtent ext =
        sequence_extent(p, b, threadIdx.x == 0 && j == 0 && bhk % p.H_kv == 0, packed);
    const int L = ext.L;
    const int n_q = (ext.Lq + C::BM - 1) / C::BM;  // query blocks of this sequence
    const int k0 = j * C::BN;
    // TMA coordinates (y, z) of row n of query head qh (= b*H + h) and of this key/value head.
    auto q_y = [&](int qh, int n) { return packed ? qh - b * p.H : n; };
    auto q_z = [&](int qh, int n) { return packed ? ext.t0 + n : qh; };
    const int kv_y = packed ? bhk % p.H_kv : k0;
    const int kv_z = packed ? ext.t0 + k0 : bhk;

    if (k0 >= L) {
        // Packed: these rows belong to no key of this sequence; nothing to write.
        if (packed) return;
        // Every key of this block is padding: dK = dV = 0 and no dQ contribution.
        const int rows = min(C::BN, p.N - k0);
        if (!in_bounds(p.err, ((size_t)bhk * p.N + k0) * D, (size_t)rows * D, p.dbg.kv)) return;
        uint4* dk = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dk) + ((size_t)bhk * p.N + k0) * D);
        uint4* dv = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dv) + ((size_t)bhk * p.N + k0) * D);
        for (int i = threadIdx.x; i < rows * D / 8; i += blockDim.x) {
            dk[i] = make_uint4(0, 0, 0, 0);
            dv[i] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    // Causal: only query blocks from the diagonal on see this key block.  Non-causal: start
    // at query block j and wrap, so the key blocks of a head add into different query
    // blocks at any moment instead of all hammering the same accumulator lines.
    const int i_start = p.causal ? j : 0;
    // Step it visits query head q_head(it) of the group (each head in turn) and query block
    // q_block(it) of that head; dK and dV accumulate over every step, so they sum over the
    // group's query heads.
    // Each role walks the steps with a Step cursor (g = head of the group, r = step within the
    // head) instead of dividing `it` by n_it_head: an integer divide by a runtime value needs a
    // reciprocal on the MUFU unit, which the exponentials of the P phase saturate.
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
        const int i = j + s.r;
        if (p.causal) return i;
        return i < n_q ? i : i - n_q;
    };

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < C::QST; ++s) {
            mbar_init(&bar_qfull[s], 1);
            mbar_init(&bar_qempty[s], 1);
        }
        mbar_init(bar_sfull, 1);
        mbar_init(bar_dpfull, 1);
        mbar_init(bar_pfull, 256);
        mbar_init(bar_dsfull, 256);
        mbar_init(bar_dqfull, 1);
        mbar_init(bar_dqempty, 128);
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

    if (warp >= 12) {
        regs_set<C::REGS_DRAIN, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ dQ drain
        const int r = threadIdx.x - 384;                // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const float factor = head_bound_factor(p, bhk);
        // Named barriers have no timeout: every drain thread executes each of them, also after
        // a failed wait (`ok` then only skips the work).
        bool ok = true;
        // ||dO|| of query row r of step s, or -1 for rows past the sequence (scale 0).  Loaded
        // one step ahead, so its latency overlaps the previous step's reductions.
        auto load_norm = [&](Step s) -> float {
            const int q = q_block(s) * C::BM + r;
            return q < ext.Lq && in_bounds(p.err, (size_t)q_head(s) * p.N + q, 1, p.dbg.vec)
                       ? p.dOnorm[(size_t)q_head(s) * p.N + q] : -1.f;
        };
        // (The packed-sequence kernel loads it in its own step: the prefetch cost it registers.)
        constexpr bool prefetch = !PACKED;
        Step st{0, 0};
        float norm = prefetch ? load_norm(st) : 0.f;
        for (int it = 0; it < n_it; ++it, st = next_step(st)) {
            const int q0 = q_block(st) * C::BM;
            // fixed-point scale of query q0 + r, shared by the drain warps; barrier 2 before the
            // reads and again after the last read of the step.  (A non-finite norm or bound
            // gives -1, which adds nothing; the dQ conversion reports it.)
            if constexpr (!prefetch) norm = load_norm(st);
            s_scale[r] = norm >= 0.f ? fmaxf(fixed_point_scale(norm, factor), 0.f) : 0.f;
            if (prefetch && it + 1 < n_it) norm = load_norm(next_step(st));
            named_barrier(2, 128);
            const float* sc = s_scale;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dqfull, it & 1, p.timeout_ns, abort_flag));
            if (ok) {
                tc_fence_after();
                constexpr int NV = (D == 128) ? 128 : 64;
                uint32_t v[NV];
#pragma unroll
                for (int q = 0; q < NV / 32; ++q) tmem_ld32(tmem + lane_base + C::TM_B + 32 * q, v + 32 * q);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < NV / 32; ++q) reg_fence32(v + 32 * q);
                tc_fence_before();
                mbar_arrive(bar_dqempty);           // B may take the next dP^T
                int* acc = p.dq_acc + ((size_t)q_head(st) * p.N_pad + q0) * D;
                if (in_bounds(p.err, ((size_t)q_head(st) * p.N_pad + q0) * D, (size_t)C::BM * D,
                              p.dbg.acc)) {
                    if constexpr (D == 128) {
                        // dQ^T: lane = feature r, column = query e; a warp instruction covers 32
                        // consecutive features of one query row: one 128-byte line.
#pragma unroll
                        for (int e = 0; e < 128; e += 4) {
                            const float4 s4 = *reinterpret_cast<const float4*>(sc + e);  // one shared load
                            const int2 x = to_fixed2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), s4.x, s4.y);
                            const int2 y = to_fixed2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]), s4.z, s4.w);
                            red_add_s32(acc + (size_t)e * D + r, x.x);
                            red_add_s32(acc + (size_t)(e + 1) * D + r, x.y);
                            red_add_s32(acc + (size_t)(e + 2) * D + r, y.x);
                            red_add_s32(acc + (size_t)(e + 3) * D + r, y.y);
                        }
                    } else {
                        // dQ: lane = query r, 64 features.  Convert, transpose 32 x 32 through
                        // shared memory, then a warp instruction covers 32 consecutive features of
                        // one row.
                        int* xp = reinterpret_cast<int*>(smem + C::SMEM_XPOSE) + (warp % 4) * 32 * 33;
                        const float s_row = sc[r];
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                const int2 x = to_fixed2(__uint_as_float(v[32 * c + e]),
                                                         __uint_as_float(v[32 * c + e + 1]), s_row, s_row);
                                xp[lane * 33 + e] = x.x;
                                xp[lane * 33 + e + 1] = x.y;
                            }
                            __syncwarp();
#pragma unroll 4
                            for (int row = 0; row < 32; ++row)
                                red_add_s32(acc + (size_t)((warp % 4) * 32 + row) * D + 32 * c + lane,
                                            xp[row * 33 + lane]);
                            __syncwarp();
                        }
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
        mbar_arrive_expect_tx(bar_kv, 2 * C::KV_TILE_BYTES);
        for (int c = 0; c < C::KCH; ++c) {
            tma_load_3d(smem + C::SMEM_K + c * C::CHUNK_BYTES, &tmK, bar_kv, c * 64, kv_y, kv_z);
            tma_load_3d(smem + C::SMEM_V + c * C::CHUNK_BYTES, &tmV, bar_kv, c * 64, kv_y, kv_z);
        }
        int it = 0;
        Step st{0, 0};
        for (; it < n_it; ++it, st = next_step(st)) {
            const int s = it % C::QST;
            const uint32_t ph = (it / C::QST) & 1;
            const int q0 = q_block(st) * C::BM;
            const int qh = q_head(st);
            if (!mbar_wait(&bar_qempty[s], ph ^ 1, p.timeout_ns, abort_flag)) { fail(); break; }
            mbar_arrive_expect_tx(&bar_qfull[s], 2 * C::Q_TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(smem + C::SMEM_Q + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES, &tmQ,
                            &bar_qfull[s], c * 64, q_y(qh, q0), q_z(qh, q0));
                tma_load_3d(smem + C::SMEM_DO + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES,
                            &tmDO, &bar_qfull[s], c * 64, q_y(qh, q0), q_z(qh, q0));
            }
        }
        // Do not leave while our copies may still be landing in shared memory.
        for (int t = max(0, it - C::QST); t < it; ++t)
            mbar_wait_drain(&bar_qfull[t % C::QST], (t / C::QST) & 1, p.timeout_ns);
        mbar_wait_drain(bar_kv, 0, p.timeout_ns);
      } else if (warp == 8 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idS = idesc_bf16(128, 128, false, false);  // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16(128, D, false, true);    // dV, dK (A in TMEM)
        constexpr uint32_t idQ = idesc_bf16(128, D == 128 ? 128 : 64, true, true);  // dQ^T / dQ
        // Descriptors of every operand tile, built once; a K step only adds the byte offset
        // (>> 4) to the start-address field, which never carries (shared memory < 256 KB).
        const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::SMEM_K), 16, 1024);   // K-major
        const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::SMEM_V), 16, 1024);
        const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + C::SMEM_K), C::CHUNK_BYTES, 1024);
        const uint64_t dDS_mn = sdesc_sw128(smem_u32(smem + C::SMEM_DS), C::CHUNK_BYTES, 1024);
        const uint64_t dDS_k = sdesc_sw128(smem_u32(smem + C::SMEM_DS), 16, 1024);
        // Q / dO stage st sits st * Q_TILE_BYTES after stage 0.
        const uint64_t dQ_k0 = sdesc_sw128(smem_u32(smem + C::SMEM_Q), 16, 1024);
        const uint64_t dDO_k0 = sdesc_sw128(smem_u32(smem + C::SMEM_DO), 16, 1024);
        const uint64_t dQ_mn0 = sdesc_sw128(smem_u32(smem + C::SMEM_Q), C::CHUNK_BYTES, 1024);
        const uint64_t dDO_mn0 = sdesc_sw128(smem_u32(smem + C::SMEM_DO), C::CHUNK_BYTES, 1024);
        auto kmaj = [](int kk) { return (uint64_t)(((kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32) >> 4); };
        auto mnmaj = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };
        auto stage_off = [](int it) { return (uint64_t)((it % C::QST) * (C::Q_TILE_BYTES >> 4)); };
        // S^T = K Q^T and dP^T = V dO^T for query step `it`: K-major operands, 16-column K
        // steps (32 bytes inside a swizzled row, then the next 64-column chunk).
        auto issue_S = [&](int it) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_A, dK_k + kmaj(kk), dQ_k0 + stage_off(it) + kmaj(kk), idS,
                       kk > 0 ? 1u : 0u);
            tc_commit(bar_sfull);
        };
        auto issue_dP = [&](int it) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_B, dV_k + kmaj(kk), dDO_k0 + stage_off(it) + kmaj(kk), idS,
                       kk > 0 ? 1u : 0u);
            tc_commit(bar_dpfull);
        };
        // Issue order per query step it:  dV(it), S^T(it+1), dK(it), dQ(it), dP^T(it+1).
        // S^T(it+1) may go as soon as dV(it) has read P^T(it) from A (MMAs of one thread run
        // in order), so the next P phase overlaps dK, dQ, the drain and dP^T.
        bool ok = mbar_wait(bar_kv, 0, p.timeout_ns, abort_flag);
        if (ok) ok = mbar_wait(&bar_qfull[0], 0, p.timeout_ns, abort_flag);
        if (ok) {
            tc_fence_after();
            issue_S(0);
            issue_dP(0);
        }
        for (int it = 0; ok && it < n_it; ++it) {
            const int s = it % C::QST;
            const uint64_t dQ_mn = dQ_mn0 + stage_off(it), dDO_mn = dDO_mn0 + stage_off(it);
            // dV += P^T dO: A = P^T in tensor memory (16 queries = 8 columns per K step),
            // B = dO MN-major (16 query rows = 2048 bytes per K step).
            if (!(ok = mbar_wait(bar_pfull, it & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BM / 16; ++kk)
                mma_ts(tmem + C::TM_DV, tmem + C::TM_A + C::a_col(OWN, kk), dDO_mn + mnmaj(kk), idKV,
                       (it > 0 || kk > 0) ? 1u : 0u);
            if (it + 1 < n_it) {
                const int s1 = (it + 1) % C::QST;
                if (!(ok = mbar_wait(&bar_qfull[s1], ((it + 1) / C::QST) & 1, p.timeout_ns, abort_flag)))
                    break;
                tc_fence_after();
                issue_S(it + 1);
            }
            if (!(ok = mbar_wait(bar_dsfull, it & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
            if constexpr (D == 128) {
                // dK += dS^T Q, same shapes as dV (A = dS^T in tensor memory).
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; ++kk)
                    mma_ts(tmem + C::TM_DK, tmem + C::TM_B + C::a_col(OWN, kk), dQ_mn + mnmaj(kk), idKV,
                           (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&bar_qempty[s]);
            }
            // The dQ block into B; K steps of 16 keys = 2048 bytes of both tiles, both
            // operands MN-major.
            if constexpr (D == 128) {
                // dQ^T = K^T dS^T: A = K^T (M = feature), B = dS^T (N = query).
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ss(tmem + C::TM_B, dK_mn + mnmaj(kk), dDS_mn + mnmaj(kk), idQ,
                           kk > 0 ? 1u : 0u);
            } else {
                // dQ = dS K: A = dS (M = query, from the dS^T tile), B = K (N = feature).
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma_ss(tmem + C::TM_B, dDS_mn + mnmaj(kk), dK_mn + mnmaj(kk), idQ,
                           kk > 0 ? 1u : 0u);
            }
            tc_commit(bar_dqfull);
            if constexpr (D == 64) {
                // d = 64: dK after dQ, so the drain starts earlier; A = dS^T read from its
                // shared-memory tile (K-major: key rows, query columns), since dQ has just
                // overwritten tensor-memory B.  Measured faster at d = 64, slower at d = 128.
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; ++kk)
                    mma_ss(tmem + C::TM_DK, dDS_k + kmaj(kk), dQ_mn + mnmaj(kk), idKV,
                           (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&bar_qempty[s]);
            }
            // dP^T(it+1) into B once the drain has copied the dQ block out.
            if (it + 1 < n_it) {
                if (!(ok = mbar_wait(bar_dqempty, it & 1, p.timeout_ns, abort_flag))) break;
                tc_fence_after();
                issue_dP(it + 1);
            }
        }
        if (!ok) fail();
        // Wait for every MMA issued here before tensor memory can be released.
        tc_commit(bar_done);
        mbar_wait_drain(bar_done, 0, p.timeout_ns);
      }
    } else {
        regs_set<C::REGS_COMPUTE, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ compute warpgroups
        const int h = warp / 4;                          // query-column half
        const int r = threadIdx.x % 128;                 // TMEM lane
        const int ct = threadIdx.x;                      // 0..255
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const int kidx = k0 + r;
        const bool key_padded = kidx >= L;
        uint8_t* ds_row = smem + C::SMEM_DS + h * C::CHUNK_BYTES + r * 128;
        const int sw = r & 7;
        const float c = p.scale_log2;

        // -lse * log2(e) and D of query block q_block(it) into buffer it & 1 (threads 0..127 the
        // lse values, 128..255 the D values); -inf / 0 past N so those queries get P = 0.
        // The global load is issued one iteration ahead (load_vectors) and stored to shared
        // memory at the end of the iteration (store_vectors), so its latency stays hidden.
        float staged = 0.f;
        // lse of query head bh_first + g, position q: lse[lse_base + g * lse_hstride + q].
        const size_t lse_hstride = packed ? (size_t)p.T : (size_t)p.N;
        const size_t lse_base = lse_of(packed, b, bh_first - b * p.H, p.H, p.N, p.T, ext.t0, 0);
        auto load_vectors = [&](Step st) {
            const int q = q_block(st) * C::BM + (ct & 127);
            if (ct < 128)
                staged = q < ext.Lq && in_bounds(p.err, lse_base + (size_t)st.g * lse_hstride + q, 1, p.dbg.lse)
                             ? -p.lse[lse_base + (size_t)st.g * lse_hstride + q] * kLog2e
                             : -INFINITY;
            else staged = q < ext.Lq && in_bounds(p.err, (size_t)q_head(st) * p.N + q, 1, p.dbg.vec)
                             ? p.Dvec[(size_t)q_head(st) * p.N + q] : 0.f;
        };
        auto store_vectors = [&](int it) {
            if (ct < 128) s_lse2[(it & 1) * C::BM + ct] = staged;
            else s_D[(it & 1) * C::BM + (ct - 128)] = staged;
        };
        Step st{0, 0};
        load_vectors(st);
        store_vectors(0);
        named_barrier(1, 256);

        // Named barriers have no timeout, so every thread executes every one of them, also
        // after a failed (timed-out or aborted) wait; `ok` then only skips the work.
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = q_block(st);
            st = next_step(st);                      // the step of it + 1 from here on
            const float* lse2 = s_lse2 + (it & 1) * C::BM + 64 * h;
            const float* Dv = s_D + (it & 1) * C::BM + 64 * h;
            if (it + 1 < n_it) load_vectors(st);   // stored at the end of this iteration
            const bool diag = p.causal && (i == j);

            // ---------------- P phase
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull, it & 1, p.timeout_ns, abort_flag));
            float P[64];
            if (ok) {
                tc_fence_after();
                uint32_t sv[64];
                tmem_ld32(tmem + lane_base + C::TM_A + 64 * h, sv);
                tmem_ld32(tmem + lane_base + C::TM_A + 64 * h + 32, sv + 32);
                tmem_ld_wait();
                reg_fence32(sv);
                reg_fence32(sv + 32);
#pragma unroll
                for (int e = 0; e < 64; e += 4) {
                    const float4 nl = *reinterpret_cast<const float4*>(lse2 + e);  // -lse2
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        const float2 x = ffma2(make_float2(__uint_as_float(sv[e + u]),
                                                           __uint_as_float(sv[e + u + 1])),
                                               make_float2(c, c),
                                               u == 0 ? make_float2(nl.x, nl.y) : make_float2(nl.z, nl.w));
                        const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                        P[e + u] = pe.x;
                        P[e + u + 1] = pe.y;
                    }
                }
                if (key_padded || diag) {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        if (key_padded || r > 64 * h + e) P[e] = 0.f;
                }
            }
            // (shared columns only) every S^T column read before P^T overwrites columns
            if constexpr (!OWN) named_barrier(1, 256);
            if (ok) {
                uint32_t pw[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pw[e] = pack_bf16x2(P[2 * e], P[2 * e + 1]);
                tmem_st32(tmem + lane_base + C::TM_A + C::bf16_col(OWN, h), pw);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar_pfull);
            }

            // ---------------- dS phase
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dpfull, it & 1, p.timeout_ns, abort_flag));
            uint32_t dw[32];
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t dp[32];
                    tmem_ld32(tmem + lane_base + C::TM_B + 64 * h + 32 * half, dp);
                    tmem_ld_wait();
                    reg_fence32(dp);
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int ee = 32 * half + e;
                        const float4 dv4 = *reinterpret_cast<const float4*>(Dv + ee);
                        const float2 a = fmul2(make_float2(P[ee], P[ee + 1]),
                                               fadd2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                                     make_float2(-dv4.x, -dv4.y)));
                        const float2 b = fmul2(make_float2(P[ee + 2], P[ee + 3]),
                                               fadd2(make_float2(__uint_as_float(dp[e + 2]), __uint_as_float(dp[e + 3])),
                                                     make_float2(-dv4.z, -dv4.w)));
                        dw[ee / 2] = pack_bf16x2(a.x, a.y);
                        dw[ee / 2 + 1] = pack_bf16x2(b.x, b.y);
                    }
                }
            }
            // Next block's lse / D into the other buffer.  Its last reads were in the previous
            // iteration, before every thread passed that iteration's barrier below, and the
            // barrier below orders these stores before the next iteration's reads.
            if (it + 1 < n_it) store_vectors(it + 1);
            named_barrier(1, 256);  // next step's lse / D stored; shared columns: dP^T read
            if (ok) {
                // d = 128: dK reads dS^T from tensor memory; d = 64 reads the shared tile below.
                if constexpr (D == 128) tmem_st32(tmem + lane_base + C::TM_B + C::bf16_col(OWN, h), dw);
                // dS^T row r, queries [64h, 64h+64) = one 128-byte row of query chunk h; 16-byte
                // unit u sits at position u ^ (r % 8) (the 128-byte swizzle the MMA reads).
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<uint4*>(ds_row + ((u ^ sw) << 4)) =
                        make_uint4(dw[4 * u], dw[4 * u + 1], dw[4 * u + 2], dw[4 * u + 3]);
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar_dsfull);
            }
        }

        // ---------------- epilogue: dV (warpgroup 0) and dK * scale (warpgroup 1)
        if (ok) ok = mbar_wait(bar_done, 0, p.timeout_ns, abort_flag);  // every MMA finished
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const bool key_row = kidx < (packed ? L : p.N);
            const size_t off =
                row_of(packed, b, bhk % p.H_kv, p.H_kv, p.N, ext.t0, key_row ? kidx : 0) * D;
            const uint32_t col0 = h ? C::TM_DK : C::TM_DV;
            const float mul = h ? p.scale : 1.0f;
            const bool in_range = key_row && in_bounds(p.err, off, D, p.dbg.kv);
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(h ? p.dk : p.dv) + off;
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
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

// Persistent backward for launches whose work units all cost the same: head-major, no causal
// mask, no per-sequence key lengths (each unit = one 128-key block of one key/value head, and
// every unit visits every query block of its group's query heads).  One CTA per SM walks the
// units blockIdx.x, blockIdx.x + gridDim.x, ... (key block j of head bhk, head by head).  Per
// query step the arithmetic and the warp roles are fa_bwd_kernel's; across units the Q/dO ring
// and every per-step barrier phase carry over.  The next unit's K and V are loaded once every
// MMA of the previous unit has completed (bar_udone), its first score MMAs overlap the
// previous unit's dK / dV epilogue, and its first dV / dK MMAs (which overwrite the
// accumulators) wait until that epilogue has read them (bar_accfree).
template <int D>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_persist_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmDO, const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr bool OWN = true;  // own-column P^T / dS^T layout
    extern __shared__ __align__(1024) uint8_t smem[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int n_kv = (p.N + C::BN - 1) / C::BN;  // key blocks per head = units per head
    const int n_q = (p.N + C::BM - 1) / C::BM;   // query blocks per head
    const int G = p.H / p.H_kv;                  // query heads sharing a key/value head
    const int n_it = G * n_q;                    // query steps of every unit
    const int n_units = n_kv * p.B * p.H_kv;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
    uint64_t* bar_kv = bars;
    uint64_t* bar_qfull = bars + 1;
    uint64_t* bar_qempty = bar_qfull + C::QST;
    uint64_t* bar_sfull = bar_qempty + C::QST;
    uint64_t* bar_dpfull = bar_sfull + 1;
    uint64_t* bar_pfull = bar_dpfull + 1;
    uint64_t* bar_dsfull = bar_pfull + 1;
    uint64_t* bar_dqfull = bar_dsfull + 1;
    uint64_t* bar_dqempty = bar_dqfull + 1;
    uint64_t* bar_done = bar_dqempty + 1;
    uint64_t* bar_udone = bar_done + 1;    // every MMA of the unit finished
    uint64_t* bar_accfree = bar_udone + 1; // the unit's dK, dV read out of tensor memory
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
    float* s_lse2 = reinterpret_cast<float*>(smem + C::SMEM_VEC);    // [2][BM]
    float* s_D = s_lse2 + 2 * C::BM;                                   // [2][BM]
    float* s_scale = reinterpret_cast<float*>(smem + C::SMEM_SCALE);  // [BM]

    if (threadIdx.x == 0 && (smem_u32(smem) & 1023u)) record_error(p.err, kErrInvalidArg);
    // Unit lin: key block j of key/value head bhk (= b * H_kv + hk).
    struct Unit {
        int bhk, j, bh_first;
    };
    auto unit = [&](int lin) {
        Unit u;
        u.bhk = lin / n_kv;
        u.j = lin - u.bhk * n_kv;
        u.bh_first = (u.bhk / p.H_kv) * p.H + (u.bhk % p.H_kv) * G;
        return u;
    };
    // Step cursor (g = query head of the group, r = step within the head); query block
    // (j + r) mod n_q: the key blocks of a head start at different query blocks.
    struct Step {
        int g, r;
    };
    auto next_step = [&](Step s) {
        return s.r + 1 == n_q ? Step{s.g + 1, 0} : Step{s.g, s.r + 1};
    };
    auto q_block = [&](const Unit& u, Step s) {
        const int i = u.j + s.r;
        return i < n_q ? i : i - n_q;
    };

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < C::QST; ++s) {
            mbar_init(&bar_qfull[s], 1);
            mbar_init(&bar_qempty[s], 1);
        }
        mbar_init(bar_sfull, 1);
        mbar_init(bar_dpfull, 1);
        mbar_init(bar_pfull, 256);
        mbar_init(bar_dsfull, 256);
        mbar_init(bar_dqfull, 1);
        mbar_init(bar_dqempty, 128);
        mbar_init(bar_done, 1);
        mbar_init(bar_udone, 1);
        mbar_init(bar_accfree, 256);
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
        regs_set<C::REGS_DRAIN_PERSIST, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ dQ drain
        const int r = threadIdx.x - 384;  // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        // Named barriers have no timeout: every drain thread executes each of them, for every
        // step of every unit, also after a failed wait (`ok` then only skips the work).
        bool ok = true;
        int gs = 0;  // query steps of earlier units
        for (int lin = blockIdx.x; lin < n_units; lin += gridDim.x, gs += n_it) {
            const Unit u = unit(lin);
            const float factor = head_bound_factor(p, u.bhk);
            // ||dO|| of query row r of step s (-1 past N: scale 0), loaded one step ahead
            auto load_norm = [&](Step s) -> float {
                const int q = q_block(u, s) * C::BM + r;
                const int qh = u.bh_first + s.g;
                return q < p.N && in_bounds(p.err, (size_t)qh * p.N + q, 1, p.dbg.vec)
                           ? p.dOnorm[(size_t)qh * p.N + q] : -1.f;
            };
            Step st{0, 0};
            float norm = load_norm(st);
            for (int it = 0; it < n_it; ++it, st = next_step(st)) {
                const int q0 = q_block(u, st) * C::BM;
                const int qh = u.bh_first + st.g;
                s_scale[r] = norm >= 0.f ? fmaxf(fixed_point_scale(norm, factor), 0.f) : 0.f;
                if (it + 1 < n_it) norm = load_norm(next_step(st));
                named_barrier(2, 128);
                const float* sc = s_scale;
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dqfull, (gs + it) & 1, p.timeout_ns, abort_flag));
                if (ok) {
                    tc_fence_after();
                    constexpr int NV = (D == 128) ? 128 : 64;
                    uint32_t v[NV];
#pragma unroll
                    for (int q = 0; q < NV / 32; ++q) tmem_ld32(tmem + lane_base + C::TM_B + 32 * q, v + 32 * q);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < NV / 32; ++q) reg_fence32(v + 32 * q);
                    tc_fence_before();
                    mbar_arrive(bar_dqempty);  // B may take the next dP^T
                    int* acc = p.dq_acc + ((size_t)qh * p.N_pad + q0) * D;
                    if (in_bounds(p.err, ((size_t)qh * p.N_pad + q0) * D, (size_t)C::BM * D, p.dbg.acc)) {
                        if constexpr (D == 128) {
#pragma unroll
                            for (int e = 0; e < 128; e += 4) {
                                const float4 s4 = *reinterpret_cast<const float4*>(sc + e);  // one shared load
                                const int2 x = to_fixed2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), s4.x, s4.y);
                                const int2 y = to_fixed2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]), s4.z, s4.w);
                                red_add_s32(acc + (size_t)e * D + r, x.x);
                                red_add_s32(acc + (size_t)(e + 1) * D + r, x.y);
                                red_add_s32(acc + (size_t)(e + 2) * D + r, y.x);
                                red_add_s32(acc + (size_t)(e + 3) * D + r, y.y);
                            }
                        } else {
                            int* xp = reinterpret_cast<int*>(smem + C::SMEM_XPOSE) + (warp % 4) * 32 * 33;
                            const float s_row = sc[r];
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
#pragma unroll
                                for (int e = 0; e < 32; e += 2) {
                                    const int2 x = to_fixed2(__uint_as_float(v[32 * c + e]),
                                                             __uint_as_float(v[32 * c + e + 1]), s_row, s_row);
                                    xp[lane * 33 + e] = x.x;
                                    xp[lane * 33 + e + 1] = x.y;
                                }
                                __syncwarp();
#pragma unroll 4
                                for (int row = 0; row < 32; ++row)
                                    red_add_s32(acc + (size_t)((warp % 4) * 32 + row) * D + 32 * c + lane,
                                                xp[row * 33 + lane]);
                                __syncwarp();
                            }
                        }
                    }
                }
                named_barrier(2, 128);  // every read of s_scale done before the next step writes
            }
        }
        if (!ok) fail();
    } else if (warp >= 8) {
      regs_set<C::REGS_OTHER_PERSIST, C::REGS_LAUNCH>();
      if (warp == 9 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmDO);
        bool ok = true;
        int gq = 0;  // Q/dO stages filled
        int uc = 0;  // units started
        for (int lin = blockIdx.x; ok && lin < n_units; lin += gridDim.x, ++uc) {
            const Unit u = unit(lin);
            // K and V stay in place for the whole unit: reload once the previous unit's MMAs,
            // the last readers, have completed.
            if (uc > 0 && !(ok = mbar_wait(bar_udone, (uc - 1) & 1, p.timeout_ns, abort_flag))) break;
            mbar_arrive_expect_tx(bar_kv, 2 * C::KV_TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(smem + C::SMEM_K + c * C::CHUNK_BYTES, &tmK, bar_kv, c * 64, u.j * C::BN, u.bhk);
                tma_load_3d(smem + C::SMEM_V + c * C::CHUNK_BYTES, &tmV, bar_kv, c * 64, u.j * C::BN, u.bhk);
            }
            Step st{0, 0};
            for (int it = 0; it < n_it; ++it, st = next_step(st), ++gq) {
                const int s = gq % C::QST;
                const uint32_t ph = (gq / C::QST) & 1;
                const int q0 = q_block(u, st) * C::BM;
                const int qh = u.bh_first + st.g;
                if (!(ok = mbar_wait(&bar_qempty[s], ph ^ 1, p.timeout_ns, abort_flag))) break;
                mbar_arrive_expect_tx(&bar_qfull[s], 2 * C::Q_TILE_BYTES);
                for (int c = 0; c < C::KCH; ++c) {
                    tma_load_3d(smem + C::SMEM_Q + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES, &tmQ,
                                &bar_qfull[s], c * 64, q0, qh);
                    tma_load_3d(smem + C::SMEM_DO + s * C::Q_TILE_BYTES + c * C::CHUNK_BYTES,
                                &tmDO, &bar_qfull[s], c * 64, q0, qh);
                }
            }
        }
        if (!ok) fail();
        // Do not leave while our copies may still be landing in shared memory.
        for (int t = max(0, gq - C::QST); t < gq; ++t)
            mbar_wait_drain(&bar_qfull[t % C::QST], (t / C::QST) & 1, p.timeout_ns);
        if (uc > 0) mbar_wait_drain(bar_kv, (uc - 1) & 1, p.timeout_ns);
      } else if (warp == 8 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idS = idesc_bf16(128, 128, false, false);  // S^T, dP^T
        constexpr uint32_t idKV = idesc_bf16(128, D, false, true);    // dV, dK (A in TMEM)
        constexpr uint32_t idQ = idesc_bf16(128, D == 128 ? 128 : 64, true, true);  // dQ^T / dQ
        const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::SMEM_K), 16, 1024);
        const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::SMEM_V), 16, 1024);
        const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + C::SMEM_K), C::CHUNK_BYTES, 1024);
        const uint64_t dDS_mn = sdesc_sw128(smem_u32(smem + C::SMEM_DS), C::CHUNK_BYTES, 1024);
        const uint64_t dDS_k = sdesc_sw128(smem_u32(smem + C::SMEM_DS), 16, 1024);
        const uint64_t dQ_k0 = sdesc_sw128(smem_u32(smem + C::SMEM_Q), 16, 1024);
        const uint64_t dDO_k0 = sdesc_sw128(smem_u32(smem + C::SMEM_DO), 16, 1024);
        const uint64_t dQ_mn0 = sdesc_sw128(smem_u32(smem + C::SMEM_Q), C::CHUNK_BYTES, 1024);
        const uint64_t dDO_mn0 = sdesc_sw128(smem_u32(smem + C::SMEM_DO), C::CHUNK_BYTES, 1024);
        auto kmaj = [](int kk) { return (uint64_t)(((kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32) >> 4); };
        auto mnmaj = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };
        auto stage_off = [](int g) { return (uint64_t)((g % C::QST) * (C::Q_TILE_BYTES >> 4)); };
        auto issue_S = [&](int g) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_A, dK_k + kmaj(kk), dQ_k0 + stage_off(g) + kmaj(kk), idS,
                       kk > 0 ? 1u : 0u);
            tc_commit(bar_sfull);
        };
        auto issue_dP = [&](int g) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::TM_B, dV_k + kmaj(kk), dDO_k0 + stage_off(g) + kmaj(kk), idS,
                       kk > 0 ? 1u : 0u);
            tc_commit(bar_dpfull);
        };
        // Per unit, as fa_bwd_kernel: S^T(0), dP^T(0), then per step dV, S^T(+1), dK, dQ,
        // dP^T(+1); g = this CTA's global step index (every per-step barrier's phase).
        bool ok = true;
        int gs = 0;  // steps of earlier units
        int uc = 0;
        for (int lin = blockIdx.x; ok && lin < n_units; lin += gridDim.x, ++uc, gs += n_it) {
            if (!(ok = mbar_wait(bar_kv, uc & 1, p.timeout_ns, abort_flag))) break;
            if (!(ok = mbar_wait(&bar_qfull[gs % C::QST], (gs / C::QST) & 1, p.timeout_ns, abort_flag)))
                break;
            tc_fence_after();
            issue_S(gs);
            // B held the previous unit's last dQ block: wait until the drain copied it out.
            if (gs > 0 && !(ok = mbar_wait(bar_dqempty, (gs - 1) & 1, p.timeout_ns, abort_flag))) break;
            tc_fence_after();
            issue_dP(gs);
            for (int it = 0; ok && it < n_it; ++it) {
                const int g = gs + it;
                const int s = g % C::QST;
                const uint64_t dQ_mn = dQ_mn0 + stage_off(g), dDO_mn = dDO_mn0 + stage_off(g);
                if (!(ok = mbar_wait(bar_pfull, g & 1, p.timeout_ns, abort_flag))) break;
                // The first dV / dK of a unit overwrite the accumulators: the previous unit's
                // epilogue must have read them.
                if (it == 0 && uc > 0 &&
                    !(ok = mbar_wait(bar_accfree, (uc - 1) & 1, p.timeout_ns, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C::BM / 16; ++kk)
                    mma_ts(tmem + C::TM_DV, tmem + C::TM_A + C::a_col(OWN, kk), dDO_mn + mnmaj(kk), idKV,
                           (it > 0 || kk > 0) ? 1u : 0u);
                if (it + 1 < n_it) {
                    if (!(ok = mbar_wait(&bar_qfull[(g + 1) % C::QST], ((g + 1) / C::QST) & 1,
                                         p.timeout_ns, abort_flag)))
                        break;
                    tc_fence_after();
                    issue_S(g + 1);
                }
                if (!(ok = mbar_wait(bar_dsfull, g & 1, p.timeout_ns, abort_flag))) break;
                tc_fence_after();
                if constexpr (D == 128) {
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)
                        mma_ts(tmem + C::TM_DK, tmem + C::TM_B + C::a_col(OWN, kk), dQ_mn + mnmaj(kk), idKV,
                               (it > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_qempty[s]);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_ss(tmem + C::TM_B, dK_mn + mnmaj(kk), dDS_mn + mnmaj(kk), idQ,
                               kk > 0 ? 1u : 0u);
                    tc_commit(bar_dqfull);
                } else {
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_ss(tmem + C::TM_B, dDS_mn + mnmaj(kk), dK_mn + mnmaj(kk), idQ,
                               kk > 0 ? 1u : 0u);
                    tc_commit(bar_dqfull);
#pragma unroll
                    for (int kk = 0; kk < C::BM / 16; ++kk)
                        mma_ss(tmem + C::TM_DK, dDS_k + kmaj(kk), dQ_mn + mnmaj(kk), idKV,
                               (it > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&bar_qempty[s]);
                }
                if (it + 1 < n_it) {
                    if (!(ok = mbar_wait(bar_dqempty, g & 1, p.timeout_ns, abort_flag))) break;
                    tc_fence_after();
                    issue_dP(g + 1);
                }
            }
            tc_commit(bar_udone);  // every MMA of the unit: K, V and the accumulators are final
        }
        if (!ok) fail();
        tc_commit(bar_done);
        mbar_wait_drain(bar_done, 0, p.timeout_ns);
      }
    } else {
        regs_set<C::REGS_COMPUTE_PERSIST, C::REGS_LAUNCH>();
        // ------------------------------------------------------------ compute warpgroups
        const int h = warp / 4;           // query-column half
        const int r = threadIdx.x % 128;  // TMEM lane
        const int ct = threadIdx.x;       // 0..255
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        uint8_t* ds_row = smem + C::SMEM_DS + h * C::CHUNK_BYTES + r * 128;
        const int sw = r & 7;
        const float c = p.scale_log2;
        float staged = 0.f;
        // Named barriers have no timeout, so every thread executes every one of them, for every
        // step of every unit, also after a failed wait; `ok` then only skips the work.
        bool ok = true;
        int gs = 0;
        int uc = 0;
        for (int lin = blockIdx.x; lin < n_units; lin += gridDim.x, ++uc, gs += n_it) {
            const Unit u = unit(lin);
            const bool key_padded = u.j * C::BN + r >= p.N;
            auto load_vectors = [&](Step st) {
                const int q = q_block(u, st) * C::BM + (ct & 127);
                const size_t idx = (size_t)(u.bh_first + st.g) * p.N + q;
                if (ct < 128)
                    staged = q < p.N && in_bounds(p.err, idx, 1, p.dbg.lse) ? -p.lse[idx] * kLog2e
                                                                           : -INFINITY;
                else
                    staged = q < p.N && in_bounds(p.err, idx, 1, p.dbg.vec) ? p.Dvec[idx] : 0.f;
            };
            auto store_vectors = [&](int g) {
                if (ct < 128) s_lse2[(g & 1) * C::BM + ct] = staged;
                else s_D[(g & 1) * C::BM + (ct - 128)] = staged;
            };
            Step st{0, 0};
            load_vectors(st);
            store_vectors(gs);
            named_barrier(1, 256);
            for (int it = 0; it < n_it; ++it) {
                const int g = gs + it;
                st = next_step(st);
                const float* lse2 = s_lse2 + (g & 1) * C::BM + 64 * h;
                const float* Dv = s_D + (g & 1) * C::BM + 64 * h;
                if (it + 1 < n_it) load_vectors(st);

                // ---------------- P phase
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull, g & 1, p.timeout_ns, abort_flag));
                float P[64];
                if (ok) {
                    tc_fence_after();
                    uint32_t sv[64];
                    tmem_ld32(tmem + lane_base + C::TM_A + 64 * h, sv);
                    tmem_ld32(tmem + lane_base + C::TM_A + 64 * h + 32, sv + 32);
                    tmem_ld_wait();
                    reg_fence32(sv);
                    reg_fence32(sv + 32);
#pragma unroll
                    for (int e = 0; e < 64; e += 4) {
                        const float4 nl = *reinterpret_cast<const float4*>(lse2 + e);
#pragma unroll
                        for (int v2 = 0; v2 < 4; v2 += 2) {
                            const float2 x = ffma2(make_float2(__uint_as_float(sv[e + v2]),
                                                               __uint_as_float(sv[e + v2 + 1])),
                                                   make_float2(c, c),
                                                   v2 == 0 ? make_float2(nl.x, nl.y) : make_float2(nl.z, nl.w));
                            P[e + v2] = ex2(x.x);
                            P[e + v2 + 1] = ex2(x.y);
                        }
                    }
                    if (key_padded) {
#pragma unroll
                        for (int e = 0; e < 64; ++e) P[e] = 0.f;
                    }
                }
                // (shared columns only) every S^T column read before P^T overwrites columns
                if constexpr (!OWN) named_barrier(1, 256);
                if (ok) {
                    uint32_t pw[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) pw[e] = pack_bf16x2(P[2 * e], P[2 * e + 1]);
                    tmem_st32(tmem + lane_base + C::TM_A + C::bf16_col(OWN, h), pw);
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(bar_pfull);
                }

                // ---------------- dS phase
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_dpfull, g & 1, p.timeout_ns, abort_flag));
                uint32_t dw[32];
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t dp[32];
                        tmem_ld32(tmem + lane_base + C::TM_B + 64 * h + 32 * half, dp);
                        tmem_ld_wait();
                        reg_fence32(dp);
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const int ee = 32 * half + e;
                            const float4 dv4 = *reinterpret_cast<const float4*>(Dv + ee);
                            const float2 a = fmul2(make_float2(P[ee], P[ee + 1]),
                                                   fadd2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                                         make_float2(-dv4.x, -dv4.y)));
                            const float2 bb = fmul2(make_float2(P[ee + 2], P[ee + 3]),
                                                    fadd2(make_float2(__uint_as_float(dp[e + 2]), __uint_as_float(dp[e + 3])),
                                                          make_float2(-dv4.z, -dv4.w)));
                            dw[ee / 2] = pack_bf16x2(a.x, a.y);
                            dw[ee / 2 + 1] = pack_bf16x2(bb.x, bb.y);
                        }
                    }
                }
                if (it + 1 < n_it) store_vectors(g + 1);
                named_barrier(1, 256);  // next step's lse / D stored; shared columns: dP^T read
                if (ok) {
                    if constexpr (D == 128) tmem_st32(tmem + lane_base + C::TM_B + C::bf16_col(OWN, h), dw);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        *reinterpret_cast<uint4*>(ds_row + ((v4 ^ sw) << 4)) =
                            make_uint4(dw[4 * v4], dw[4 * v4 + 1], dw[4 * v4 + 2], dw[4 * v4 + 3]);
                    tmem_st_wait();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(bar_dsfull);
                }
            }

            // ---------------- epilogue of the unit: dV (warpgroup 0) and dK * scale (1)
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_udone, uc & 1, p.timeout_ns, abort_flag));
            if (ok) {
                tc_fence_after();
                const int kidx = u.j * C::BN + r;
                const size_t off = ((size_t)u.bhk * p.N + (kidx < p.N ? kidx : 0)) * D;
                const uint32_t col0 = h ? C::TM_DK : C::TM_DV;
                const float mul = h ? p.scale : 1.0f;
                const bool in_range = kidx < p.N && in_bounds(p.err, off, D, p.dbg.kv);
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(h ? p.dk : p.dv) + off;
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
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
                tc_fence_before();
                mbar_arrive(bar_accfree);  // the next unit's first dV / dK may overwrite them
            }
        }
        if (!ok) fail();
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
cudaError_t launch_bwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream,
                         cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    using C = BwdCfg<D>;
    static std::atomic<uint64_t> configured{0};  // one bit per device
    if (cudaError_t e = set_smem_limit_once(configured, C::SMEM_BYTES,
                                            fa_bwd_kernel<D, PACKED, false>,
                                            fa_bwd_kernel<D, PACKED, !PACKED>,
                                            fa_bwd_persist_kernel<D>);
        e != cudaSuccess)
        return e;
    const int BH = p.B * p.H;
    const int n_kv = (p.N + C::BN - 1) / C::BN;
    const int BHkv = p.B * p.H_kv;
    const dim3 chunks(p.N_pad / 128, BH);
    fa_bwd_pre_kernel<D><<<chunks, 256, 0, stream>>>(p);
    if (ev_start) cudaEventRecord(ev_start, stream);
    // Units of equal cost (head-major, no causal mask, no key lengths), more of them than SMs,
    // and short (at most 16 query steps, where a unit's start-up and epilogue are a large part
    // of it): the persistent kernel, one CTA per SM.  Measured +6 to +14 % up to N = 2048,
    // neutral or 1-2 % slower at N = 4096 (its register split is tighter).  Otherwise one CTA
    // per key block, in the heaviest-first order for causal launches, which the hardware's CTA
    // scheduler balances better than a static assignment when units differ in cost.  Both
    // compute the same arithmetic in the same order: the results are bitwise identical.
    const int steps = (p.H / p.H_kv) * ((p.N + C::BM - 1) / C::BM);
    if (!PACKED && !p.causal && p.seqlens == nullptr && p.num_sms > 0 && steps <= 16 &&
        (long long)BHkv * n_kv > p.num_sms)
        fa_bwd_persist_kernel<D><<<p.num_sms, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    // Head-major causal launches take the grouped heaviest-first order (their own
    // instantiation, so that the other launches keep their code unchanged).
    else if (!PACKED && p.causal)
        fa_bwd_kernel<D, PACKED, !PACKED><<<BHkv * n_kv, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    else
        fa_bwd_kernel<D, PACKED, false><<<BHkv * n_kv, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
    if (ev_stop) cudaEventRecord(ev_stop, stream);
    fa_bwd_dq_kernel<D><<<chunks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

// d = 256 (fa_bwd_d256.cu, both layouts): Q and dO maps with 64-row boxes.
cudaError_t launch_bwd_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream,
                            cudaEvent_t ev_start, cudaEvent_t ev_stop);

cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream,
                       cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    const bool packed = p.cu_seqlens != nullptr;
    if (d == 256) return launch_bwd_d256(tq, tk, tv, tdo, p, stream, ev_start, ev_stop);
    if (d == 64)
        return packed ? launch_bwd_d<64, true>(tq, tk, tv, tdo, p, stream, ev_start, ev_stop)
                      : launch_bwd_d<64, false>(tq, tk, tv, tdo, p, stream, ev_start, ev_stop);
    return packed ? launch_bwd_d<128, true>(tq, tk, tv, tdo, p, stream, ev_start, ev_stop)
                  : launch_bwd_d<128, false>(tq, tk, tv, tdo, p, stream, ev_start, ev_stop);
}

}  // namespace fa
