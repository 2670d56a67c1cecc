// fa_bwd_common.cuh -- pieces shared by the backward kernels of every head dim (fa_bwd.cu
// for d = 64 and 128, fa_bwd_d256.cu for d = 256): the fixed-point dQ scale, the preprocess
// kernel (D, norms, bound maxima, clearing the dQ accumulator) and the dQ conversion kernel.
// Included inside namespace fa { namespace { ... } } of each translation unit.
#pragma once

constexpr float kLog2e = 1.4426950408889634f;


__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// Head constant 2 max_j |v_j| max_{j,l} |k_jl| from the per-chunk maxima (same arithmetic in
// every kernel that needs it, so every kernel derives the same scales).
__device__ __forceinline__ float head_bound_factor(const BwdParams& p, int bh) {
    const int chunks = p.N_pad / 128;
    const float* hm = p.headmax + (size_t)bh * chunks * 2;
    float vmax = 0.f, kmax = 0.f;
    if (!in_bounds(p.err, (size_t)bh * chunks * 2, (size_t)chunks * 2, p.dbg.hmax)) return 0.f;
    for (int c = 0; c < chunks; ++c) {
        vmax = fmaxf(vmax, hm[2 * c]);
        kmax = fmaxf(kmax, hm[2 * c + 1]);
    }
    return 2.0f * vmax * kmax;
}

// Fixed-point scale of a query row: the largest power of two s with s * bound <= 2^29.  The
// bound caps every partial sum of the row's dQ (see the file comments of the kernels), so the
// integer sums stay below 2^29 plus one rounding per key block: int32 never overflows, with a
// factor 4 to spare for the rounding of P, dS and O.  0 when the bound is 0 (every
// contribution of the row is then 0); -1 when the bound is not finite (input norms beyond
// fp32 range), which the dQ conversion reports as FA_ERR_INVALID_ARG.
__device__ __forceinline__ float fixed_point_scale(float dO_norm, float head_factor) {
    const float bound = dO_norm * head_factor;
    if (bound == 0.f) return 0.f;
    if (!(bound <= 3.4e38f)) return -1.f;
    // a tiny bound would push s past the fp32 range: any s with s * bound <= 2^29 will do
    const float x = fminf(536870912.0f / bound, 0x1p100f);
    return __int_as_float(__float_as_int(x) & 0x7F800000);  // 2^floor(log2 x), exact
}

// round(v * s) to the nearest integer (ties to even) for |v * s| < 2^38, on the FMA and
// integer pipes (the conversion instruction would run on the unit the exponentials need).
// x = v * s is split as x = h + l: adding 1.5 * 2^39 rounds x to h, a multiple of 2^16, whose
// quotient h / 2^16 sits in the low mantissa bits of the sum (last place 2^16); l = x - h,
// |l| <= 2^15, is exact (one fused multiply-add) and is rounded the same way with 1.5 * 2^23.
// Then round(x) = h + round(l), formed as a 32-bit integer (the callers keep |x| < 2^30).
__device__ __forceinline__ int to_fixed(float v, float s) {
    constexpr float kHi = 824633720832.0f;  // 1.5 * 2^39
    constexpr float kLo = 12582912.0f;      // 1.5 * 2^23
    const float t = fmaf(v, s, kHi);
    const float h = t - kHi;
    const float u = fmaf(v, s, -h) + kLo;
    return (__float_as_int(t) - __float_as_int(kHi)) * 65536 + (__float_as_int(u) - __float_as_int(kLo));
}

// to_fixed of two values with their own scales, the floating-point steps as packed pairs.
__device__ __forceinline__ int2 to_fixed2(float v0, float v1, float s0, float s1) {
    constexpr float kHi = 824633720832.0f;
    constexpr float kLo = 12582912.0f;
    const float2 v = make_float2(v0, v1), s = make_float2(s0, s1);
    const float2 t = ffma2(v, s, make_float2(kHi, kHi));
    const float2 h = fadd2(t, make_float2(-kHi, -kHi));
    const float2 u = fadd2(ffma2(v, s, make_float2(-h.x, -h.y)), make_float2(kLo, kLo));
    return make_int2(
        (__float_as_int(t.x) - __float_as_int(kHi)) * 65536 + (__float_as_int(u.x) - __float_as_int(kLo)),
        (__float_as_int(t.y) - __float_as_int(kHi)) * 65536 + (__float_as_int(u.y) - __float_as_int(kLo)));
}

// ---------------------------------------------------------------------------- preprocess
// Grid (N_pad / 128 chunks, B*H).  Per query row: D = dO . O (fp32) and |dO|; per chunk of
// key/value head (blocks y < B*H_kv): the largest |v_j| and |k_jl| of its visible key rows
// (j < L_b); and the chunk's rows of the dQ accumulator set to zero.  TPR threads per row, each reading 16 bytes of every tensor.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p) {
    constexpr int TPR = D / 8;               // threads per row
    constexpr int RPP = 256 / TPR;           // rows per pass
    const int chunk = blockIdx.x;
    const int bh = blockIdx.y;                       // query head (b, h)
    const int part = threadIdx.x % TPR;
    // Blocks of the first B * H_kv heads also scan key/value head bh for the bound maxima; only
    // keys some query can see enter them (padded keys contribute nothing to dQ).
    const bool packed = p.cu_seqlens != nullptr;
    const bool kv_head = bh < p.B * p.H_kv;
    const int bq = bh / p.H, bk = bh / p.H_kv;
    const SeqExtent eq = sequence_extent(p, bq, false, packed);
    const SeqExtent ek = kv_head ? sequence_extent(p, bk, false, packed) : SeqExtent{0, 0, 0};
    const int L = ek.L;
    float vmax = 0.f, kmax = 0.f;
    for (int rr = threadIdx.x / TPR; rr < 128; rr += RPP) {
        const int n = chunk * 128 + rr;
        float dd = 0.f, nn = 0.f, vv = 0.f, ka = 0.f;
        if (n < eq.Lq) {
            const size_t off = row_of(packed, bq, bh % p.H, p.H, p.N, eq.t0, n) * TPR + part;
            if (in_bounds(p.err, off * 8, 8, p.dbg.q)) {
                const uint4 a = reinterpret_cast<const uint4*>(p.dO)[off];
                const uint4 o = reinterpret_cast<const uint4*>(p.o)[off];
                const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
                const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 fa = __bfloat1622float2(a2[i]);
                    const float2 fo = __bfloat1622float2(o2[i]);
                    dd = fmaf(fa.x, fo.x, fmaf(fa.y, fo.y, dd));
                    nn = fmaf(fa.x, fa.x, fmaf(fa.y, fa.y, nn));
                }
            }
        }
        if (n < L) {
            const size_t off = row_of(packed, bk, bh % p.H_kv, p.H_kv, p.N, ek.t0, n) * TPR + part;
            if (in_bounds(p.err, off * 8, 8, p.dbg.kv)) {
                const uint4 v = reinterpret_cast<const uint4*>(p.v)[off];
                const uint4 k = reinterpret_cast<const uint4*>(p.k)[off];
                const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&k);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 fv = __bfloat1622float2(v2[i]);
                    const float2 fk = __bfloat1622float2(k2[i]);
                    vv = fmaf(fv.x, fv.x, fmaf(fv.y, fv.y, vv));
                    ka = fmaxf(ka, fmaxf(fabsf(fk.x), fabsf(fk.y)));
                }
            }
        }
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) {
            dd += __shfl_xor_sync(0xffffffffu, dd, off);
            nn += __shfl_xor_sync(0xffffffffu, nn, off);
            vv += __shfl_xor_sync(0xffffffffu, vv, off);
            ka = fmaxf(ka, __shfl_xor_sync(0xffffffffu, ka, off));
        }
        if (n < p.N && part == 0 && in_bounds(p.err, (size_t)bh * p.N + n, 1, p.dbg.vec)) {
            p.Dvec[(size_t)bh * p.N + n] = dd;
            p.dOnorm[(size_t)bh * p.N + n] = sqrtf(nn);
        }
        vmax = fmaxf(vmax, sqrtf(vv));
        kmax = fmaxf(kmax, ka);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
        kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    __shared__ float red[2][8];
    if (threadIdx.x % 32 == 0) {
        red[0][threadIdx.x / 32] = vmax;
        red[1][threadIdx.x / 32] = kmax;
    }
    // zero this chunk's 128 rows of the accumulator
    int4* acc = reinterpret_cast<int4*>(p.dq_acc + ((size_t)bh * p.N_pad + (size_t)chunk * 128) * D);
    if (in_bounds(p.err, ((size_t)bh * p.N_pad + (size_t)chunk * 128) * D, 128 * D, p.dbg.acc))
        for (int i = threadIdx.x; i < 128 * D / 4; i += 256) acc[i] = make_int4(0, 0, 0, 0);
    __syncthreads();
    if (threadIdx.x == 0 && kv_head &&
        in_bounds(p.err, ((size_t)bh * (p.N_pad / 128) + chunk) * 2, 2, p.dbg.hmax)) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < 8; ++w) {
            a = fmaxf(a, red[0][w]);
            b = fmaxf(b, red[1][w]);
        }
        float* hm = p.headmax + ((size_t)bh * (p.N_pad / 128) + chunk) * 2;
        hm[0] = a;
        hm[1] = b;
    }
}

// ---------------------------------------------------------------------------- dQ convert
// Grid (N_pad / 128 chunks, B*H): dq = bf16(scale * acc / s_i) for the chunk's real rows.  A row
// whose bound is not finite gets dq = 0 and FA_ERR_INVALID_ARG in the error flag.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p) {
    const int chunk = blockIdx.x;
    const int bh = blockIdx.y;
    __shared__ float s_factor;
    if (threadIdx.x == 0)
        s_factor = head_bound_factor(p, (bh / p.H) * p.H_kv + (bh % p.H) / (p.H / p.H_kv));
    __syncthreads();
    const float factor = s_factor;
    const bool packed = p.cu_seqlens != nullptr;
    const int b = bh / p.H;
    const SeqExtent e = sequence_extent(p, b, false, packed);
    constexpr int PER_ROW = D / 8;  // 8 elements per thread-step
    for (int i = threadIdx.x; i < 128 * PER_ROW; i += 256) {
        const int rr = i / PER_ROW, c8 = (i % PER_ROW) * 8;
        const int n = chunk * 128 + rr;
        if (n >= e.Lq) continue;
        const size_t a_off = ((size_t)bh * p.N_pad + n) * D + c8;
        const size_t q_off = row_of(packed, b, bh % p.H, p.H, p.N, e.t0, n) * D + c8;
        if (!in_bounds(p.err, (size_t)bh * p.N + n, 1, p.dbg.vec) ||
            !in_bounds(p.err, a_off, 8, p.dbg.acc) || !in_bounds(p.err, q_off, 8, p.dbg.q))
            continue;
        const float s = fixed_point_scale(p.dOnorm[(size_t)bh * p.N + n], factor);
        if (s < 0.f && c8 == 0) record_error(p.err, kErrInvalidArg);  // bound beyond fp32
        const float mul = s > 0.f ? p.scale / s : 0.f;  // 1 / s is a power of two: exact
        const int4* src = reinterpret_cast<const int4*>(p.dq_acc + a_off);
        const int4 x = src[0], y = src[1];
        uint4 out;
        out.x = pack_bf16x2((float)x.x * mul, (float)x.y * mul);
        out.y = pack_bf16x2((float)x.z * mul, (float)x.w * mul);
        out.z = pack_bf16x2((float)y.x * mul, (float)y.y * mul);
        out.w = pack_bf16x2((float)y.z * mul, (float)y.w * mul);
        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dq) + q_off) = out;
    }
}

