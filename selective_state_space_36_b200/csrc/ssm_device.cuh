// ssm_device.cuh -- device helpers shared by the scan and decode kernels:
// element I/O for fp32 / bf16 tensors and the transcendental functions of
// the selective SSM (exp of the decay, softplus for tau_Delta, silu gate).
//
// Two precision tiers:
//  * PRECISE (fp32 I/O): libdevice expf / log1pf and IEEE division.
//  * fast (bf16 I/O): the SFU's ex2.approx / lg2.approx / rcp.approx, with a
//    short series for log1p of small arguments so that tau_Delta keeps ~1e-7
//    relative accuracy where Delta is small (Delta ~ 1e-3 is the common case
//    and the state integrates its error over ~1/(Delta |A|) steps).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- element I/O
template <typename T> struct io_traits;

template <> struct io_traits<float> {
    static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ float load_stream(const float *p) { return __ldcs(p); }
    static __device__ __forceinline__ float load_smem(const float *p) { return *p; }
    // four consecutive values from a 16-byte aligned shared-memory address
    static __device__ __forceinline__ void load4_smem(const float *p, float *v) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
    // four consecutive values from a 16-byte aligned address
    static __device__ __forceinline__ void load4(const float *p, float *v) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
    static __device__ __forceinline__ void store(float *p, float v) { __stcs(p, v); }
    static __device__ __forceinline__ void store_smem(float *p, float v) { *p = v; }
};

template <> struct io_traits<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
        return __bfloat162float(__ldg(p));
    }
    static __device__ __forceinline__ float load_stream(const __nv_bfloat16 *p) {
        unsigned short r = __ldcs(reinterpret_cast<const unsigned short *>(p));
        return __uint_as_float(static_cast<uint32_t>(r) << 16);
    }
    static __device__ __forceinline__ float load_smem(const __nv_bfloat16 *p) {
        return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(p)) << 16);
    }
    // four consecutive values from an 8-byte aligned shared-memory address
    static __device__ __forceinline__ void load4_smem(const __nv_bfloat16 *p, float *v) {
        const uint2 t = *reinterpret_cast<const uint2 *>(p);
        v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
    // four consecutive values from an 8-byte aligned address
    static __device__ __forceinline__ void load4(const __nv_bfloat16 *p, float *v) {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
        v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        __stcs(reinterpret_cast<unsigned short *>(p), *reinterpret_cast<unsigned short *>(&b));
    }
    static __device__ __forceinline__ void store_smem(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// ------------------------------------------------------------- SFU wrappers
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ softplus
// softplus(s) = log(1 + e^s) = max(s, 0) + log1p(e), e = exp(-|s|) in (0, 1].
//
// Fast tier: e from the SFU, then log1p(e) = e * q(e) with q a degree-8
// polynomial fitted to log1p(e)/e on [0, 1] (Lawson-weighted least squares on
// 4000 Chebyshev nodes, relative error; q(0) = 1 exactly).  Evaluated in fp32
// its relative error is below 1.6e-7 over the whole interval, so Delta keeps
// full fp32-level relative accuracy even when it is ~1e-3 (the common case,
// where an absolute-error logarithm would lose three digits).
#define SSM_LOG1P_Q                                                                          \
    {1.0f, -0.49999648332595825f, 0.3332132399082184f, -0.24857163429260254f,               \
     0.1915365308523178f, -0.13753798604011536f, 0.0792044997215271f, -0.03006576932966709f, \
     0.005364818498492241f}

__device__ __forceinline__ float log1p_unit(float e) {  // e in [0, 1]
    constexpr float q[9] = SSM_LOG1P_Q;
    float p = q[8];
#pragma unroll
    for (int k = 7; k >= 0; --k) p = fmaf(p, e, q[k]);
    return p * e;
}

template <bool PRECISE>
__device__ __forceinline__ float softplus(float s) {
    if (PRECISE) return fmaxf(s, 0.f) + log1pf(expf(-fabsf(s)));
    return fmaxf(s, 0.f) + log1p_unit(ex2_approx(-fabsf(s) * kLog2e));
}

// -------------------------------------------------------------------- silu
// Fast tier: silu(z) = z sigmoid(z) = h (1 + tanh(h)), h = z / 2 -- one SFU op.
template <bool PRECISE>
__device__ __forceinline__ float silu(float z) {
    if (PRECISE) return z / (1.f + expf(-z));
    const float hz = 0.5f * z;
    return fmaf(hz, tanh_approx(hz), hz);
}

// Decay Abar = exp(Delta * A).  The fast tier takes A pre-multiplied by log2(e).
template <bool PRECISE>
__device__ __forceinline__ float decay(float dl, float a_scaled) {
    if (PRECISE) return expf(dl * a_scaled);
    return ex2_approx(dl * a_scaled);
}

// The same, given the product x = Delta * A (times log2(e) in the fast tier).
template <bool PRECISE>
__device__ __forceinline__ float decay_of(float x) {
    if (PRECISE) return expf(x);
    return ex2_approx(x);
}

// Fast-tier decay pair exp2(Delta * Aw) evaluated anew, bit for bit what
// mul2 + decay_of<false> give.  The statement is volatile so that the
// compiler does not merge it with an earlier evaluation of the same decays: a
// kernel that recomputes decays instead of keeping them (to save the registers
// that would hold them) gets the recomputation it asked for.
__device__ __forceinline__ float2 decay2_fresh(float2 dl2, float2 aw2) {
    float2 r;
    asm volatile(
        "{\n.reg .b64 ra, rb, rd;\n.reg .f32 x0, x1;\nmov.b64 ra, {%2,%3};\nmov.b64 rb, {%4,%5};\n"
        "mul.rn.f32x2 rd, ra, rb;\nmov.b64 {x0,x1}, rd;\nex2.approx.ftz.f32 %0, x0;\nex2.approx.ftz.f32 %1, x1;\n}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(dl2.x), "f"(dl2.y), "f"(aw2.x), "f"(aw2.y));
    return r;
}

// ------------------------------------------------- packed fp32 pairs (f32x2)
// One instruction operates on two fp32 lanes held in a register pair; each
// lane is rounded exactly like the scalar instruction (round to nearest even).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n.reg .b64 ra, rb, rc, rd;\nmov.b64 ra, {%2,%3};\nmov.b64 rb, {%4,%5};\n"
        "mov.b64 rc, {%6,%7};\nfma.rn.f32x2 rd, ra, rb, rc;\nmov.b64 {%0,%1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n.reg .b64 ra, rb, rd;\nmov.b64 ra, {%2,%3};\nmov.b64 rb, {%4,%5};\n"
        "add.rn.f32x2 rd, ra, rb;\nmov.b64 {%0,%1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n.reg .b64 ra, rb, rd;\nmov.b64 ra, {%2,%3};\nmov.b64 rb, {%4,%5};\n"
        "mul.rn.f32x2 rd, ra, rb;\nmov.b64 {%0,%1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n.reg .b64 ra, rb, rd;\nmov.b64 ra, {%2,%3};\nmov.b64 rb, {%4,%5};\n"
        "sub.rn.f32x2 rd, ra, rb;\nmov.b64 {%0,%1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ------------------------------------------- 2^x on the FMA pipe (two lanes)
// The SFU computes 16 ex2 per SM clock, which caps a scan that needs one
// decay per state and step; part of the decays are therefore computed on the
// FMA pipe instead.  Method (Cody and Waite's argument reduction followed by
// a polynomial, as in Muller, "Elementary Functions", ch. 11):
//   x is clamped to [-125, 127] (below, 2^x is < 2^-125: the SFU result would
//   be flushed to zero and either is negligible against the input term; above,
//   fp32 would overflow);
//   r = round(x) by adding and subtracting 1.5 * 2^23, which rounds to an
//   integer in fp32; f = x - r, exact, in [-1/2, 1/2];
//   2^f = 1 + f (c1 + f (c2 + f (c3 + f (c4 + f c5)))), a degree-5 polynomial
//   fitted here to 2^f on [-1/2, 1/2] (Lawson-weighted least squares on 4000
//   Chebyshev nodes, relative error; constant term 1 exactly, so x = 0 gives
//   exactly 1); relative error 1.1e-7, 1.6e-7 with fp32 Horner evaluation,
//   against ~2^-22.5 for ex2.approx;
//   2^r is inserted into the exponent field: the low bits of t = x + 1.5 2^23
//   hold r, so bits(2^f) + (bits(t) << 23) is the result (exponent 126 or 127
//   of 2^f plus r in [-125, 127] stays a normal number).
#define SSM_EXP2_C {0.6931470036506653f, 0.24022242426872253f, 0.05550733581185341f, \
                    0.009671512991189957f, 0.001326472731307149f}

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float c[5] = SSM_EXP2_C;
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    x.x = fminf(fmaxf(x.x, -125.f), 127.f);
    x.y = fminf(fmaxf(x.y, -125.f), 127.f);
    const float2 t = add2(x, make_float2(kRound, kRound));
    const float2 f = sub2(x, sub2(t, make_float2(kRound, kRound)));
    float2 p = make_float2(c[4], c[4]);
    p = fma2(p, f, make_float2(c[3], c[3]));
    p = fma2(p, f, make_float2(c[2], c[2]));
    p = fma2(p, f, make_float2(c[1], c[1]));
    p = fma2(p, f, make_float2(c[0], c[0]));
    p = fma2(p, f, make_float2(1.f, 1.f));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// Pairs of states whose decays use exp2_poly2 instead of the SFU: pair p of a
// lane's states does when (p mod 4) < SSM_POLY_PAIRS, i.e. SSM_POLY_PAIRS / 4
// of the decays (for lanes holding at least 8 states).  Off by default: on
// B200 the one-lane scan at the 1.4B-layer shape measured 156.6 Gelem/s with
// every decay on the SFU, 126.9 with a quarter and 111.7 with half of them on
// the polynomial -- with ~1.75 warps per scheduler the kernel is bound by
// the latency of each warp's instruction stream, not by SFU throughput, and
// the polynomial lengthens that stream.
#ifndef SSM_POLY_PAIRS
#define SSM_POLY_PAIRS 0
#endif
// The same share for the first pass of the sequence split (segment
// aggregates, no readout), which keeps the SFU ~91 % busy: bound by its
// throughput rather than by latency.  A quarter by default: one call at
// L = 1,048,576, dim 1536 measured 15.35 ms with a quarter of that pass's
// decays on the polynomial, 15.53 ms with none and 18.55 ms with half.
#ifndef SSM_SEGAGG_POLY_PAIRS
#define SSM_SEGAGG_POLY_PAIRS 1
#endif
template <int POLY>
__device__ __forceinline__ constexpr bool poly_pair(int p) { return (p & 3) < POLY; }

template <bool PRECISE>
__device__ __forceinline__ float scale_A(float a) {
    return PRECISE ? a : a * kLog2e;
}

// The G lanes that share one channel: lanes base + i STRIDE, i < G, of the
// warp (STRIDE 1: G consecutive lanes; STRIDE 8 with G = 4: lanes c, c + 8,
// c + 16, c + 24, so that the 8 lanes of a quarter-warp belong to 8 channels
// and read the same shared-memory address when they load B or C -- two L1
// wavefronts per 128-bit load instead of four).
template <int G, int STRIDE>
struct LaneGroup {
    static_assert(STRIDE == 1 || STRIDE * G == 32, "consecutive lanes, or a group spread over the warp");
    static __device__ __forceinline__ unsigned base() {
        const unsigned lane = threadIdx.x & 31u;
        return STRIDE == 1 ? (lane & ~(unsigned)(G - 1)) : (lane % STRIDE);
    }
    static __device__ __forceinline__ unsigned mask() {
        unsigned m = 0;
#pragma unroll
        for (int i = 0; i < G; ++i) m |= 1u << (i * STRIDE);
        return G == 32 ? 0xffffffffu : (m << base());
    }
};

// Sum of a value over the G lanes that share one channel.
template <int G, int STRIDE = 1>
__device__ __forceinline__ float group_sum(float v) {
    if (G > 1) {
        const unsigned mask = LaneGroup<G, STRIDE>::mask();
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o * STRIDE);
    }
    return v;
}

// Fast-tier softplus of two values at once (log1p polynomial on fp32 pairs).
__device__ __forceinline__ float2 softplus2_fast(float2 s) {
    constexpr float q[9] = SSM_LOG1P_Q;
    const float2 e = make_float2(ex2_approx(-fabsf(s.x) * kLog2e), ex2_approx(-fabsf(s.y) * kLog2e));
    float2 p = make_float2(q[8], q[8]);
#pragma unroll
    for (int k = 7; k >= 0; --k) p = fma2(p, e, make_float2(q[k], q[k]));
    return add2(make_float2(fmaxf(s.x, 0.f), fmaxf(s.y, 0.f)), mul2(p, e));
}

// Exact zero-order hold on B: Bbar = (exp(z) - 1) / z * Delta B with
// z = Delta A, i.e. phi(z) = expm1(z) / z multiplies the Euler input term.
// Near z = 0 the quotient cancels, so |z| < 1/16 uses the Taylor series of
// phi to z^4 (remainder < z^5 / 720 < 1.4e-9); elsewhere (a - 1) * (1/A) * (1/Delta)
// with a = exp(z) already computed for the decay.  Two lanes at once.
__device__ __forceinline__ float2 zoh_phi2(float2 z, float2 a, float2 inv_a, float2 inv_dl) {
    float2 s = make_float2(1.f / 120.f, 1.f / 120.f);
    s = fma2(s, z, make_float2(1.f / 24.f, 1.f / 24.f));
    s = fma2(s, z, make_float2(1.f / 6.f, 1.f / 6.f));
    s = fma2(s, z, make_float2(0.5f, 0.5f));
    s = fma2(s, z, make_float2(1.f, 1.f));
    const float2 d = mul2(mul2(add2(a, make_float2(-1.f, -1.f)), inv_a), inv_dl);
    return make_float2(fabsf(z.x) < 0.0625f ? s.x : d.x, fabsf(z.y) < 0.0625f ? s.y : d.y);
}
__device__ __forceinline__ float zoh_phi_precise(float z) { return z == 0.f ? 1.f : expm1f(z) / z; }

template <int G, int STRIDE = 1>
__device__ __forceinline__ double group_sum_d(double v) {
    if (G > 1) {
        const unsigned mask = LaneGroup<G, STRIDE>::mask();
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o * STRIDE);
    }
    return v;
}

// Lane q of a group of G consecutive lanes holds the scalars of steps
// q, q + G, q + 2G, ... (own[j] is step j G + q); afterwards every lane of
// the group holds all K steps.
template <int K, int G, int STRIDE = 1>
__device__ __forceinline__ void exchange_steps(const float (&dlo)[K / G], const float (&duo)[K / G],
                                               float (&dl)[K], float (&du)[K]) {
    if (G == 1) {
#pragma unroll
        for (int k = 0; k < K; ++k) { dl[k] = dlo[k]; du[k] = duo[k]; }
        return;
    }
    const unsigned base = LaneGroup<G, STRIDE>::base(), mask = LaneGroup<G, STRIDE>::mask();
#pragma unroll
    for (int k = 0; k < K; ++k) {
        dl[k] = __shfl_sync(mask, dlo[k / G], base + (k % G) * STRIDE);
        du[k] = __shfl_sync(mask, duo[k / G], base + (k % G) * STRIDE);
    }
}

// Each lane holds partial sums y[k] for K steps; afterwards lane q of the
// group holds the full sums of its own steps, yo[j] = sum over the group of
// y[j G + q] (a butterfly reduce-scatter: log2 G rounds, each halving the
// steps a lane keeps).
template <int K, int G, int STRIDE = 1>
__device__ __forceinline__ void reduce_scatter_steps(const float (&y)[K], float (&yo)[K / G], int q) {
    if (G == 1) {
#pragma unroll
        for (int k = 0; k < K; ++k) yo[k] = y[k];
        return;
    }
    const unsigned mask = LaneGroup<G, STRIDE>::mask();
#pragma unroll
    for (int j = 0; j < K / G; ++j) {
        if (G == 2) {
            const float keep = q ? y[2 * j + 1] : y[2 * j];
            const float send = q ? y[2 * j] : y[2 * j + 1];
            yo[j] = keep + __shfl_xor_sync(mask, send, STRIDE);
        } else if (G > 4) {
            // log2 G butterfly rounds on the group's G values of block j:
            // in the round of distance o a lane keeps the half of its values
            // selected by bit o of q and adds its partner's copy of that half
            float v[G];
#pragma unroll
            for (int i = 0; i < G; ++i) v[i] = y[G * j + i];
#pragma unroll
            for (int o = G / 2, n = G; o >= 1; o >>= 1, n >>= 1) {
                const bool hi = (q & o) != 0;
#pragma unroll
                for (int i = 0; i < n / 2; ++i) {
                    const float keep = hi ? v[n / 2 + i] : v[i];
                    const float send = hi ? v[i] : v[n / 2 + i];
                    v[i] = keep + __shfl_xor_sync(mask, send, o * STRIDE);
                }
            }
            yo[j] = v[0];
        } else {  // G == 4
            const bool hi = (q & 2) != 0;
            const float k0 = hi ? y[4 * j + 2] : y[4 * j + 0], k1 = hi ? y[4 * j + 3] : y[4 * j + 1];
            const float s0 = hi ? y[4 * j + 0] : y[4 * j + 2], s1 = hi ? y[4 * j + 1] : y[4 * j + 3];
            const float m0 = k0 + __shfl_xor_sync(mask, s0, 2 * STRIDE);
            const float m1 = k1 + __shfl_xor_sync(mask, s1, 2 * STRIDE);
            const bool odd = (q & 1) != 0;
            yo[j] = (odd ? m1 : m0) + __shfl_xor_sync(mask, odd ? m0 : m1, STRIDE);
        }
    }
}

}  // namespace ssm
