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
    static __device__ __forceinline__ void store(float *p, float v) { __stcs(p, v); }
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
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        __stcs(reinterpret_cast<unsigned short *>(p), *reinterpret_cast<unsigned short *>(&b));
    }
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

// ------------------------------------------------------------------ softplus
// softplus(s) = log(1 + e^s) = max(s, 0) + log1p(e), e = exp(-|s|) in (0, 1].
template <bool PRECISE>
__device__ __forceinline__ float softplus(float s) {
    if (PRECISE) return fmaxf(s, 0.f) + log1pf(expf(-fabsf(s)));
    const float e = ex2_approx(-fabsf(s) * kLog2e);
    // Small e: alternating Taylor series of log1p truncated after e^7; the
    // remainder is below e^8 / 8, i.e. < 7e-8 relative for e < 1/8.
    float p = 1.f / 7.f;
    p = fmaf(p, e, -1.f / 6.f);
    p = fmaf(p, e, 1.f / 5.f);
    p = fmaf(p, e, -1.f / 4.f);
    p = fmaf(p, e, 1.f / 3.f);
    p = fmaf(p, e, -1.f / 2.f);
    p = fmaf(p, e, 1.f);
    const float series = p * e;
    // Larger e: 1 + e >= 1.125, where the SFU logarithm's absolute error is
    // small relative to the result.
    const float direct = lg2_approx(1.f + e) * kLn2;
    return fmaxf(s, 0.f) + (e < 0.125f ? series : direct);
}

// -------------------------------------------------------------------- silu
template <bool PRECISE>
__device__ __forceinline__ float silu(float z) {
    if (PRECISE) return z / (1.f + expf(-z));
    return z * rcp_approx(1.f + ex2_approx(-z * kLog2e));
}

// Decay Abar = exp(Delta * A).  The fast tier takes A pre-multiplied by log2(e).
template <bool PRECISE>
__device__ __forceinline__ float decay(float dl, float a_scaled) {
    if (PRECISE) return expf(dl * a_scaled);
    return ex2_approx(dl * a_scaled);
}

template <bool PRECISE>
__device__ __forceinline__ float scale_A(float a) {
    return PRECISE ? a : a * kLog2e;
}

// Sum of a value over the G consecutive lanes that share one channel.
template <int G>
__device__ __forceinline__ float group_sum(float v) {
    if (G > 1) {
        const unsigned lane = threadIdx.x & 31u;
        const unsigned mask = ((G == 32) ? 0xffffffffu : ((1u << G) - 1u)) << (lane & ~(unsigned)(G - 1));
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o);
    }
    return v;
}

}  // namespace ssm
