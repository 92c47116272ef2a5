// state_update.cu -- one recurrent (decode) step of the selective SSM.
//
// Recurrent mode takes constant time and memory per generated token (NL-345
// Mamba translation, section 1 "Fast training and inference"; section 2,
// eq. (2) for one t).  For each channel (b, d):
//     h_n <- exp(dt A_n) h_n + dt B_n x;   y = sum_n C_n h_n + D x;
//     out = y * silu(z)
// dt is the time step itself (already positive).  The step is bound by the
// state's HBM traffic (read and write N fp32 values per channel), so the
// layout is chosen for coalescing: G lanes share one channel and each lane
// moves NS consecutive fp32 state values with 128-bit accesses, so one warp
// instruction touches one contiguous span of 32 * 16 bytes.
#include "scan_kernels.cuh"

namespace ssm {

template <typename IO, int NS, int G, bool PRECISE, bool VEC>
__global__ void __launch_bounds__(kBlock)
state_update_kernel(const DecodeArgs args) {
    using io = io_traits<IO>;
    constexpr int CPB = kBlock / G;
    const int64_t Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x;
    const int q = tid % G;
    const int64_t tiles = (Dm + CPB - 1) / CPB;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d = (blockIdx.x % tiles) * CPB + tid / G;
    if (d >= Dm) return;  // whole groups leave together

    const int64_t bd = b * Dm + d;
    float *hp = args.state + bd * N + q * NS;
    float h[NS];
    if (VEC) {
#pragma unroll
        for (int i = 0; i < NS; i += 4) {
            const float4 v = __ldcs(reinterpret_cast<const float4 *>(hp + i));
            h[i] = v.x; h[i + 1] = v.y; h[i + 2] = v.z; h[i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NS; ++i) h[i] = (q * NS + i < N) ? __ldcs(hp + i) : 0.f;
    }
    const IO *px = static_cast<const IO *>(args.x);
    const IO *pB = static_cast<const IO *>(args.B) + b * N;
    const IO *pC = static_cast<const IO *>(args.C) + b * N;
    const float xv = io::load_stream(px + bd);
    const float dl = io::load_stream(static_cast<const IO *>(args.dt) + bd);
    const float dx = dl * xv;
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = q * NS + i;
        if (VEC || n < N) {
            const float a = decay<PRECISE>(dl, scale_A<PRECISE>(__ldg(args.A + d * N + n)));
            h[i] = fmaf(a, h[i], dx * io::load(pB + n));
            if (i & 1) y1 = fmaf(io::load(pC + n), h[i], y1);
            else y0 = fmaf(io::load(pC + n), h[i], y0);
        }
    }
    float y = group_sum<G>(y0 + y1);
    if (q == 0) {
        if (args.Dskip) y = fmaf(__ldg(args.Dskip + d), xv, y);
        if (args.z) y *= silu<PRECISE>(io::load_stream(static_cast<const IO *>(args.z) + bd));
        io::store(static_cast<IO *>(args.out) + bd, y);
    }
    if (VEC) {
#pragma unroll
        for (int i = 0; i < NS; i += 4)
            __stcs(reinterpret_cast<float4 *>(hp + i), make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]));
    } else {
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (q * NS + i < N) __stcs(hp + i, h[i]);
    }
}

template <typename IO, int NS, int G>
static cudaError_t launch_t(const DecodeArgs &a, bool vec, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    constexpr int CPB = kBlock / G;
    const int64_t tiles = (a.dim + CPB - 1) / CPB;
    const dim3 grid((unsigned)(a.batch * tiles));
    if (vec) state_update_kernel<IO, NS, G, P, true><<<grid, kBlock, 0, st>>>(a);
    else state_update_kernel<IO, NS, G, P, false><<<grid, kBlock, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename IO>
static cudaError_t launch_io(const DecodeArgs &a, int ns, int g, bool vec, cudaStream_t st) {
    if (ns == 4 && g == 1) return launch_t<IO, 4, 1>(a, vec, st);
    if (ns == 4 && g == 2) return launch_t<IO, 4, 2>(a, vec, st);
    if (ns == 4 && g == 4) return launch_t<IO, 4, 4>(a, vec, st);
    if (ns == 4 && g == 8) return launch_t<IO, 4, 8>(a, vec, st);
    if (ns == 4 && g == 16) return launch_t<IO, 4, 16>(a, vec, st);
    return cudaErrorInvalidConfiguration;
}

cudaError_t launch_state_update(const DecodeArgs &a, bool bf16, int ns, int g, cudaStream_t st) {
    // 128-bit state accesses need every lane's slice complete and 16-byte aligned
    const bool vec = (a.dstate % 4 == 0) && ((uintptr_t)a.state % 16 == 0) && (ns * g == a.dstate);
    return bf16 ? launch_io<__nv_bfloat16>(a, ns, g, vec, st) : launch_io<float>(a, ns, g, vec, st);
}

}  // namespace ssm
