// state_update.cu -- one recurrent (decode) step of the selective SSM.
//
// Recurrent mode takes constant time and memory per generated token (NL-345
// Mamba translation, section 1 "Fast training and inference"; section 2,
// eq. (2) for one t).  For each channel (b, d):
//     h_n <- exp(dt A_n) h_n + dt B_n x;   y = sum_n C_n h_n + D x;
//     out = y * silu(z)
// dt is the time step itself (already positive).
//
// The step moves the state through memory (N fp32 values read and written per
// channel) and does little arithmetic, so it is laid out for memory-level
// parallelism: G lanes share a channel, each owning NS consecutive states (one
// 128-bit access when NS = 4, so a warp instruction covers 512 contiguous
// bytes), A, B and C arrive with one vector load each, and a thread handles
// kDecodeItems slices with their loads issued before any arithmetic.  One
// slice per thread measured best: it keeps the kernel at ~32 registers, i.e.
// full occupancy, and occupancy is what keeps enough requests in flight.  The
// state uses default caching (the next step re-reads it); the per-step inputs
// and the output are streamed.
#include "scan_kernels.cuh"

namespace ssm {

#ifndef SSM_DECODE_ITEMS
#define SSM_DECODE_ITEMS 1
#endif
constexpr int kDecodeItems = SSM_DECODE_ITEMS;

template <typename IO, int NS>
struct SliceIn {
    float h[NS], a[NS], b[NS], c[NS];
    float x, dt, z;
};

template <typename IO, int NS, int G, bool PRECISE, bool VEC>
__global__ void __launch_bounds__(kBlock)
state_update_kernel(const DecodeArgs args) {
    using io = io_traits<IO>;
    const int64_t Dm = args.dim;
    const int N = args.dstate;
    const int64_t total = args.batch * Dm * G;  // slices (b, d, q)
    const int64_t base = (int64_t)blockIdx.x * kBlock * kDecodeItems + threadIdx.x;
    const IO *px = static_cast<const IO *>(args.x);
    const IO *pdt = static_cast<const IO *>(args.dt);
    const IO *pz = static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);

    SliceIn<IO, NS> in[kDecodeItems];
    // ---- loads of every slice first
#pragma unroll
    for (int it = 0; it < kDecodeItems; ++it) {
        const int64_t s = base + (int64_t)it * kBlock;
        if (s >= total) continue;
        const int64_t bd = s / G;
        const int q = (int)(s % G);
        const int64_t b = bd / Dm, d = bd % Dm;
        const float *hp = args.state + bd * N + q * NS;
        const float *ap = args.A + d * N + q * NS;
        const IO *bp = pB + b * N + q * NS;
        const IO *cp = pC + b * N + q * NS;
        if (VEC) {
#pragma unroll
            for (int i = 0; i < NS; i += 4) {
                const float4 hv = *reinterpret_cast<const float4 *>(hp + i);
                const float4 av = __ldg(reinterpret_cast<const float4 *>(ap + i));
                in[it].h[i] = hv.x; in[it].h[i + 1] = hv.y; in[it].h[i + 2] = hv.z; in[it].h[i + 3] = hv.w;
                in[it].a[i] = av.x; in[it].a[i + 1] = av.y; in[it].a[i + 2] = av.z; in[it].a[i + 3] = av.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const bool ok = q * NS + i < N;
                in[it].h[i] = ok ? hp[i] : 0.f;
                in[it].a[i] = ok ? __ldg(ap + i) : 0.f;
            }
        }
        if (VEC) {
#pragma unroll
            for (int i = 0; i < NS; i += 4) {
                io::load4(bp + i, in[it].b + i);
                io::load4(cp + i, in[it].c + i);
            }
        } else {
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const bool ok = q * NS + i < N;
                in[it].b[i] = ok ? io::load(bp + i) : 0.f;
                in[it].c[i] = ok ? io::load(cp + i) : 0.f;
            }
        }
        in[it].x = io::load_stream(px + bd);
        in[it].dt = io::load_stream(pdt + bd);
        in[it].z = (pz && q == 0) ? io::load_stream(pz + bd) : 0.f;
    }
    // ---- arithmetic and stores
#pragma unroll
    for (int it = 0; it < kDecodeItems; ++it) {
        const int64_t s = base + (int64_t)it * kBlock;
        if (s >= total) continue;  // whole channel groups leave together (total is a multiple of G)
        const int64_t bd = s / G;
        const int q = (int)(s % G);
        const int64_t d = bd % Dm;
        const float dl = in[it].dt, dx = dl * in[it].x;
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const float a = decay<PRECISE>(dl, scale_A<PRECISE>(in[it].a[i]));
            in[it].h[i] = fmaf(a, in[it].h[i], dx * in[it].b[i]);
            if (i & 1) y1 = fmaf(in[it].c[i], in[it].h[i], y1);
            else y0 = fmaf(in[it].c[i], in[it].h[i], y0);
        }
        float y = group_sum<G>(y0 + y1);
        if (q == 0) {
            if (args.Dskip) y = fmaf(__ldg(args.Dskip + d), in[it].x, y);
            if (pz) y *= silu<PRECISE>(in[it].z);
            io::store(static_cast<IO *>(args.out) + bd, y);
        }
        float *hp = args.state + bd * N + q * NS;
        if (VEC) {
#pragma unroll
            for (int i = 0; i < NS; i += 4)
                *reinterpret_cast<float4 *>(hp + i) =
                    make_float4(in[it].h[i], in[it].h[i + 1], in[it].h[i + 2], in[it].h[i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < NS; ++i)
                if (q * NS + i < N) hp[i] = in[it].h[i];
        }
    }
}

template <typename IO, int NS, int G>
static cudaError_t launch_t(const DecodeArgs &a, bool vec, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    const int64_t total = a.batch * a.dim * G;
    const int64_t per_block = (int64_t)kBlock * kDecodeItems;
    const dim3 grid((unsigned)((total + per_block - 1) / per_block));
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
    // 128-bit state/A accesses need every lane's slice complete and 16-byte
    // aligned; the NS-element B/C rows then start on NS * sizeof(io) bytes.
    const size_t es = bf16 ? 2 : 4;
    auto al = [](const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; };
    const bool vec = (a.dstate % 4 == 0) && (ns * g == a.dstate) && al(a.state, 16) && al(a.A, 16) &&
                     al(a.B, 4 * es) && al(a.C, 4 * es);
    return bf16 ? launch_io<__nv_bfloat16>(a, ns, g, vec, st) : launch_io<float>(a, ns, g, vec, st);
}

}  // namespace ssm
