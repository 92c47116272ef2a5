// scan_fwd.cu -- selective-scan forward kernels for sm_100a.
//
// Computes, per channel (b, d) (NL-345 Mamba translation, section 2, eq. (2),
// "Discretization", "Structure and Dimensions"; 【論文要約】Mamba notes, S6
// Algorithm 2 and 数式解説 3):
//     Delta = softplus(delta + bias);  h_n <- exp(Delta A_n) h_n + Delta B_n u;
//     y = sum_n C_n h_n + D u;  out = y * silu(z)
// with the fp32 state held in registers for the whole sequence, so the
// expanded (batch, L, dim, N) state is never materialised (the notes'
// hardware-aware algorithm: parameters are read from HBM once, discretisation
// and recurrence happen on chip, and only the outputs go back to HBM).
//
// Thread layout: a group of G consecutive lanes owns one channel; lane q of
// the group holds states [q*NS, q*NS + NS).  A block of 128 threads covers
// 128/G channels of one batch row.  B_t and C_t (shared by all channels of a
// batch row) are staged per chunk of kChunk steps in shared memory as fp32 and
// read as broadcast 128-bit loads; u, delta, z are read straight from global
// memory, coalesced across the channels of a warp.
//
// Modes:
//  kFull     one pass over [0, L): h from last_state (or 0), writes out and
//            last_state.
//  kSegAgg   sequence split, first pass: segment s scanned from h = 0 without
//            readout; stores its local end state h_loc[b,s,d,:] and the segment's
//            Delta sum (so that the segment's decay product is exp(A * sum)).
//  kSegFinal second pass: the carry into segment s is the left fold of
//            (P_s', h_loc_s') over s' < s with the associative operator
//            (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2), the associative operator
//            behind the parallel scan the notes cite; then the segment is
//            re-scanned with readout.
#include "scan_common.cuh"

namespace ssm {

template <typename IO, int NS, int G, bool PRECISE, int MODE, bool ZOH>
__global__ void __launch_bounds__(kBlock)
scan_fwd_kernel(const ScanArgs args) {
    using io = io_traits<IO>;
    constexpr int NSP = NS * G;  // padded states per channel
    __shared__ __align__(16) float sB[kChunk][NSP];
    __shared__ __align__(16) float sC[kChunk][NSP];

    const LaneGeom<G> g(args);
    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x;
    const int seg = blockIdx.y;
    const int64_t t_begin = (int64_t)seg * args.seg_len;
    const int64_t t_end = t_begin + args.seg_len < L ? t_begin + args.seg_len : L;

    float Aw[NS], h[NS];
    lane_init<NS, PRECISE, MODE>(args, lane_ref(g), seg, Aw, h);
    const float bias = (g.active && args.bias) ? args.bias[g.d] : 0.f;
    const float dskip = (g.active && args.Dskip) ? args.Dskip[g.d] : 0.f;

    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);
    IO *po = static_cast<IO *>(args.out);
    double dsum = 0.0;

    for (int64_t tc = t_begin; tc < t_end; tc += kChunk) {
        const int rows = (int)(t_end - tc < kChunk ? t_end - tc : kChunk);
        __syncthreads();
        for (int idx = tid; idx < kChunk * NSP; idx += kBlock) {
            const int r = idx / NSP, n = idx % NSP;
            float vb = 0.f, vc = 0.f;
            if (r < rows && n < N) {
                const int64_t o = (g.b * L + tc + r) * N + n;
                vb = io::load(pB + o);
                vc = io::load(pC + o);
            }
            sB[r][n] = vb;
            sC[r][n] = vc;
        }
        __syncthreads();
        if (!g.active) continue;
        int64_t off = (g.b * L + tc) * Dm + g.d;
#pragma unroll 2
        for (int r = 0; r < rows; ++r, off += Dm) {
            const float uv = io::load_stream(pu + off);
            const float s = io::load_stream(pd + off) + bias;
            const float dl = args.softplus ? softplus<PRECISE>(s) : s;
            const float yl = lane_step<NS, PRECISE, ZOH>(dl, dl * uv, &sB[r][g.q * NS], &sC[r][g.q * NS], Aw, h);
            if (MODE == kSegAgg) {
                dsum += (double)dl;
            } else {
                float y = group_sum<G>(yl);
                if (g.q == 0) {
                    y = fmaf(dskip, uv, y);
                    if (pz) y *= silu<PRECISE>(io::load_stream(pz + off));
                    io::store(po + off, y);
                }
            }
        }
    }
    lane_finish<NS, MODE>(args, lane_ref(g), seg, t_end, h, dsum);
}

// ------------------------------------------------------------------ launchers
// The staged kernel copies 16-byte pieces: rows of u/delta/z tiles and of
// B/C must start on 16-byte boundaries.
bool staged_eligible(const ScanArgs &a, int es) {
    auto al = [](const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) % 16) == 0; };
    return (a.dim * es) % 16 == 0 && (a.dstate * es) % 16 == 0 && al(a.u) && al(a.delta) &&
           al(a.z) && al(a.B) && al(a.C) && al(a.out);
}
template <typename IO, int NS, int G, bool ZOH>
static cudaError_t launch_z(const ScanArgs &a, int variant, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    constexpr int CPB = kBlock / G;
    const int64_t tiles = (a.dim + CPB - 1) / CPB;
    const dim3 block(kBlock);
    if (variant == kVariantSlab) {
        scan_fwd_kernel<IO, NS, G, P, kFull, ZOH><<<dim3((unsigned)(a.batch * tiles), 1), block, 0, st>>>(a);
        return cudaGetLastError();
    }
    if (a.nseg > 1)
        scan_fwd_kernel<IO, NS, G, P, kSegAgg, ZOH>
            <<<dim3((unsigned)(a.batch * tiles), (unsigned)(a.nseg - 1)), block, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scan_fwd_kernel<IO, NS, G, P, kSegFinal, ZOH>
        <<<dim3((unsigned)(a.batch * tiles), (unsigned)a.nseg), block, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename IO, int NS, int G>
static cudaError_t launch_t(const ScanArgs &a, int variant, cudaStream_t st) {
    return a.zoh_b ? launch_z<IO, NS, G, true>(a, variant, st) : launch_z<IO, NS, G, false>(a, variant, st);
}

template <typename IO>
static cudaError_t launch_io(const ScanArgs &a, int ns, int g, int variant, cudaStream_t st) {
    if (ns == 4 && g == 1) return launch_t<IO, 4, 1>(a, variant, st);
    if (ns == 8 && g == 1) return launch_t<IO, 8, 1>(a, variant, st);
    if (ns == 16 && g == 1) return launch_t<IO, 16, 1>(a, variant, st);
    if (ns == 8 && g == 2) return launch_t<IO, 8, 2>(a, variant, st);
    if (ns == 4 && g == 4) return launch_t<IO, 4, 4>(a, variant, st);
    if (ns == 16 && g == 2) return launch_t<IO, 16, 2>(a, variant, st);
    if (ns == 8 && g == 4) return launch_t<IO, 8, 4>(a, variant, st);
    if (ns == 16 && g == 4) return launch_t<IO, 16, 4>(a, variant, st);
    return cudaErrorInvalidConfiguration;
}

cudaError_t launch_scan_fwd(const ScanArgs &a, bool bf16, int ns, int g, int cpl, int variant,
                            int family, cudaStream_t st) {
    const bool eligible = staged_eligible(a, bf16 ? 2 : 4);
    if (family == kFamilyStaged && !eligible) return cudaErrorInvalidValue;
    if (family != kFamilyGeneric && eligible) return launch_scan_staged(a, bf16, ns, g, cpl, variant, st);
    return bf16 ? launch_io<__nv_bfloat16>(a, ns, g, variant, st)
                : launch_io<float>(a, ns, g, variant, st);
}

bool scan_shape_supported(int ns, int g) {
    return (ns == 4 && g == 1) || (ns == 8 && g == 1) || (ns == 16 && g == 1) ||
           (ns == 8 && g == 2) || (ns == 4 && g == 4) || (ns == 16 && g == 2) ||
           (ns == 8 && g == 4) || (ns == 16 && g == 4);
}

}  // namespace ssm
