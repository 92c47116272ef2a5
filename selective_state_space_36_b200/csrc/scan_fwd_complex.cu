// scan_fwd_complex.cu -- selective-scan forward with a complex diagonal A.
//
// The complex parameterisation the Mamba notes single out for audio
// (【論文要約】Mamba notes, Figure 10 and Table 8), read as the real recurrence
// (NL-345 Mamba translation, section 2, eq. (2)) carried out in complex
// numbers; Delta, u, z, D and the output stay real:
//     Abar_n = exp(Delta A_n) = e^{Delta Re A_n} (cos(Delta Im A_n) + i sin(Delta Im A_n))
//     h_n   <- Abar_n h_n + Delta B_n u          (complex state)
//     y      = Re(sum_n C_n h_n) + D u,   out = y * silu(z)
// Complex arrays are (re, im) pairs: A (dim, N, 2) and the state
// (batch, dim, N, 2) in fp32, B and C (batch, L, N, 2) in the I/O type.
//
// Layout as the generic real kernel: G = 4 lanes share a channel, lane q
// holding complex states [q NS, q NS + NS); a block of 128 threads covers 32
// channels of one batch row; B and C of a chunk of 32 steps are widened to
// fp32 pairs in shared memory.  Per state and step the decay takes one
// exponential (SFU in the fast tier) and the accurate sincosf in both tiers:
// the SFU sine's absolute error (~5e-7) would be a relative phase error of up
// to 5e-4 per step at the small angles Delta Im A of small Delta, and the
// phase error of a state adds up over its memory of up to ~1/(Delta |Re A|)
// steps.
#include "scan_kernels.cuh"

namespace ssm {

namespace {

constexpr int kCG = 4;                 // lanes per channel
constexpr int kCCPB = kBlock / kCG;    // channels per block
constexpr int kCChunk = 32;            // steps of B, C staged at once


template <typename IO, int NS, bool PRECISE>
__global__ void __launch_bounds__(kBlock)
scan_fwd_complex_kernel(const ScanArgs args) {
    using io = io_traits<IO>;
    constexpr int G = kCG, NSP = NS * G;
    __shared__ __align__(16) float2 sB[kCChunk][NSP];
    __shared__ __align__(16) float2 sC[kCChunk][NSP];

    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x, q = tid % G, ch = tid / G;
    const int64_t tiles = (Dm + kCCPB - 1) / kCCPB;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d = (blockIdx.x % tiles) * kCCPB + ch;
    const bool active = d < Dm;

    float are[NS], aim[NS], hr[NS], hi[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = q * NS + i;
        const bool ok = active && n < N;
        are[i] = ok ? scale_A<PRECISE>(args.A[2 * (d * N + n)]) : 0.f;
        aim[i] = ok ? args.A[2 * (d * N + n) + 1] : 0.f;
        const bool h0 = ok && args.last_state;
        hr[i] = h0 ? args.last_state[2 * ((b * Dm + d) * N + n)] : 0.f;
        hi[i] = h0 ? args.last_state[2 * ((b * Dm + d) * N + n) + 1] : 0.f;
    }
    const float bias = (active && args.bias) ? args.bias[d] : 0.f;
    const float dskip = (active && args.Dskip) ? args.Dskip[d] : 0.f;
    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);
    IO *po = static_cast<IO *>(args.out);

    for (int64_t tc = 0; tc < L; tc += kCChunk) {
        const int rows = (int)(L - tc < kCChunk ? L - tc : kCChunk);
        __syncthreads();
        for (int idx = tid; idx < kCChunk * NSP; idx += kBlock) {
            const int r = idx / NSP, n = idx % NSP;
            float2 vb = make_float2(0.f, 0.f), vc = vb;
            if (r < rows && n < N) {
                const int64_t o = 2 * ((b * L + tc + r) * N + n);
                vb = make_float2(io::load(pB + o), io::load(pB + o + 1));
                vc = make_float2(io::load(pC + o), io::load(pC + o + 1));
            }
            sB[r][n] = vb;
            sC[r][n] = vc;
        }
        __syncthreads();
        if (!active) continue;
        int64_t off = (b * L + tc) * Dm + d;
        for (int r = 0; r < rows; ++r, off += Dm) {
            const float uv = io::load_stream(pu + off);
            const float s = io::load_stream(pd + off) + bias;
            const float dl = args.softplus ? softplus<PRECISE>(s) : s;
            const float du = dl * uv;
            float yp = 0.f;
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const float2 bv = sB[r][q * NS + i], cv = sC[r][q * NS + i];
                const float e = decay<PRECISE>(dl, are[i]);
                float sn, cs;
                sincosf(dl * aim[i], &sn, &cs);
                const float ar = e * cs, ai = e * sn;
                const float nr = fmaf(ar, hr[i], fmaf(-ai, hi[i], du * bv.x));
                const float ni = fmaf(ar, hi[i], fmaf(ai, hr[i], du * bv.y));
                hr[i] = nr;
                hi[i] = ni;
                yp = fmaf(cv.x, nr, fmaf(-cv.y, ni, yp));
            }
            float y = group_sum<G>(yp);
            if (q == 0) {
                y = fmaf(dskip, uv, y);
                if (pz) y *= silu<PRECISE>(io::load_stream(pz + off));
                io::store(po + off, y);
            }
        }
    }
    if (!active || !args.last_state) return;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = q * NS + i;
        if (n < N) {
            args.last_state[2 * ((b * Dm + d) * N + n)] = hr[i];
            args.last_state[2 * ((b * Dm + d) * N + n) + 1] = hi[i];
        }
    }
}

template <typename IO, int NS>
cudaError_t launch_ns(const ScanArgs &a, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    const int64_t tiles = (a.dim + kCCPB - 1) / kCCPB;
    scan_fwd_complex_kernel<IO, NS, P><<<dim3((unsigned)(a.batch * tiles)), kBlock, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int64_t scan_complex_channels_per_block() { return kCCPB; }

cudaError_t launch_scan_complex(const ScanArgs &a, bool bf16, cudaStream_t st) {
    const int ns = a.dstate <= 16 ? 4 : (a.dstate <= 32 ? 8 : 16);
    if (bf16) {
        if (ns == 4) return launch_ns<__nv_bfloat16, 4>(a, st);
        if (ns == 8) return launch_ns<__nv_bfloat16, 8>(a, st);
        return launch_ns<__nv_bfloat16, 16>(a, st);
    }
    if (ns == 4) return launch_ns<float, 4>(a, st);
    if (ns == 8) return launch_ns<float, 8>(a, st);
    return launch_ns<float, 16>(a, st);
}

}  // namespace ssm
