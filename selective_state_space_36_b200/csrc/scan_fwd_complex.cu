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
// fp32 pairs in shared memory; u, delta, z of kCAhead steps are loaded ahead
// of their arithmetic.  Per state and step the decay takes one exponential and a
// sine and cosine of Delta Im A.  The fp32 tier calls sincosf.  The fast tier
// reduces the angle to [-pi, pi] (round to nearest by the 1.5 2^23 addition,
// then Cody and Waite's two-part 2 pi) and takes the SFU's sine and cosine,
// whose absolute error (<= 2^-21.4 on [-pi, pi]) is a phase error of that
// size per step; over a state's memory of ~1/(Delta |Re A|) steps it stays
// far inside the bf16 tier's 1e-3 state bound.  The complex products run on
// fp32 pairs (f32x2): (re, im) of a state is one register pair.
#include "scan_kernels.cuh"

namespace ssm {

namespace {

constexpr int kCG = 4;                 // lanes per channel
constexpr int kCCPB = kBlock / kCG;    // channels per block
constexpr int kCChunk = 32;            // steps of B, C staged at once
// Steps whose u, delta, z are loaded together, ahead of their arithmetic:
// with 4 the loads' latency was exposed (ncu: long-scoreboard stalls 3.55 per
// issued instruction at the 130M layer).
#ifndef SSM_COMPLEX_AHEAD
#define SSM_COMPLEX_AHEAD 16
#endif
constexpr int kCAhead = SSM_COMPLEX_AHEAD;

constexpr float kInvTwoPi = 0.15915494309189535f;
constexpr float kTwoPiHi = 6.28125f;               // 9 significant bits: k * kTwoPiHi is exact
constexpr float kTwoPiLo = 1.9353071795864769e-3f;  // 2 pi - kTwoPiHi

template <bool PRECISE>
__device__ __forceinline__ void phase(float x, float &s, float &c) {
    if (PRECISE) {
        sincosf(x, &s, &c);
        return;
    }
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23: x * (1 / 2 pi) + kRound - kRound = rint(x / 2 pi)
    const float k = fmaf(x, kInvTwoPi, kRound) - kRound;
    const float r = fmaf(-k, kTwoPiLo, fmaf(-k, kTwoPiHi, x));
    __sincosf(r, &s, &c);
}

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
        const int64_t off0 = (b * L + tc) * Dm + d;
        // one step: row r of the chunk with its u, (delta + bias), z
        auto step = [&](int r, float uv, float s, float zv) {
            const float dl = args.softplus ? softplus<PRECISE>(s) : s;
            const float du = dl * uv;
            float yp;
            if (PRECISE) {
                yp = 0.f;
#pragma unroll
                for (int i = 0; i < NS; ++i) {
                    const float2 bv = sB[r][q * NS + i], cv = sC[r][q * NS + i];
                    const float e = decay<PRECISE>(dl, are[i]);
                    float sn, cs;
                    phase<PRECISE>(dl * aim[i], sn, cs);
                    const float ar = e * cs, ai = e * sn;
                    const float nr = fmaf(ar, hr[i], fmaf(-ai, hi[i], du * bv.x));
                    const float ni = fmaf(ar, hi[i], fmaf(ai, hr[i], du * bv.y));
                    hr[i] = nr;
                    hi[i] = ni;
                    yp = fmaf(cv.x, nr, fmaf(-cv.y, ni, yp));
                }
            } else {
                // states as (re, im) pairs: h <- (ar, ar) h + (-ai, ai) (im, re) + du (br, bi);
                // readout Re(C h) = cr hr - ci hi summed on a pair
                const float2 du2 = make_float2(du, du);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < NS; ++i) {
                    const float2 bv = sB[r][q * NS + i], cv = sC[r][q * NS + i];
                    const float e = ex2_approx(dl * are[i]);
                    float sn, cs;
                    phase<false>(dl * aim[i], sn, cs);
                    const float2 h2 = make_float2(hr[i], hi[i]);
                    float2 t = mul2(du2, bv);
                    t = fma2(make_float2(-e * sn, e * sn), make_float2(hi[i], hr[i]), t);
                    t = fma2(make_float2(e * cs, e * cs), h2, t);
                    hr[i] = t.x;
                    hi[i] = t.y;
                    acc = fma2(make_float2(cv.x, -cv.y), t, acc);
                }
                yp = acc.x + acc.y;
            }
            float y = group_sum<G>(yp);
            if (q == 0) {
                y = fmaf(dskip, uv, y);
                if (pz) y *= silu<PRECISE>(zv);
                io::store(po + off0 + (int64_t)r * Dm, y);
            }
        };
        int r = 0;
        for (; r + kCAhead <= rows; r += kCAhead) {
            float uv[kCAhead], sv[kCAhead], zv[kCAhead];
#pragma unroll
            for (int j = 0; j < kCAhead; ++j) {
                const int64_t o = off0 + (int64_t)(r + j) * Dm;
                uv[j] = io::load_stream(pu + o);
                sv[j] = io::load_stream(pd + o) + bias;
                zv[j] = (pz && q == 0) ? io::load_stream(pz + o) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kCAhead; ++j) step(r + j, uv[j], sv[j], zv[j]);
        }
        for (; r < rows; ++r) {
            const int64_t o = off0 + (int64_t)r * Dm;
            step(r, io::load_stream(pu + o), io::load_stream(pd + o) + bias,
                 (pz && q == 0) ? io::load_stream(pz + o) : 0.f);
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
