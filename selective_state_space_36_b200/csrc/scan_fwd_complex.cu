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
#include <atomic>

#include "cp_async.cuh"
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

// ---------------------------------------------------------------------------
// Staged kernel for the common case (bf16 I/O, N = 16, rows of 16-byte
// multiples): the same four-lane layout with every input brought through
// shared memory, as in the real staged scan.  Chunks of T = 48 steps of the
// (batch row, 32-channel) tile move by cp.async two stages deep (u, delta,
// z tiles and the raw B, C rows); B and C are widened once per chunk to fp32
// pairs, C with its imaginary part negated so that Re(C h) is one f32x2 FMA.
// Per block of K steps (16) lane q computes Delta, Delta u of steps 4 j + q
// (softplus on pairs) and the values go to the other lanes by shuffles; each
// lane then runs its 4 complex states over the K steps, and the per-step partial
// readouts are reduce-scattered back to the owning lanes, which finish out and
// write it over the consumed u row of the tile; the chunk's out leaves in
// 16-byte stores.
#ifndef SSM_COMPLEX_LANES
#define SSM_COMPLEX_LANES 4
#endif
// Steps per block (Delta and Delta u of the block's steps computed by their
// owning lanes and shuffled to the group): at the 130M shape 16-step blocks
// measured 55.0 Gelem/s against 51.0 with 8 (32 steps spill registers).
#ifndef SSM_COMPLEX_KSTEP
#define SSM_COMPLEX_KSTEP 16
#endif
// Chunks of 48 steps in two stages (48 KB of shared memory per block) measured
// 55.6-55.7 Gelem/s against 54.7-54.9 for 32 steps in three.
#ifndef SSM_COMPLEX_CHUNK
#define SSM_COMPLEX_CHUNK 48
#endif
#ifndef SSM_COMPLEX_STAGES
#define SSM_COMPLEX_STAGES 2
#endif
template <int GL>  // lanes per channel: 4 (4 complex states each) or 8 (2 each)
struct CxLayout {
    static constexpr int G = GL, NS = 16 / GL, NSP = 16, CPB = kBlock / G;
    static constexpr int T = SSM_COMPLEX_CHUNK, K = SSM_COMPLEX_KSTEP, KG = K / G, S = SSM_COMPLEX_STAGES;
    static constexpr int LS = 32 / G;                       // lane stride of a channel's group
    static constexpr int MIN_BLOCKS = G == 8 ? 6 : 4;
    static constexpr int ROW = CPB + 8;                     // bf16 tile row, padded by 16 bytes
    static constexpr int TILE = T * ROW;                    // elements
    static constexpr int RAW = T * NSP * 2;                 // raw B or C chunk (elements)
    static constexpr size_t STAGE_BYTES = (3 * (size_t)TILE + 2 * RAW) * 2;
    static constexpr size_t W_BYTES = 2 * (size_t)T * NSP * sizeof(float2);  // widened B, C
    static constexpr size_t SMEM = S * STAGE_BYTES + W_BYTES;
};

template <int GL>
__global__ void __launch_bounds__(kBlock, CxLayout<GL>::MIN_BLOCKS)
scan_fwd_complex_staged_kernel(const ScanArgs args) {
    using io = io_traits<__nv_bfloat16>;
    using Lay = CxLayout<GL>;
    constexpr int G = Lay::G, NS = Lay::NS, NSP = Lay::NSP, CPB = Lay::CPB;
    constexpr int T = Lay::T, K = Lay::K, KG = Lay::KG, S = Lay::S, ROW = Lay::ROW, TILE = Lay::TILE;
    constexpr int EPV = 8;             // bf16 elements per 16-byte piece
    constexpr int ROWV = CPB / EPV;    // pieces per tile row
    extern __shared__ __align__(16) unsigned char smem[];
    float2 *wB = reinterpret_cast<float2 *>(smem + S * Lay::STAGE_BYTES);  // [T][NSP]
    float2 *wC = wB + T * NSP;                                              // [T][NSP], (re, -im)

    const int64_t L = args.seqlen, Dm = args.dim;
    // lane c + LS q of warp w: complex states [NS q, NS q + NS) of channel
    // LS w + c (a quarter-warp's 8 lanes read at most two B/C addresses)
    constexpr int LS = Lay::LS;
    const int tid = threadIdx.x, q = (tid & 31) / LS, grp = (tid >> 5) * LS + (tid & (LS - 1));
    const int64_t tiles = (Dm + CPB - 1) / CPB;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d0 = (blockIdx.x % tiles) * CPB;
    const int64_t d = d0 + grp;
    const bool active = d < Dm;
    const int nchunks = (int)((L + T - 1) / T);
    using bf = __nv_bfloat16;
    const bf *pu = static_cast<const bf *>(args.u);
    const bf *pd = static_cast<const bf *>(args.delta);
    const bf *pz = static_cast<const bf *>(args.z);
    const bf *pB = static_cast<const bf *>(args.B);
    const bf *pC = static_cast<const bf *>(args.C);
    bf *po = static_cast<bf *>(args.out);

    auto stage_ptr = [&](int s) { return reinterpret_cast<bf *>(smem + s * Lay::STAGE_BYTES); };
    auto issue = [&](int c) {  // chunk c into stage c % S
        const int64_t tc = (int64_t)c * T;
        const int rows = (int)(L - tc < T ? L - tc : T);
        bf *st = stage_ptr(c % S);
        bf *su = st, *sd = st + TILE, *sz = st + 2 * TILE, *rb = st + 3 * TILE, *rc = rb + Lay::RAW;
        for (int p = tid; p < T * ROWV; p += kBlock) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            const bool ok = r < rows && col < Dm;
            const int64_t go = ok ? (b * L + tc + r) * Dm + col : 0;
            const int so = r * ROW + v * EPV;
            cp_async16(su + so, pu + go, ok);
            cp_async16(sd + so, pd + go, ok);
            if (pz) cp_async16(sz + so, pz + go, ok);
        }
        const int pieces = rows * NSP * 2 / EPV;  // the chunk's B/C rows are contiguous
        const int64_t gbc = (b * L + tc) * NSP * 2;
        for (int p = tid; p < pieces; p += kBlock) {
            cp_async16(rb + p * EPV, pB + gbc + p * EPV, true);
            cp_async16(rc + p * EPV, pC + gbc + p * EPV, true);
        }
    };

    // per-lane constants: A of this lane's 4 states (Re scaled for the decay)
    float are[NS], aim[NS];
    float2 h2[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int64_t n = (int64_t)(d * NSP + q * NS + i);
        are[i] = active ? scale_A<false>(args.A[2 * n]) : 0.f;
        aim[i] = active ? args.A[2 * n + 1] : 0.f;
        const bool h0 = active && args.last_state;
        h2[i] = make_float2(h0 ? args.last_state[2 * (b * Dm * NSP + n)] : 0.f,
                            h0 ? args.last_state[2 * (b * Dm * NSP + n) + 1] : 0.f);
    }
    const float bias = (active && args.bias) ? args.bias[d] : 0.f;
    const float dskip = (active && args.Dskip) ? args.Dskip[d] : 0.f;

#pragma unroll
    for (int c = 0; c < S - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        cp_async_wait<S - 2>();
        // chunk c has landed for every thread, and every thread is done with
        // the stage that chunk c + S - 1 goes to and with the widened rows
        __syncthreads();
        if (c + S - 1 < nchunks) issue(c + S - 1);
        cp_async_commit();
        const int64_t tc = (int64_t)c * T;
        const int rows = (int)(L - tc < T ? L - tc : T);
        bf *st = stage_ptr(c % S);
        {
            const bf *rb = st + 3 * TILE, *rc = rb + Lay::RAW;
            for (int i = 4 * tid; i < T * NSP * 2; i += 4 * kBlock) {  // 2 complex values per thread and pass
                float v[4], w[4];
                const bool ok = i / (NSP * 2) < rows;
                io::load4_smem(rb + i, v);
                io::load4_smem(rc + i, w);
                float4 *db = reinterpret_cast<float4 *>(wB) + i / 4, *dc = reinterpret_cast<float4 *>(wC) + i / 4;
                *db = ok ? make_float4(v[0], v[1], v[2], v[3]) : make_float4(0.f, 0.f, 0.f, 0.f);
                *dc = ok ? make_float4(w[0], -w[1], w[2], -w[3]) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncthreads();
        bf *su = st + grp + q * ROW, *sd = st + TILE + grp + q * ROW, *sz = st + 2 * TILE + grp + q * ROW;
        const float4 *wBq = reinterpret_cast<const float4 *>(wB + q * NS);
        const float4 *wCq = reinterpret_cast<const float4 *>(wC + q * NS);

        auto block = [&](const int k0, const int nrows) {
            // the step scalars of the owned steps k0 + j G + q
            float uo[KG], zo[KG], dlo[KG], duo[KG];
            float so[KG];
#pragma unroll
            for (int j = 0; j < KG; ++j) {
                const int rr = k0 + j * G;
                uo[j] = io::load_smem(su + rr * ROW);
                so[j] = io::load_smem(sd + rr * ROW) + bias;
                zo[j] = pz ? io::load_smem(sz + rr * ROW) : 0.f;
            }
            if (args.softplus) {
                if constexpr (KG == 2) {
                    const float2 sp = softplus2_fast(make_float2(so[0], so[1]));
                    dlo[0] = sp.x;
                    dlo[1] = sp.y;
                } else {
#pragma unroll
                    for (int j = 0; j < KG; ++j) dlo[j] = softplus<false>(so[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < KG; ++j) dlo[j] = so[j];
            }
#pragma unroll
            for (int j = 0; j < KG; ++j) {
                if (k0 + j * G + q >= nrows || !active) dlo[j] = 0.f;
                duo[j] = dlo[j] * uo[j];
            }
            float dl[K], du[K];
            exchange_steps<K, G, LS>(dlo, duo, dl, du);
            float yp[K];
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int row = (k0 + k) * (NSP / 2);  // float4 index of the row (2 complex values each)
                const float2 du2 = make_float2(du[k], du[k]);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int i2 = 0; i2 < NS / 2; ++i2) {
                    const float4 b4 = wBq[row + i2], c4 = wCq[row + i2];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int i = 2 * i2 + e2;
                        const float2 bv = e2 ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y);
                        const float2 cv = e2 ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
                        const float e = ex2_approx(dl[k] * are[i]);
                        float sn, cs;
                        phase<false>(dl[k] * aim[i], sn, cs);
                        const float ec = e * cs, es = e * sn;
                        float2 t = fma2(make_float2(ec, ec), h2[i], mul2(du2, bv));
                        t.x = fmaf(-es, h2[i].y, t.x);
                        t.y = fmaf(es, h2[i].x, t.y);
                        h2[i] = t;
                        acc = fma2(cv, t, acc);  // (cr hr, -ci hi)
                    }
                }
                yp[k] = acc.x + acc.y;
            }
            float yo[KG];
            reduce_scatter_steps<K, G, LS>(yp, yo, q);
#pragma unroll
            for (int j = 0; j < KG; ++j) {
                const int rr = k0 + j * G;
                float y = fmaf(dskip, uo[j], yo[j]);
                if (pz) y *= silu<false>(zo[j]);
                io::store_smem(su + rr * ROW, y);  // out over the consumed u
            }
        };
        if (rows == T) {
#pragma unroll 1
            for (int k0 = 0; k0 < T; k0 += K) block(k0, T);
        } else {
            for (int k0 = 0; k0 < rows; k0 += K) block(k0, rows);
        }
        __syncthreads();
        // the chunk's out leaves in 16-byte pieces
        for (int p = tid; p < T * ROWV; p += kBlock) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            if (r < rows && col < Dm)
                __stcs(reinterpret_cast<uint4 *>(po + (b * L + tc + r) * Dm + col),
                       *reinterpret_cast<const uint4 *>(st + r * ROW + v * EPV));
        }
    }
    cp_async_wait<0>();
    if (!active || !args.last_state) return;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int64_t n = (int64_t)(d * NSP + q * NS + i);
        args.last_state[2 * (b * Dm * NSP + n)] = h2[i].x;
        args.last_state[2 * (b * Dm * NSP + n) + 1] = h2[i].y;
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

bool scan_complex_staged_eligible(const ScanArgs &a, bool bf16) {
    auto al = [](const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) % 16) == 0; };
    return bf16 && a.dstate == CxLayout<SSM_COMPLEX_LANES>::NSP && (a.dim * 2) % 16 == 0 && al(a.u) &&
           al(a.delta) && al(a.z) && al(a.B) && al(a.C) && al(a.out);
}

cudaError_t launch_scan_complex(const ScanArgs &a, bool bf16, cudaStream_t st) {
    if (scan_complex_staged_eligible(a, bf16)) {
        using Lay = CxLayout<SSM_COMPLEX_LANES>;
        auto kern = scan_fwd_complex_staged_kernel<SSM_COMPLEX_LANES>;
        static std::atomic<unsigned long long> configured{0};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const unsigned long long bit = 1ull << (dev & 63);
        if (!(configured.load(std::memory_order_relaxed) & bit)) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::SMEM);
            if (e != cudaSuccess) return e;
            configured.fetch_or(bit, std::memory_order_relaxed);
        }
        const int64_t tiles = (a.dim + Lay::CPB - 1) / Lay::CPB;
        kern<<<dim3((unsigned)(a.batch * tiles)), kBlock, Lay::SMEM, st>>>(a);
        return cudaGetLastError();
    }
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
