// scan_fwd_staged.cu -- selective-scan forward, staged variant (sm_100a).
//
// Same arithmetic and thread layout as the generic kernel in scan_fwd.cu
// (NL-345 Mamba translation, section 2 eq. (2); 【論文要約】Mamba notes, S6
// Algorithm 2, 数式解説 3), but every input reaches the compute loop through
// shared memory: each chunk of T time steps of the block's u, delta, z tiles
// ([T x channels-per-block]) and of B, C ([T x N]) is brought in with 16-byte
// cp.async copies, STAGES chunks ahead, so global-memory latency overlaps the
// recurrence of earlier chunks (the notes' hardware-aware algorithm: inputs go
// from HBM to on-chip memory once and only the outputs are written back).  B and C are widened to fp32 once per chunk
// and per block, then read by every channel with broadcast 128-bit loads.
//
// The waits are cp.async.wait_group (hardware-tracked completion of this
// thread's own copies) followed by a block barrier: there is no polling loop.
//
// Eligibility (checked on the host): dim * sizeof(io) and dstate * sizeof(io)
// are multiples of 16 bytes and u, delta, z, B, C start on 16-byte boundaries.
#include <atomic>

#include "scan_common.cuh"

namespace ssm {

#ifndef SSM_KSTEP
#define SSM_KSTEP 4
#endif
// Time steps processed together: a multiple of 2G (so each lane owns an even
// number of them) that divides the chunk.
template <int G>
struct KStep {
    static constexpr int value = SSM_KSTEP > 2 * G ? SSM_KSTEP : 2 * G;
};

template <typename IO>
struct StagedCfg {
    static constexpr int T = sizeof(IO) == 2 ? 32 : 16;  // time steps per chunk
    static constexpr int STAGES = 3;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool full) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = full ? 16 : 0;  // 0: no global read, destination zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <typename IO, int NS, int G>
struct StagedLayout {
    static constexpr int T = StagedCfg<IO>::T;
    static constexpr int S = StagedCfg<IO>::STAGES;
    static constexpr int CPB = kBlock / G;
    static constexpr int NSP = NS * G;
    static constexpr int TILE = T * CPB;  // elements of one u/delta/z tile
    static constexpr int RAW = T * NSP;   // elements reserved for one raw B or C tile
    static constexpr size_t STAGE_BYTES = (3 * TILE + 2 * RAW) * sizeof(IO);
    static constexpr size_t BC_BYTES = 2 * (size_t)T * NSP * sizeof(float);
    static constexpr size_t SMEM = S * STAGE_BYTES + BC_BYTES;
};

template <typename IO, int NS, int G, bool PRECISE, int MODE>
__global__ void __launch_bounds__(kBlock)
scan_fwd_staged_kernel(const ScanArgs args) {
    using io = io_traits<IO>;
    using Lay = StagedLayout<IO, NS, G>;
    constexpr int T = Lay::T, S = Lay::S, CPB = Lay::CPB, NSP = Lay::NSP;
    constexpr int EPV = 16 / sizeof(IO);  // elements per 16-byte piece
    constexpr int ROWV = CPB / EPV;       // pieces per tile row
    constexpr int KSTEP = KStep<G>::value;
    constexpr int KG = KSTEP / G;         // steps whose scalar work this lane does
    extern __shared__ __align__(16) unsigned char smem[];
    float *fB = reinterpret_cast<float *>(smem + S * Lay::STAGE_BYTES);
    float *fC = fB + T * NSP;

    const LaneGeom<G> g(args);
    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x;
    const int seg = blockIdx.y;
    const int64_t t_begin = (int64_t)seg * args.seg_len;
    const int64_t t_end = t_begin + args.seg_len < L ? t_begin + args.seg_len : L;
    const int64_t d0 = (blockIdx.x % ((Dm + CPB - 1) / CPB)) * CPB;

    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = MODE == kSegAgg ? nullptr : static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);
    IO *po = static_cast<IO *>(args.out);

    auto stage_ptr = [&](int s) { return reinterpret_cast<IO *>(smem + s * Lay::STAGE_BYTES); };
    const int nchunks = (int)((t_end - t_begin + T - 1) / T);

    // enqueue the copies of chunk c into stage c % S
    auto issue = [&](int c) {
        const int64_t tc = t_begin + (int64_t)c * T;
        const int rows = (int)(t_end - tc < T ? t_end - tc : T);
        IO *st = stage_ptr(c % S);
        IO *su = st, *sd = st + Lay::TILE, *sz = st + 2 * Lay::TILE;
        IO *rb = st + 3 * Lay::TILE, *rc = rb + Lay::RAW;
        for (int p = tid; p < T * ROWV; p += kBlock) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            const bool ok = r < rows && col < Dm;
            const int64_t go = ok ? (g.b * L + tc + r) * Dm + col : 0;
            const int so = r * CPB + v * EPV;
            cp_async16(su + so, pu + go, ok);
            cp_async16(sd + so, pd + go, ok);
            if (pz) cp_async16(sz + so, pz + go, ok);
        }
        const int pieces = rows * N / EPV;  // B/C rows of this chunk are contiguous
        const int64_t gbc = (g.b * L + tc) * N;
        for (int p = tid; p < pieces; p += kBlock) {
            cp_async16(rb + p * EPV, pB + gbc + p * EPV, true);
            cp_async16(rc + p * EPV, pC + gbc + p * EPV, true);
        }
    };

    float Aw[NS], h[NS];
    lane_init<NS, G, PRECISE, MODE>(args, g, seg, Aw, h);
    float2 A2[NS / 2], h2[NS / 2];
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
        A2[p] = make_float2(Aw[2 * p], Aw[2 * p + 1]);
        h2[p] = make_float2(h[2 * p], h[2 * p + 1]);
    }
    const float bias = (g.active && args.bias) ? args.bias[g.d] : 0.f;
    const float dskip = (g.active && args.Dskip) ? args.Dskip[g.d] : 0.f;
    double dsum = 0.0;

#pragma unroll
    for (int c = 0; c < S - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        if (c + S - 1 < nchunks) issue(c + S - 1);
        cp_async_commit();
        cp_async_wait<S - 1>();  // this thread's copies of chunk c have landed
        __syncthreads();         // ... and everyone else's
        const int64_t tc = t_begin + (int64_t)c * T;
        const int rows = (int)(t_end - tc < T ? t_end - tc : T);
        const IO *st = stage_ptr(c % S);
        const IO *rb = st + 3 * Lay::TILE, *rc = rb + Lay::RAW;
        for (int i = tid; i < T * NSP; i += kBlock) {
            const int r = i / NSP, n = i % NSP;
            const bool ok = r < rows && n < N;
            fB[i] = ok ? io::load_smem(rb + r * N + n) : 0.f;
            fC[i] = ok ? io::load_smem(rc + r * N + n) : 0.f;
        }
        __syncthreads();
        if (g.active) {
            const IO *su = st + g.ch, *sd = st + Lay::TILE + g.ch, *sz = st + 2 * Lay::TILE + g.ch;
            const int64_t off0 = (g.b * L + tc) * Dm + g.d;
            // KSTEP steps at a time.  The G lanes of a channel split its states;
            // the per-step scalar work (softplus, Delta u, skip, gate, store) of
            // step r0 + j G + q is done once, by lane q, and Delta, Delta u and
            // the partial readouts travel between the lanes by shuffles.  Rows
            // past the end of the sequence were zero-filled by the copy and get
            // Delta = 0 (decay 1, no input): the state passes through them.
            for (int r0 = 0; r0 < rows; r0 += KSTEP) {
                float uvo[KG], dlo[KG], duo[KG];
#pragma unroll
                for (int j = 0; j < KG; ++j) {
                    const int r = r0 + j * G + g.q;
                    uvo[j] = io::load_smem(su + r * CPB);
                    dlo[j] = io::load_smem(sd + r * CPB) + bias;
                }
                if (args.softplus) {
                    if (!PRECISE && KG % 2 == 0) {
#pragma unroll
                        for (int j = 0; j < KG; j += 2) {
                            const float2 sp = softplus2_fast(make_float2(dlo[j], dlo[j + 1]));
                            dlo[j] = sp.x;
                            dlo[j + 1] = sp.y;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < KG; ++j) dlo[j] = softplus<PRECISE>(dlo[j]);
                    }
                }
#pragma unroll
                for (int j = 0; j < KG; ++j) {
                    if (r0 + j * G + g.q >= rows) dlo[j] = 0.f;
                    duo[j] = dlo[j] * uvo[j];
                }
                float dl[KSTEP], du[KSTEP], y[KSTEP];
                exchange_steps<KSTEP, G>(dlo, duo, dl, du);
                recur_block<KSTEP, NS, PRECISE>(dl, du, fB + r0 * NSP + g.q * NS, fC + r0 * NSP + g.q * NS,
                                                NSP, A2, h2, y);
                if (MODE == kSegAgg) {
#pragma unroll
                    for (int j = 0; j < KG; ++j) dsum += (double)dlo[j];
                } else {
                    float yo[KG];
                    reduce_scatter_steps<KSTEP, G>(y, yo, g.q);
#pragma unroll
                    for (int j = 0; j < KG; ++j) {
                        const int r = r0 + j * G + g.q;
                        if (r < rows) {
                            float yy = fmaf(dskip, uvo[j], yo[j]);
                            if (pz) yy *= silu<PRECISE>(io::load_smem(sz + r * CPB));
                            io::store(po + off0 + (int64_t)r * Dm, yy);
                        }
                    }
                }
            }
        }
        __syncthreads();  // stage c % S and the fp32 B/C buffers are free again
    }
    cp_async_wait<0>();
    if (MODE == kSegAgg) dsum = group_sum_d<G>(dsum);
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
        h[2 * p] = h2[p].x;
        h[2 * p + 1] = h2[p].y;
    }
    lane_finish<NS, G, MODE>(args, g, seg, t_end, h, dsum);
}

template <typename IO, int NS, int G, int MODE>
static cudaError_t launch_mode(const ScanArgs &a, dim3 grid, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    using Lay = StagedLayout<IO, NS, G>;
    auto kern = scan_fwd_staged_kernel<IO, NS, G, P, MODE>;
    // the shared-memory opt-in is a per-device function attribute: set it once per device
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
    kern<<<grid, kBlock, Lay::SMEM, st>>>(a);
    return cudaGetLastError();
}

template <typename IO, int NS, int G>
static cudaError_t launch_t(const ScanArgs &a, int variant, cudaStream_t st) {
    constexpr int CPB = kBlock / G;
    const unsigned bx = (unsigned)(a.batch * ((a.dim + CPB - 1) / CPB));
    if (variant == kVariantSlab) return launch_mode<IO, NS, G, kFull>(a, dim3(bx, 1), st);
    cudaError_t e = launch_mode<IO, NS, G, kSegAgg>(a, dim3(bx, (unsigned)(a.nseg - 1)), st);
    if (e != cudaSuccess) return e;
    return launch_mode<IO, NS, G, kSegFinal>(a, dim3(bx, (unsigned)a.nseg), st);
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

cudaError_t launch_scan_staged(const ScanArgs &a, bool bf16, int ns, int g, int variant, cudaStream_t st) {
    return bf16 ? launch_io<__nv_bfloat16>(a, ns, g, variant, st) : launch_io<float>(a, ns, g, variant, st);
}

}  // namespace ssm
