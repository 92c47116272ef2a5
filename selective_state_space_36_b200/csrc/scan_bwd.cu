// scan_bwd.cu -- gradient of the selective scan (Euler Bbar), sm_100a.
//
// Training through the scan by recomputation (【論文要約】Mamba notes,
// "3.ハードウェアを考慮した効率的なアルゴリズム": intermediate states are
// recomputed rather than kept; NL-345 Mamba translation, section 1, "Fast
// training and inference").  The forward recurrence is the one of
// scan_fwd.cu; differentiating the loss sum(dout * out) through it gives, per
// channel (b, d), with lambda_t = dL/dh_t:
//     dy_t = dout_t silu(z_t),  dz_t = dout_t y_t sigmoid(z_t)(1 + z_t (1 - sigmoid(z_t)))
//     lambda_t = dy_t C_t + Abar_{t+1} lambda_{t+1}         (adjoint, backwards in t)
//     dC_t += dy_t h_t,  dB_t += lambda_t Delta_t u_t       (summed over channels)
//     dDelta_t = sum_n lambda_t,n (A_n Abar_t,n h_{t-1},n + B_t,n u_t)
//     dA_n += lambda_t,n Delta_t Abar_t,n h_{t-1},n         (summed over batch, time)
//     du_t = dy_t D + Delta_t sum_n lambda_t,n B_t,n,  dD += dy_t u_t
//     ddelta_t = dDelta_t sigmoid(delta_t + bias) (softplus) or dDelta_t,
//     dbias += ddelta_t,  dh0 = Abar_0 lambda_0.
//
// Layout: G = 4 lanes share a channel, each holding NS states; a block of 128
// threads covers 32 channels of one batch row.
//   phase 1  runs the forward recurrence once and stores the state entering
//            every chunk of KC steps (KC * NS = 64) in the workspace
//            (batch, chunk, dim, N) -- 1/KC of the expanded state;
//   phase 2  walks the chunks backwards: it recomputes the chunk's KC states
//            from the checkpoint into registers, then runs the adjoint
//            recurrence over them.
// Channel-shared gradients dB, dC: each lane writes its per-step products to a
// shared-memory tile [step][channel][state]; after every RK = KC / 2 steps
// the block sums the tile over its 32 channels (64 threads, one float4 of
// states each) and adds the sums to global memory with vector atomics.  dA,
// dD, dbias are accumulated per lane and added once per block.
#include <atomic>

#include "cp_async.cuh"
#include "scan_kernels.cuh"

namespace ssm {

namespace {

constexpr int kBwdG = 4;                  // lanes per channel
constexpr int kBwdCPB = kBlock / kBwdG;   // channels per block

template <int NS>
struct BwdShape {
    static constexpr int KC = 64 / NS;    // steps per recomputed chunk
    static constexpr int RK = KC / 2;     // steps per dB/dC reduction round
    static constexpr int NSP = NS * kBwdG;
    static constexpr int NQ = NSP / 4;    // float4 columns of a tile row
    // [2 (dC, dB)][RK][channel][NSP] floats
    static constexpr size_t smem_bytes = sizeof(float) * 2 * RK * kBwdCPB * NSP;
    static_assert(2 * RK * NQ == 64, "one reduction column per thread of two warps");
};

template <bool PRECISE>
__device__ __forceinline__ float sigmoid_of(float x) {
    if (PRECISE) return 1.f / (1.f + expf(-x));
    return rcp_approx(1.f + ex2_approx(-x * kLog2e));
}

template <typename IO, int NS, bool PRECISE>
__global__ void __launch_bounds__(kBlock)
scan_bwd_kernel(const ScanBwdArgs args) {
    using io = io_traits<IO>;
    using S = BwdShape<NS>;
    constexpr int G = kBwdG, KC = S::KC, RK = S::RK, NSP = S::NSP, NQ = S::NQ;
    extern __shared__ float4 sred4[];
    float *sred = reinterpret_cast<float *>(sred4);

    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x;
    const int q = tid % G, ch = tid / G;
    const int64_t tiles = (Dm + kBwdCPB - 1) / kBwdCPB;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d = (blockIdx.x % tiles) * kBwdCPB + ch;
    const bool active = d < Dm;
    const int64_t nchunks = (L + KC - 1) / KC;

    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);
    const IO *pdo = static_cast<const IO *>(args.dout);

    float Aw[NS], An[NS], h[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = q * NS + i;
        const bool ok = active && n < N;
        An[i] = ok ? args.A[d * N + n] : 0.f;
        Aw[i] = scale_A<PRECISE>(An[i]);
        h[i] = (ok && args.h0) ? args.h0[(b * Dm + d) * N + n] : 0.f;
    }
    const float bias = (active && args.bias) ? args.bias[d] : 0.f;
    const float dskip = (active && args.Dskip) ? args.Dskip[d] : 0.f;
    // checkpoint c of this lane: ckpt[b][c][d][q * NS ...]
    float *const ck_lane = args.ckpt + (b * nchunks * Dm + d) * N + q * NS;
    const int64_t ck_stride = Dm * N;

    // ---- phase 1: forward recurrence, checkpoint the state entering each chunk
    if (active) {
        for (int64_t c = 0; c < nchunks; ++c) {
            float *cp = ck_lane + c * ck_stride;
#pragma unroll
            for (int i = 0; i < NS; ++i)
                if (q * NS + i < N) cp[i] = h[i];
            const int64_t t0 = c * KC;
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                if (t0 + k >= L) break;
                const int64_t off = (b * L + t0 + k) * Dm + d;
                const float s = io::load(pd + off) + bias;
                const float dl = args.softplus ? softplus<PRECISE>(s) : s;
                const float du = dl * io::load(pu + off);
                const IO *brow = pB + (b * L + t0 + k) * N + q * NS;
#pragma unroll
                for (int i = 0; i < NS; ++i) {
                    const float bv = (q * NS + i < N) ? io::load(brow + i) : 0.f;
                    h[i] = fmaf(decay<PRECISE>(dl, Aw[i]), h[i], du * bv);
                }
            }
        }
    }

    // ---- phase 2: adjoint recurrence over the chunks, last to first
    float lam[NS], dA_acc[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) { lam[i] = 0.f; dA_acc[i] = 0.f; }
    float dD_acc = 0.f, dbias_acc = 0.f;
    IO *gdu = static_cast<IO *>(args.du);
    IO *gdd = static_cast<IO *>(args.ddelta);
    IO *gdz = static_cast<IO *>(args.dz);

    for (int64_t c = nchunks - 1; c >= 0; --c) {
        const int64_t t0 = c * KC;
        const int kc = (int)(L - t0 < KC ? L - t0 : KC);
        // recompute the chunk's states: hs[k] = h_{t0 + k}; h0c = h_{t0 - 1}
        float hs[KC][NS], h0c[NS];
#pragma unroll
        for (int i = 0; i < NS; ++i)
            h0c[i] = (active && q * NS + i < N) ? ck_lane[c * ck_stride + i] : 0.f;
#pragma unroll
        for (int i = 0; i < NS; ++i) h[i] = h0c[i];
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (k < kc && active) {
                const int64_t off = (b * L + t0 + k) * Dm + d;
                const float s = io::load(pd + off) + bias;
                const float dl = args.softplus ? softplus<PRECISE>(s) : s;
                const float du = dl * io::load(pu + off);
                const IO *brow = pB + (b * L + t0 + k) * N + q * NS;
#pragma unroll
                for (int i = 0; i < NS; ++i) {
                    const float bv = (q * NS + i < N) ? io::load(brow + i) : 0.f;
                    h[i] = fmaf(decay<PRECISE>(dl, Aw[i]), h[i], du * bv);
                }
            }
#pragma unroll
            for (int i = 0; i < NS; ++i) hs[k][i] = h[i];
        }

        // reverse sweep; every lane of the block runs every step (tile rows of
        // steps past the end are written but never reduced)
#pragma unroll
        for (int k = KC - 1; k >= 0; --k) {
            const int64_t t = t0 + k;
            const bool live = active && k < kc;
            const int64_t off = (b * L + t) * Dm + d;
            const int64_t row = (b * L + t) * N + q * NS;
            float uv = 0.f, raw = 0.f, zv = 0.f, go = 0.f, bv[NS], cv[NS];
            if (live) {
                uv = io::load(pu + off);
                raw = io::load(pd + off);
                go = io::load(pdo + off);
                if (pz) zv = io::load(pz + off);
            }
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const bool ok = live && q * NS + i < N;
                bv[i] = ok ? io::load(pB + row + i) : 0.f;
                cv[i] = ok ? io::load(pC + row + i) : 0.f;
            }
            const float s = raw + bias;
            const float dl = live ? (args.softplus ? softplus<PRECISE>(s) : s) : 0.f;
            // y_t, needed by the gate's derivative
            float yp = 0.f;
#pragma unroll
            for (int i = 0; i < NS; ++i) yp = fmaf(cv[i], hs[k][i], yp);
            const float y = group_sum<G>(yp) + dskip * uv;
            float dy = go;
            if (pz) {
                const float sg = sigmoid_of<PRECISE>(zv);
                dy = go * zv * sg;
                if (q == 0 && live) io::store(gdz + off, go * y * sg * (1.f + zv * (1.f - sg)));
            }
            const float dlu = dl * uv;
            float ddl_p = 0.f, dub_p = 0.f, pc[NS], pb[NS];
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const float hprev = k > 0 ? hs[k - 1][i] : h0c[i];
                const float a = decay<PRECISE>(dl, Aw[i]);
                lam[i] = fmaf(dy, cv[i], lam[i]);
                pc[i] = dy * hs[k][i];
                pb[i] = lam[i] * dlu;
                const float ga = lam[i] * hprev * a;
                ddl_p = fmaf(ga, An[i], fmaf(lam[i], bv[i] * uv, ddl_p));
                dA_acc[i] = fmaf(ga, dl, dA_acc[i]);
                dub_p = fmaf(lam[i], bv[i], dub_p);
                lam[i] *= a;
            }
            const int j = k % RK;
#pragma unroll
            for (int m = 0; m < NS; m += 4) {
                float *rc = sred + ((size_t)(0 * RK + j) * kBwdCPB + ch) * NSP + q * NS + m;
                float *rb = sred + ((size_t)(1 * RK + j) * kBwdCPB + ch) * NSP + q * NS + m;
                *reinterpret_cast<float4 *>(rc) = make_float4(pc[m], pc[m + 1], pc[m + 2], pc[m + 3]);
                *reinterpret_cast<float4 *>(rb) = make_float4(pb[m], pb[m + 1], pb[m + 2], pb[m + 3]);
            }
            const float ddl = group_sum<G>(ddl_p);
            const float dub = group_sum<G>(dub_p);
            if (q == 0 && live) {
                io::store(gdu + off, fmaf(dy, dskip, dl * dub));
                const float dd = args.softplus ? ddl * sigmoid_of<PRECISE>(s) : ddl;
                io::store(gdd + off, dd);
                dbias_acc += dd;
                dD_acc = fmaf(dy, uv, dD_acc);
            }
            if (j == 0) {
                // round done (steps k .. k + RK - 1): sum the tile over the
                // block's channels
                __syncthreads();
                if (tid < 64) {
                    const int nq = tid % NQ;
                    const int jj = (tid / NQ) % RK;
                    const int which = tid / (NQ * RK);  // 0: dC, 1: dB
                    const float4 *col = sred4 + (size_t)(which * RK + jj) * kBwdCPB * NQ + nq;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
                    for (int cc = 0; cc < kBwdCPB; ++cc) {
                        // start each row at a different channel so that the
                        // rows of a quarter-warp fall in different banks
                        const float4 v = col[(size_t)((cc + jj) & (kBwdCPB - 1)) * NQ];
                        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                    }
                    const int64_t tt = t0 + k + jj;
                    const int n = nq * 4;
                    if (tt < L && n < N) {
                        float *dst = (which ? args.dB : args.dC) + (b * L + tt) * N + n;
                        if (args.vec_red) {
                            atomicAdd(reinterpret_cast<float4 *>(dst), acc);
                        } else {
                            const float av[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (n + e < N) atomicAdd(dst + e, av[e]);
                        }
                    }
                }
                __syncthreads();
            }
        }
    }
    if (!active) return;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = q * NS + i;
        if (n < N) {
            atomicAdd(args.dA + d * N + n, dA_acc[i]);
            if (args.dh0) args.dh0[(b * Dm + d) * N + n] = lam[i];
        }
    }
    if (q == 0) {
        if (args.dD) atomicAdd(args.dD + d, dD_acc);
        if (args.dbias) atomicAdd(args.dbias + d, dbias_acc);
    }
}

// ---------------------------------------------------------------------------
// Staged backward (N <= 16, rows 16-byte aligned): the second pass of the
// backward scan with every input brought through shared memory.
//
// The first pass is the staged forward kernel in checkpoint mode, which
// stores the state entering every KC-th step.  This kernel walks the chunks of
// T steps of its (batch row, 32-channel) tile from the last to the first; the
// copies of the next S - 1 chunks (u, delta, z, dout tiles and the B, C rows)
// are in flight while the current one is processed.  Within a chunk it takes
// the sub-chunks of KC steps from last to first:
//   scalars    lane q of a channel's group of 4 computes Delta, Delta u,
//              sigmoid(z) and dy = dout silu(z) for steps k0 + 4 j + q and the
//              values travel to the other lanes by shuffles;
//   recompute  from the checkpoint, the KC states of this lane's 4 states
//              (kept in registers; the decays are recomputed in the reverse
//              sweep rather than kept, which leaves room for four blocks per
//              SM);
//   reverse    the adjoint recurrence over the KC steps, G steps at a time;
//              after each group of G steps the per-step partial sums of
//              dDelta, sum_n lambda B and y are reduce-scattered to the owning
//              lanes, which finish du, ddelta, dz and write them into the
//              consumed input rows of the tile (u, delta, z) -- the chunk's
//              gradients then leave in 16-byte pieces;
//   dB, dC     a [KC][channel][state] tile in shared memory, summed over the
//              32 channels by all 128 threads (two threads per output quad,
//              16 channels each, joined by a shuffle) and added to global
//              memory with one vector atomic per quad.
#ifndef SSM_BWD_MIN_BLOCKS_BF16
#define SSM_BWD_MIN_BLOCKS_BF16 4
#endif
// Chunks of 24 steps in two stages (55 KB of shared memory per block, four
// blocks per SM) measured a backward call at the 1.4B layer 1.934 ms against
// 1.958 with 16 steps in three stages: fewer chunk barriers and waits.
#ifndef SSM_BWD_CHUNK
#define SSM_BWD_CHUNK 24
#endif
#ifndef SSM_BWD_STAGES
#define SSM_BWD_STAGES 2
#endif

template <typename IO>
struct BwdStagedLayout {
    static constexpr int G = 4, NS = 4, NSP = 16, CPB = kBlock / G;
    static constexpr int T = SSM_BWD_CHUNK;               // steps per staged chunk
    static constexpr int KC = kCkptEvery;                 // steps per sub-chunk (checkpoint spacing)
    static constexpr int S = SSM_BWD_STAGES;              // pipeline stages
    static constexpr int ROW = CPB + 8;                   // tile row, padded against bank conflicts
    static constexpr int TILE = T * ROW;
    static constexpr int RAW = T * NSP;                   // raw B or C rows (elements)
    static constexpr size_t STAGE_BYTES = (4 * (size_t)TILE + 2 * RAW) * sizeof(IO);
    static constexpr size_t BC_BYTES = 2 * (size_t)T * NSP * sizeof(float);
    // reduction tile [2 (dC, dB)][KC][CPB][NSP]; each step's slab is padded by
    // 16 floats
    static constexpr int KSTRIDE = CPB * NSP + 16;
    static constexpr size_t RED_BYTES = 2 * (size_t)KC * KSTRIDE * sizeof(float);
    static constexpr size_t SMEM = S * STAGE_BYTES + BC_BYTES + RED_BYTES;
    // blocks per SM the kernel is compiled for: four for the bf16 tier
    // (65536 / (128 x 4) = 128 registers per thread, 53 KB of shared memory
    // per block), three for fp32 I/O (larger tiles)
    static constexpr int MIN_BLOCKS = sizeof(IO) == 2 ? SSM_BWD_MIN_BLOCKS_BF16 : 3;
    static_assert(T % KC == 0 && KC % G == 0, "chunks hold whole sub-chunks of whole step groups");
    static_assert((ROW * sizeof(IO)) % 16 == 0, "tile rows leave in 16-byte pieces");
};

template <int K, int G>
__device__ __forceinline__ void exchange_one(const float (&own)[K / G], float (&all)[K]) {
    const unsigned lane = threadIdx.x & 31u;
    const unsigned base = lane & ~(unsigned)(G - 1);
    const unsigned mask = ((1u << G) - 1u) << base;
#pragma unroll
    for (int k = 0; k < K; ++k) all[k] = __shfl_sync(mask, own[k / G], base + k % G);
}

template <typename IO, bool PRECISE>
__global__ void __launch_bounds__(kBlock, BwdStagedLayout<IO>::MIN_BLOCKS)
scan_bwd_staged_kernel(const ScanBwdArgs args) {
    using io = io_traits<IO>;
    using Lay = BwdStagedLayout<IO>;
    constexpr int G = Lay::G, NS = Lay::NS, NSP = Lay::NSP, CPB = Lay::CPB;
    constexpr int T = Lay::T, KC = Lay::KC, S = Lay::S, ROW = Lay::ROW, TILE = Lay::TILE;
    constexpr int EPV = 16 / sizeof(IO);   // elements per 16-byte piece
    constexpr int ROWV = CPB / EPV;        // pieces per tile row
    constexpr int KG = KC / G;             // steps per sub-chunk whose scalars this lane owns
    constexpr int NQ = NSP / 4;            // float4 columns of a reduction row
    extern __shared__ __align__(16) unsigned char smem[];
    float *fB = reinterpret_cast<float *>(smem + S * Lay::STAGE_BYTES);
    float *fC = fB + T * NSP;
    float *sred = fC + T * NSP;            // [2 (dC, dB)][KC] slabs of [CPB][NSP], KSTRIDE apart
    constexpr int KSTRIDE = Lay::KSTRIDE;

    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    // lane c + 8 q of warp w: state slot q of channel 8 w + c (the 8 lanes of
    // a quarter-warp hold 8 channels and read the same B/C address)
    constexpr int LS = 8;  // lane stride of a channel's group
    const int tid = threadIdx.x, q = (tid & 31) / LS, grp = (tid >> 5) * LS + (tid & (LS - 1));
    const int64_t tiles = (Dm + CPB - 1) / CPB;
    const int64_t b = blockIdx.x / tiles;
    const int64_t d0 = (blockIdx.x % tiles) * CPB;
    const int64_t d = d0 + grp;
    const bool active = d < Dm;
    const int nchunks = (int)((L + T - 1) / T);
    const int64_t nck = (L + KC - 1) / KC;

    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = static_cast<const IO *>(args.z);
    const IO *pB = static_cast<const IO *>(args.B);
    const IO *pC = static_cast<const IO *>(args.C);
    const IO *pdo = static_cast<const IO *>(args.dout);
    IO *gdu = static_cast<IO *>(args.du);
    IO *gdd = static_cast<IO *>(args.ddelta);
    IO *gdz = static_cast<IO *>(args.dz);

    auto stage_ptr = [&](int s) { return reinterpret_cast<IO *>(smem + s * Lay::STAGE_BYTES); };
    // the o-th chunk processed is chunk nchunks - 1 - o; it lands in stage o % S
    auto issue = [&](int o) {
        const int64_t tc = (int64_t)(nchunks - 1 - o) * T;
        const int rows = (int)(L - tc < T ? L - tc : T);
        IO *st = stage_ptr(o % S);
        IO *su = st, *sd = st + TILE, *sz = st + 2 * TILE, *sg = st + 3 * TILE;
        IO *rb = st + 4 * TILE, *rc = rb + Lay::RAW;
        for (int p = tid; p < T * ROWV; p += kBlock) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            const bool ok = r < rows && col < Dm;
            const int64_t go = ok ? (b * L + tc + r) * Dm + col : 0;
            const int so = r * ROW + v * EPV;
            cp_async16(su + so, pu + go, ok);
            cp_async16(sd + so, pd + go, ok);
            if (pz) cp_async16(sz + so, pz + go, ok);
            cp_async16(sg + so, pdo + go, ok);
        }
        const int pieces = rows * N / EPV;  // the chunk's B/C rows are contiguous
        const int64_t gbc = (b * L + tc) * N;
        for (int p = tid; p < pieces; p += kBlock) {
            cp_async16(rb + p * EPV, pB + gbc + p * EPV, true);
            cp_async16(rc + p * EPV, pC + gbc + p * EPV, true);
        }
    };

    // per-lane constants: A pairs, scaled for the decay (the fast tier's
    // log2(e) factor comes off the dDelta sums once per step, below)
    float2 Aw2[NS / 2];
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
        float v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = q * NS + 2 * p + e;
            v[e] = (active && n < N) ? args.A[d * N + n] : 0.f;
        }
        Aw2[p] = make_float2(scale_A<PRECISE>(v[0]), scale_A<PRECISE>(v[1]));
    }
    constexpr float kAUnscale = PRECISE ? 1.f : kLn2;
    const float bias = (active && args.bias) ? args.bias[d] : 0.f;
    const float dskip = (active && args.Dskip) ? args.Dskip[d] : 0.f;
    const float *ck_lane = args.ckpt + (b * nck * Dm + d) * N + q * NS;

    float2 lam2[NS / 2], dA2[NS / 2];
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) { lam2[p] = make_float2(0.f, 0.f); dA2[p] = make_float2(0.f, 0.f); }
    float dD_acc = 0.f, dbias_acc = 0.f;

#pragma unroll
    for (int o = 0; o < S - 1; ++o) {
        if (o < nchunks) issue(o);
        cp_async_commit();
    }
    for (int o = 0; o < nchunks; ++o) {
        cp_async_wait<S - 2>();
        // chunk o has landed for every thread, and every thread is done with
        // the stage that chunk o + S - 1 goes to (it held chunk o - 1)
        __syncthreads();
        if (o + S - 1 < nchunks) issue(o + S - 1);
        cp_async_commit();
        const int64_t tc = (int64_t)(nchunks - 1 - o) * T;
        const int rows = (int)(L - tc < T ? L - tc : T);
        IO *st = stage_ptr(o % S);
        {
            const IO *rb = st + 4 * TILE, *rc = rb + Lay::RAW;
            if (rows == T && N == NSP) {
                for (int i = 4 * tid; i < T * NSP; i += 4 * kBlock) {
                    float v[4];
                    io::load4_smem(rb + i, v);
                    *reinterpret_cast<float4 *>(fB + i) = make_float4(v[0], v[1], v[2], v[3]);
                    io::load4_smem(rc + i, v);
                    *reinterpret_cast<float4 *>(fC + i) = make_float4(v[0], v[1], v[2], v[3]);
                }
            } else {
                for (int i = tid; i < T * NSP; i += kBlock) {
                    const int r = i / NSP, n = i % NSP;
                    const bool ok = r < rows && n < N;
                    fB[i] = ok ? io::load_smem(rb + r * N + n) : 0.f;
                    fC[i] = ok ? io::load_smem(rc + r * N + n) : 0.f;
                }
            }
        }
        __syncthreads();
        // this lane's rows of the tiles start at step q
        IO *su = st + grp + q * ROW, *sd = st + TILE + grp + q * ROW;
        IO *sz = st + 2 * TILE + grp + q * ROW, *sg = st + 3 * TILE + grp + q * ROW;
        const float *fBq = fB + q * NS, *fCq = fC + q * NS;
        float *sredq = sred + q * (CPB * NS) + grp * NS;  // [q][channel][4] slabs

        // One sub-chunk of KC steps starting at chunk row k0 (nrows: the rows
        // of this chunk; the constant T for full chunks).
        auto sub_chunk = [&](const int k0, const int nrows) {
            const int64_t t0 = tc + k0;
            // the state entering the sub-chunk, loaded first so that the step
            // scalars below cover its latency
            float2 hc[NS / 2];
            {
                const float *cp = ck_lane + (t0 / KC) * Dm * N;
#pragma unroll
                for (int p = 0; p < NS / 2; ++p) {
                    const int n = q * NS + 2 * p;
                    hc[p] = make_float2((active && n < N) ? __ldcs(cp + 2 * p) : 0.f,
                                        (active && n + 1 < N) ? __ldcs(cp + 2 * p + 1) : 0.f);
                }
            }
            // ---- per-step scalars of the owned steps k0 + j G + q (the raw
            // inputs are read again from the tile where the end of the
            // sub-chunk needs them)
            float so[KG], szo[KG], dlo[KG], duo[KG], dyo[KG];
#pragma unroll
            for (int j = 0; j < KG; ++j) so[j] = io::load_smem(sd + (k0 + j * G) * ROW) + bias;
            if (args.softplus) {
                if (!PRECISE && KG % 2 == 0) {
#pragma unroll
                    for (int j = 0; j < KG; j += 2) {
                        const float2 sp = softplus2_fast(make_float2(so[j], so[j + 1]));
                        dlo[j] = sp.x;
                        dlo[j + 1] = sp.y;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < KG; ++j) dlo[j] = softplus<PRECISE>(so[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < KG; ++j) dlo[j] = so[j];
            }
#pragma unroll
            for (int j = 0; j < KG; ++j) {
                const int rr = k0 + j * G;
                const float uo = io::load_smem(su + rr * ROW);
                float go = io::load_smem(sg + rr * ROW);
                if (rr + q >= nrows || !active) { dlo[j] = 0.f; go = 0.f; }
                duo[j] = dlo[j] * uo;
                if (pz) {
                    const float zo = io::load_smem(sz + rr * ROW);
                    szo[j] = sigmoid_of<PRECISE>(zo);
                    dyo[j] = go * zo * szo[j];
                } else {
                    szo[j] = 0.f;
                    dyo[j] = go;
                }
            }
            // ---- recompute the sub-chunk's states
            float2 hs[KC][NS / 2];
            {
                float dl[KC], du[KC];
                exchange_steps<KC, G, LS>(dlo, duo, dl, du);
                float2 h2[NS / 2];
#pragma unroll
                for (int p = 0; p < NS / 2; ++p) h2[p] = hc[p];
#pragma unroll
                for (int k = 0; k < KC; ++k) {
                    const float4 bv = *reinterpret_cast<const float4 *>(fBq + (k0 + k) * NSP);
                    const float2 d2 = make_float2(dl[k], dl[k]), u2 = make_float2(du[k], du[k]);
#pragma unroll
                    for (int p = 0; p < NS / 2; ++p) {
                        const float2 b2 = p ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y);
                        const float2 x2 = mul2(d2, Aw2[p]);
                        const float2 a2 = make_float2(decay_of<PRECISE>(x2.x), decay_of<PRECISE>(x2.y));
                        h2[p] = fma2(a2, h2[p], mul2(u2, b2));
                        hs[k][p] = h2[p];
                    }
                }
            }

            // ---- adjoint recurrence, last step first, G steps at a time (the
            // step scalars come from their owning lanes again, rather than
            // being held through the sweep)
            const unsigned gbase = LaneGroup<G, LS>::base(), gmask = LaneGroup<G, LS>::mask();
#pragma unroll
            for (int jg = KG - 1; jg >= 0; --jg) {
                float ddl_p[G], dub_p[G], y_p[G];
#pragma unroll
                for (int i = G - 1; i >= 0; --i) {
                    const int k = jg * G + i;
                    const float4 bv = *reinterpret_cast<const float4 *>(fBq + (k0 + k) * NSP);
                    const float4 cv = *reinterpret_cast<const float4 *>(fCq + (k0 + k) * NSP);
                    const float dyk = __shfl_sync(gmask, dyo[jg], gbase + i * LS);
                    const float dlk = __shfl_sync(gmask, dlo[jg], gbase + i * LS);
                    const float duk = __shfl_sync(gmask, duo[jg], gbase + i * LS);
                    const float2 dy2 = make_float2(dyk, dyk), dl2 = make_float2(dlk, dlk);
                    const float2 du2 = make_float2(duk, duk);
                    float2 accy = make_float2(0.f, 0.f), accd = accy, accb = accy, pc[NS / 2], pb[NS / 2];
#pragma unroll
                    for (int p = 0; p < NS / 2; ++p) {
                        const float2 b2 = p ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y);
                        const float2 c2 = p ? make_float2(cv.z, cv.w) : make_float2(cv.x, cv.y);
                        const float2 hprev = k > 0 ? hs[k - 1][p] : hc[p];
                        // the decay of step k, as the recomputation took it
                        float2 a2;
                        if (PRECISE) {
                            const float2 x2 = mul2(dl2, Aw2[p]);
                            a2 = make_float2(decay_of<PRECISE>(x2.x), decay_of<PRECISE>(x2.y));
                        } else {
                            a2 = decay2_fresh(dl2, Aw2[p]);
                        }
                        lam2[p] = fma2(dy2, c2, lam2[p]);
                        pc[p] = mul2(dy2, hs[k][p]);
                        pb[p] = mul2(lam2[p], du2);
                        accy = fma2(c2, hs[k][p], accy);
                        accb = fma2(lam2[p], b2, accb);
                        const float2 la = mul2(lam2[p], a2);
                        const float2 ga = mul2(la, hprev);
                        accd = fma2(ga, Aw2[p], accd);
                        dA2[p] = fma2(ga, dl2, dA2[p]);
                        lam2[p] = la;
                    }
                    *reinterpret_cast<float4 *>(sredq + k * KSTRIDE) =
                        make_float4(pc[0].x, pc[0].y, pc[1].x, pc[1].y);
                    *reinterpret_cast<float4 *>(sredq + (KC + k) * KSTRIDE) =
                        make_float4(pb[0].x, pb[0].y, pb[1].x, pb[1].y);
                    ddl_p[i] = (accd.x + accd.y) * kAUnscale;
                    dub_p[i] = accb.x + accb.y;
                    y_p[i] = accy.x + accy.y;
                }
                // lane q keeps the sums of step jg G + q (the step it owns)
                // and finishes that step's du, ddelta, dz
                float r[1];
                reduce_scatter_steps<G, G, LS>(ddl_p, r, q);
                const float ddl_o = r[0];
                reduce_scatter_steps<G, G, LS>(dub_p, r, q);
                const float dub = r[0];
                reduce_scatter_steps<G, G, LS>(y_p, r, q);
                const float y_o = r[0];
                const int rr = k0 + jg * G;
                if (rr + q < nrows && active) {
                    const float uo = io::load_smem(su + rr * ROW);
                    const float ddl = fmaf(uo, dub, ddl_o);
                    const float dd = args.softplus ? ddl * sigmoid_of<PRECISE>(so[jg]) : ddl;
                    io::store_smem(su + rr * ROW, fmaf(dyo[jg], dskip, dlo[jg] * dub));
                    io::store_smem(sd + rr * ROW, dd);
                    if (pz) {
                        const float zo = io::load_smem(sz + rr * ROW), go = io::load_smem(sg + rr * ROW);
                        const float y = fmaf(dskip, uo, y_o);
                        io::store_smem(sz + rr * ROW, go * y * szo[jg] * (1.f + zo * (1.f - szo[jg])));
                    }
                    dbias_acc += dd;
                    dD_acc = fmaf(dyo[jg], uo, dD_acc);
                }
            }
            // ---- dB, dC of the sub-chunk: 64 (which, step, quad) sums over
            // the block's 32 channels, two threads (adjacent lanes) per sum,
            // 16 channels each; thread (quad nq, half part) starts 2 nq + part
            // channels in, so that the 8 threads of a quarter-warp fall in 8
            // different banks
            __syncthreads();
            {
                const int task = tid >> 1, part = tid & 1;
                const int nq = task % NQ;
                const int kk = (task / NQ) % KC;
                const int which = task / (NQ * KC);  // 0: dC, 1: dB
                const float4 *col = reinterpret_cast<const float4 *>(sred + (which * KC + kk) * KSTRIDE) +
                                    nq * CPB + part * (CPB / 2);
                const int rot = 2 * nq + part;
                float2 a01 = make_float2(0.f, 0.f), a23 = a01, b01 = a01, b23 = a01;
#pragma unroll
                for (int cc = 0; cc < CPB / 2; cc += 2) {
                    const float4 v = col[(cc + rot) & (CPB / 2 - 1)];
                    const float4 w = col[(cc + 1 + rot) & (CPB / 2 - 1)];
                    a01 = add2(a01, make_float2(v.x, v.y));
                    a23 = add2(a23, make_float2(v.z, v.w));
                    b01 = add2(b01, make_float2(w.x, w.y));
                    b23 = add2(b23, make_float2(w.z, w.w));
                }
                a01 = add2(a01, b01);
                a23 = add2(a23, b23);
                a01.x += __shfl_xor_sync(0xffffffffu, a01.x, 1);
                a01.y += __shfl_xor_sync(0xffffffffu, a01.y, 1);
                a23.x += __shfl_xor_sync(0xffffffffu, a23.x, 1);
                a23.y += __shfl_xor_sync(0xffffffffu, a23.y, 1);
                const int n = nq * 4;
                if (part == 0 && k0 + kk < nrows && n < N) {
                    float *dst = (which ? args.dB : args.dC) + (b * L + t0 + kk) * N + n;
                    if (args.vec_red) {
                        atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(a01.x, a01.y, a23.x, a23.y));
                    } else {
                        const float av[4] = {a01.x, a01.y, a23.x, a23.y};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (n + e < N) atomicAdd(dst + e, av[e]);
                    }
                }
            }
            __syncthreads();
        };
        if (rows == T) {
#pragma unroll 1
            for (int sc = T / KC - 1; sc >= 0; --sc) sub_chunk(sc * KC, T);
        } else {
            for (int sc = (rows + KC - 1) / KC - 1; sc >= 0; --sc) sub_chunk(sc * KC, rows);
        }
        // ---- the chunk's du, ddelta, dz leave in 16-byte pieces (the stage
        // is reused S chunks later, after the barrier at the top of the loop)
        for (int p = tid; p < T * ROWV; p += kBlock) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            if (r < rows && col < Dm) {
                const int64_t go = (b * L + tc + r) * Dm + col;
                const int so = r * ROW + v * EPV;
                __stcs(reinterpret_cast<uint4 *>(gdu + go), *reinterpret_cast<const uint4 *>(st + so));
                __stcs(reinterpret_cast<uint4 *>(gdd + go), *reinterpret_cast<const uint4 *>(st + TILE + so));
                if (pz)
                    __stcs(reinterpret_cast<uint4 *>(gdz + go), *reinterpret_cast<const uint4 *>(st + 2 * TILE + so));
            }
        }
    }
    cp_async_wait<0>();
    // dD and dbias were accumulated by the owner of each step: sum the group
    dD_acc = group_sum<G, LS>(dD_acc);
    dbias_acc = group_sum<G, LS>(dbias_acc);
    if (!active) return;
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
        const int n = q * NS + 2 * p;
        const float lv[2] = {lam2[p].x, lam2[p].y}, av[2] = {dA2[p].x, dA2[p].y};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (n + e < N) {
                atomicAdd(args.dA + d * N + n + e, av[e]);
                if (args.dh0) args.dh0[(b * Dm + d) * N + n + e] = lv[e];
            }
        }
    }
    if (q == 0) {
        if (args.dD) atomicAdd(args.dD + d, dD_acc);
        if (args.dbias) atomicAdd(args.dbias + d, dbias_acc);
    }
}

template <typename IO>
cudaError_t launch_staged(const ScanBwdArgs &a, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    using Lay = BwdStagedLayout<IO>;
    auto kern = scan_bwd_staged_kernel<IO, P>;
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

template <typename IO, int NS>
cudaError_t launch_ns(const ScanBwdArgs &a, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    constexpr size_t smem = BwdShape<NS>::smem_bytes;
    auto kern = scan_bwd_kernel<IO, NS, P>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t tiles = (a.dim + kBwdCPB - 1) / kBwdCPB;
    kern<<<dim3((unsigned)(a.batch * tiles)), kBlock, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool scan_bwd_staged_eligible(const ScanBwdArgs &a, int es) {
    auto al = [](const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) % 16) == 0; };
    return a.dstate <= 16 && (a.dim * es) % 16 == 0 && (a.dstate * es) % 16 == 0 && al(a.u) && al(a.delta) &&
           al(a.z) && al(a.B) && al(a.C) && al(a.dout) && al(a.du) && al(a.ddelta) && al(a.dz);
}

int scan_bwd_staged_chunk() { return BwdStagedLayout<float>::KC; }

cudaError_t launch_scan_bwd_staged(const ScanBwdArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_staged<__nv_bfloat16>(a, st) : launch_staged<float>(a, st);
}

int scan_bwd_states_per_lane(int dstate) { return dstate <= 16 ? 4 : (dstate <= 32 ? 8 : 16); }

int64_t scan_bwd_chunk(int dstate) { return 64 / scan_bwd_states_per_lane(dstate); }

int64_t scan_bwd_channels_per_block() { return kBwdCPB; }

cudaError_t launch_scan_bwd(const ScanBwdArgs &a, bool bf16, cudaStream_t st) {
    const int ns = scan_bwd_states_per_lane(a.dstate);
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
