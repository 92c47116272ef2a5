// scan_fwd_staged.cuh -- selective-scan forward, staged variant (sm_100a).
//
// Same arithmetic as the generic kernel in scan_fwd.cu (NL-345 Mamba
// translation, section 2 eq. (2); 【論文要約】Mamba notes, S6 Algorithm 2,
// 数式解説 3), but every input reaches the compute loop through shared memory:
// each chunk of T time steps of the block's u, delta, z tiles
// ([T x channels-per-block]) and of B, C ([T x N]) is brought in with 16-byte
// cp.async copies, STAGES chunks ahead, so global-memory latency overlaps the
// recurrence of earlier chunks (the notes' hardware-aware algorithm: inputs go
// from HBM to on-chip memory once and only the outputs are written back).  B
// and C are widened to fp32 once per chunk and per block.
//
// Thread layout: G lanes share a group of CPL adjacent channels; lane q holds
// states [q NS, q NS + NS) of each of them.  B_t and C_t are read once per lane
// and step and serve all CPL channels, so the shared-memory traffic of the
// broadcast operands (the largest) falls by a factor CPL, and u, delta, z and
// out move CPL channels per access (one channel per lane is the default: at
// the benchmark shapes halving the warps costs more than the traffic saved).
// Tile rows are padded by 32 bytes so that the G rows the lanes of a group
// read at once fall in different banks.  With four lanes per channel the
// lanes of a group sit 8 apart in the warp, so that the 8 lanes of a
// quarter-warp read one B/C address (two L1 wavefronts per 128-bit load, not
// four).
//
// The waits are cp.async.wait_group (hardware-tracked completion of this
// thread's own copies) followed by a block barrier: there is no polling loop.
//
// Eligibility (checked on the host): dim * sizeof(io) and dstate * sizeof(io)
// are multiples of 16 bytes and u, delta, z, B, C, out start on 16-byte
// boundaries.
#pragma once

#include <atomic>

#include "cp_async.cuh"
#include "scan_common.cuh"

namespace ssm {

// Time steps processed together, by lanes per channel (measured at the
// 1.4B layer: two lanes 165.3 Gelem/s with 16-step blocks, 167.9 with 8; four
// lanes 163.6 with 16, 152.6 with 8).
#ifndef SSM_KSTEP_G1
#define SSM_KSTEP_G1 16
#endif
#ifndef SSM_KSTEP_G2
#define SSM_KSTEP_G2 8
#endif
#ifndef SSM_KSTEP_G4
#define SSM_KSTEP_G4 16
#endif
// Step blocks of the passes that produce states only (the backward's
// checkpoint pass, the sequence split's first pass; 0: the lane count's):
// 32-step blocks measured a backward call at the 1.4B layer 1.966 ms against
// 1.976 with 16, and the split at L = 1,048,576 15.24 ms against 15.37.
#ifndef SSM_KSTEP_STATES
#define SSM_KSTEP_STATES 32
#endif
// A multiple of G that divides the chunk, and with one channel per lane a
// multiple of 2G, so the per-step scalar work of a lane comes in pairs for
// the packed softplus.
template <int G, int CPL>
struct KStep {
    static constexpr int want = G == 1 ? SSM_KSTEP_G1 : (G == 2 ? SSM_KSTEP_G2 : SSM_KSTEP_G4);
    static constexpr int need = CPL == 2 ? G : 2 * G;
    static constexpr int value = want > need ? want : need;
};

// Two stages: one chunk computes while the next one lands.  A third stage
// costs enough shared memory to drop a resident block per SM at the 4-lane
// layout, which at the 1.4B-layer shape turns one wave of blocks into two.
#ifndef SSM_STAGES
#define SSM_STAGES 2
#endif
#ifndef SSM_CHUNK_BF16
#define SSM_CHUNK_BF16 32
#endif
// Four lanes per channel run 128-thread blocks (not the packed virtual
// blocks of two lanes), whose shared memory leaves room for 64-step chunks:
// at the 130M layer 130.7-131.1 Gelem/s against 128.8-129.4 with 32.
#ifndef SSM_CHUNK_BF16_G4
#define SSM_CHUNK_BF16_G4 64
#endif
// Step blocks of a full chunk unrolled together (1 = no unrolling).
#ifndef SSM_R0_UNROLL
#define SSM_R0_UNROLL 4
#endif
#define SSM_PRAGMA_(x) _Pragma(#x)
#define SSM_UNROLL_N(n) SSM_PRAGMA_(unroll n)

template <typename IO, int G>
struct StagedCfg {
    // time steps per chunk
    static constexpr int T = sizeof(IO) == 2 ? (G == 4 ? SSM_CHUNK_BF16_G4 : SSM_CHUNK_BF16) : 16;
    static constexpr int STAGES = SSM_STAGES;
};

// Row padding: with G > 1 the lanes of a group read G different rows at once,
// and 32 bytes of padding put those rows in different banks; with G = 1 all
// lanes read one row and padding would only cost shared memory.
#ifndef SSM_ROW_PAD_BYTES
#define SSM_ROW_PAD_BYTES 32
#endif

template <typename IO, int NS, int G, int CPL, int TPB = kBlock>
struct StagedLayout {
    static constexpr int T = StagedCfg<IO, G>::T;
    static constexpr int S = StagedCfg<IO, G>::STAGES;
    static constexpr int GROUPS = TPB / G;                    // channel groups per block
    static constexpr int CPB = GROUPS * CPL;                  // channels per block
    static constexpr int NSP = NS * G;                        // padded states per channel
    static constexpr int ROW = CPB + (G > 1 ? SSM_ROW_PAD_BYTES / (int)sizeof(IO) : 0);  // tile row (elements)
    static constexpr int TILE = T * ROW;                      // elements of one u/delta/z tile
    static constexpr int RAW = T * NSP;                       // elements reserved for one raw B or C tile
    static constexpr size_t STAGE_BYTES = (3 * (size_t)TILE + 2 * RAW) * sizeof(IO);
    static constexpr size_t BC_BYTES = 2 * (size_t)T * NSP * sizeof(float);
    static constexpr size_t SMEM = S * STAGE_BYTES + BC_BYTES;
};

// CPL consecutive values from shared memory / to global memory.
template <typename IO, int CPL>
__device__ __forceinline__ void load_vals(const IO *p, float (&v)[CPL]) {
    if (CPL == 2 && sizeof(IO) == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
        v[0] = __uint_as_float(w << 16);
        v[CPL - 1] = __uint_as_float(w & 0xffff0000u);
    } else if (CPL == 2) {
        const float2 w = *reinterpret_cast<const float2 *>(p);
        v[0] = w.x;
        v[CPL - 1] = w.y;
    } else {
        v[0] = io_traits<IO>::load_smem(p);
    }
}

template <typename IO, int CPL>
__device__ __forceinline__ void store_vals(IO *p, const float (&v)[CPL]) {
    if (CPL == 2 && sizeof(IO) == 2) {
        const __nv_bfloat162 w = __floats2bfloat162_rn(v[0], v[CPL - 1]);
        __stcs(reinterpret_cast<unsigned int *>(p), *reinterpret_cast<const unsigned int *>(&w));
    } else if (CPL == 2) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(v[0], v[CPL - 1]));
    } else {
        io_traits<IO>::store(p, v[0]);
    }
}

// Barrier of one virtual block (below): a warp barrier when the virtual block
// is one warp, else hardware barrier 1 + vb with the virtual block's threads.
// Only the one-pass mode packs several virtual blocks per CTA; the others
// use the CTA barrier.
template <int TPB, int MODE>
__device__ __forceinline__ void vblock_sync(int vb) {
    if (TPB == 32) __syncwarp();
    else if (MODE != kFull && MODE != kCkpt) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(vb + 1), "n"(TPB) : "memory");
}

// Threads a CTA of the staged kernel may have.  The one-pass modes (the scan
// and the backward's checkpoint pass) pack several virtual blocks per CTA: up
// to 512 threads for layouts whose lanes hold at most 8 states (they stay
// below 128 registers), else 256, so that ptxas may give every thread up to
// 255 registers.  The split passes launch one 128-thread block per unit.
template <int G, int NS, int CPL, int MODE>
struct StagedMaxThreads {
    static constexpr int value =
        (MODE != kFull && MODE != kCkpt) ? kBlock : (G > 1 && NS * CPL <= 8 ? 512 : 256);
};

template <typename IO, int NS, int G, int CPL, bool PRECISE, int MODE, bool ZOH, int TPB>
__global__ void __launch_bounds__(StagedMaxThreads<G, NS, CPL, MODE>::value)
scan_fwd_staged_kernel(const ScanArgs args) {
    using io = io_traits<IO>;
    using Lay = StagedLayout<IO, NS, G, CPL, TPB>;
    constexpr int T = Lay::T, S = Lay::S, CPB = Lay::CPB, NSP = Lay::NSP, ROW = Lay::ROW;
    constexpr int EPV = 16 / sizeof(IO);  // elements per 16-byte piece
    constexpr int ROWV = CPB / EPV;       // pieces per tile row
    // the checkpoint pass and the split's first pass produce states only:
    // no C rows staged, no readout
    constexpr bool kReadout = MODE != kCkpt && MODE != kSegAgg;
    // Step block: the lane count's, longer for the state-only passes (no
    // readout to hold); at most a chunk, and in the checkpoint pass whole
    // numbers of the checkpoint spacing.
    constexpr int KSTEP_WANT = (!kReadout && SSM_KSTEP_STATES > 0) ? SSM_KSTEP_STATES : KStep<G, CPL>::value;
    constexpr int KSTEP = KSTEP_WANT < T ? KSTEP_WANT : T;
    static_assert(MODE != kCkpt || KSTEP % kCkptEvery == 0, "checkpoints fall on step-block pieces");
    constexpr int KG = KSTEP / G;         // steps whose scalar work this lane does
    static_assert(T % KSTEP == 0, "a chunk holds whole step blocks");
    // A CTA holds blockDim.x / TPB virtual blocks.  Virtual block vb of CTA
    // k works on unit k + vb * gridDim.x -- one (batch row, channel tile) for
    // the whole sequence (segment) -- with its own shared memory and its own
    // barrier, independently of the CTA's other virtual blocks; several of
    // them per CTA let the launch place the units evenly over the SMs.
    extern __shared__ __align__(16) unsigned char smem_all[];
    const int vb = threadIdx.x / TPB;
    const int64_t unit = blockIdx.x + (int64_t)vb * gridDim.x;
    if (unit >= args.units) return;  // no barrier is shared with other virtual blocks
    unsigned char *smem = smem_all + vb * Lay::SMEM;
    float *fB = reinterpret_cast<float *>(smem + S * Lay::STAGE_BYTES);
    float *fC = fB + T * NSP;

    const int64_t L = args.seqlen, Dm = args.dim;
    const int N = args.dstate;
    const int tid = threadIdx.x % TPB;
    // With four lanes per channel they sit 8 apart (lane c + 8 q of a warp:
    // state slice q of the warp's channel c), so that the 8 lanes of a
    // quarter-warp read one B/C address (two L1 wavefronts per 128-bit load
    // instead of four); with one or two lanes they are adjacent.
    constexpr int LS = G == 4 ? 8 : 1;
    static_assert(G != 4 || TPB % 32 == 0, "four-lane groups spread over whole warps");
    const int q = G == 4 ? (tid & 31) / LS : tid % G;
    const int grp = G == 4 ? (tid >> 5) * LS + (tid & (LS - 1)) : tid / G;
    const int64_t tiles = (Dm + CPB - 1) / CPB;
    const int64_t b = unit / tiles;
    const int64_t d0 = (unit % tiles) * CPB;
    const int64_t dfirst = d0 + (int64_t)grp * CPL;  // first channel of this group
    const bool active = dfirst < Dm;                  // dim is a multiple of CPL here
    // checkpoint c of this lane (kCkpt): ckpt[b][c][dfirst][q NS ...]
    const int64_t ck_stride = Dm * N;
    float *const ck_base = MODE == kCkpt ? args.ckpt + (b * ((L + kCkptEvery - 1) / kCkptEvery) * Dm + dfirst) * N + q * NS
                                         : nullptr;
    const int seg = blockIdx.y;
    const int64_t t_begin = (int64_t)seg * args.seg_len;
    const int64_t t_end = t_begin + args.seg_len < L ? t_begin + args.seg_len : L;

    const IO *pu = static_cast<const IO *>(args.u);
    const IO *pd = static_cast<const IO *>(args.delta);
    const IO *pz = (MODE == kSegAgg || MODE == kCkpt) ? nullptr : static_cast<const IO *>(args.z);
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
        for (int p = tid; p < T * ROWV; p += TPB) {
            const int r = p / ROWV, v = p % ROWV;
            const int64_t col = d0 + v * EPV;
            const bool ok = r < rows && col < Dm;
            const int64_t go = ok ? (b * L + tc + r) * Dm + col : 0;
            const int so = r * ROW + v * EPV;
            cp_async16(su + so, pu + go, ok);
            cp_async16(sd + so, pd + go, ok);
            if (pz) cp_async16(sz + so, pz + go, ok);
        }
        const int pieces = rows * N / EPV;  // B/C rows of this chunk are contiguous
        const int64_t gbc = (b * L + tc) * N;
        for (int p = tid; p < pieces; p += TPB) {
            cp_async16(rb + p * EPV, pB + gbc + p * EPV, true);
            if (kReadout) cp_async16(rc + p * EPV, pC + gbc + p * EPV, true);
        }
    };

    // per-channel constants and state
    float2 A2[CPL][NS / 2], h2[CPL][NS / 2], invA2[CPL][NS / 2];
    float bias[CPL], dskip[CPL];
    double dsum[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const LaneRef lr{b, dfirst + c, q, active};
        float Aw[NS], h[NS];
        lane_init<NS, PRECISE, MODE>(args, lr, seg, Aw, h);
#pragma unroll
        for (int p = 0; p < NS / 2; ++p) {
            A2[c][p] = make_float2(Aw[2 * p], Aw[2 * p + 1]);
            h2[c][p] = make_float2(h[2 * p], h[2 * p + 1]);
            if (ZOH) {  // 1 / A in natural units (Aw carries log2(e) in the fast tier)
                const float s0 = PRECISE ? 1.f : kLn2;
                invA2[c][p] = make_float2(1.f / (Aw[2 * p] * s0), 1.f / (Aw[2 * p + 1] * s0));
            }
        }
        bias[c] = (active && args.bias) ? args.bias[dfirst + c] : 0.f;
        dskip[c] = (active && args.Dskip) ? args.Dskip[dfirst + c] : 0.f;
        dsum[c] = 0.0;
    }

#pragma unroll
    for (int c = 0; c < S - 1; ++c) {
        if (c < nchunks) issue(c);
        cp_async_commit();
    }
    for (int c = 0; c < nchunks; ++c) {
        if (c + S - 1 < nchunks) issue(c + S - 1);
        cp_async_commit();
        cp_async_wait<S - 1>();  // this thread's copies of chunk c have landed
        vblock_sync<TPB, MODE>(vb);    // ... and everyone else's
        const int64_t tc = t_begin + (int64_t)c * T;
        const int rows = (int)(t_end - tc < T ? t_end - tc : T);
        const IO *st = stage_ptr(c % S);
        const IO *rb = st + 3 * Lay::TILE, *rc = rb + Lay::RAW;
        if (rows == T && N == NSP) {
            // whole chunk, no padded states: four values per thread and copy
            for (int i = 4 * tid; i < T * NSP; i += 4 * TPB) {
                float v[4];
                io::load4_smem(rb + i, v);
                *reinterpret_cast<float4 *>(fB + i) = make_float4(v[0], v[1], v[2], v[3]);
                if (kReadout) {
                    io::load4_smem(rc + i, v);
                    *reinterpret_cast<float4 *>(fC + i) = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
        } else {
            for (int i = tid; i < T * NSP; i += TPB) {
                const int r = i / NSP, n = i % NSP;
                const bool ok = r < rows && n < N;
                fB[i] = ok ? io::load_smem(rb + r * N + n) : 0.f;
                if (kReadout) fC[i] = ok ? io::load_smem(rc + r * N + n) : 0.f;
            }
        }
        vblock_sync<TPB, MODE>(vb);
        if (active) {
            const int col = grp * CPL;
            // this lane's rows of the tiles start at step q, its B/C slice at state q NS
            const IO *su = st + col + q * ROW, *sd = st + Lay::TILE + col + q * ROW;
            const IO *sz = st + 2 * Lay::TILE + col + q * ROW;
            const float *fBq = fB + q * NS, *fCq = fC + q * NS;
            IO *poq = po ? po + (b * L + tc + q) * Dm + dfirst : nullptr;
            // KSTEP steps at a time.  The per-step scalar work (softplus,
            // Delta u, skip, gate, store) of step r0 + j G + q is done once, by
            // lane q, for the group's CPL channels; Delta, Delta u and the
            // partial readouts travel between the lanes by shuffles.  Rows past
            // the end of the sequence were zero-filled by the copy and get
            // Delta = 0 (decay 1, no input): the state passes through them.
            // Full chunks take an unrolled copy of the block in which nrows is
            // the constant T (no row tests, immediate shared-memory offsets).
            auto step_block = [&](const int r0, const int nrows) {
                float uvo[KG][CPL], dlo[KG][CPL], duo[KG][CPL];
#pragma unroll
                for (int j = 0; j < KG; ++j) {
                    const int rr = r0 + j * G;  // this lane's step is rr + q
                    load_vals<IO, CPL>(su + rr * ROW, uvo[j]);
                    load_vals<IO, CPL>(sd + rr * ROW, dlo[j]);
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) dlo[j][cc] += bias[cc];
                }
                if (args.softplus) {
                    if (!PRECISE && CPL == 2) {
#pragma unroll
                        for (int j = 0; j < KG; ++j) {
                            const float2 sp = softplus2_fast(make_float2(dlo[j][0], dlo[j][CPL - 1]));
                            dlo[j][0] = sp.x;
                            dlo[j][CPL - 1] = sp.y;
                        }
                    } else if (!PRECISE && KG % 2 == 0) {
#pragma unroll
                        for (int j = 0; j < KG; j += 2) {
                            const float2 sp = softplus2_fast(make_float2(dlo[j][0], dlo[j + 1][0]));
                            dlo[j][0] = sp.x;
                            dlo[j + 1][0] = sp.y;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < KG; ++j)
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) dlo[j][cc] = softplus<PRECISE>(dlo[j][cc]);
                    }
                }
#pragma unroll
                for (int j = 0; j < KG; ++j) {
                    const bool ok = r0 + j * G + q < nrows;
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) {
                        if (!ok) dlo[j][cc] = 0.f;
                        duo[j][cc] = dlo[j][cc] * uvo[j][cc];
                    }
                }
                float dl[KSTEP][CPL], du[KSTEP][CPL], y[KSTEP][CPL];
                exchange_steps_cpl<KSTEP, G, CPL, LS>(dlo, duo, dl, du);
                if (MODE == kCkpt) {
                    // the block in pieces of the checkpoint spacing, each
                    // preceded by the store of the state entering it (step
                    // tc + rs, a multiple of the spacing); pieces past the
                    // end of the sequence store nothing
                    constexpr int KC = kCkptEvery;
#pragma unroll
                    for (int hb = 0; hb < KSTEP / KC; ++hb) {
                        const int rs = r0 + hb * KC;
                        if (rs < nrows) {
                            float *cp = ck_base + ((tc + rs) / KC) * ck_stride;
#pragma unroll
                            for (int p = 0; p < NS / 2; ++p) {
                                if (q * NS + 2 * p < N) cp[2 * p] = h2[0][p].x;
                                if (q * NS + 2 * p + 1 < N) cp[2 * p + 1] = h2[0][p].y;
                            }
                        }
                        float yp[KC][CPL];
                        recur_block_cpl<KC, NS, CPL, PRECISE, ZOH, false, SSM_POLY_PAIRS>(
                            *reinterpret_cast<const float(*)[KC][CPL]>(&dl[hb * KC]),
                            *reinterpret_cast<const float(*)[KC][CPL]>(&du[hb * KC]), fBq + rs * NSP,
                            fCq + rs * NSP, NSP, A2, h2, yp, invA2);
                    }
                } else {
                    recur_block_cpl<KSTEP, NS, CPL, PRECISE, ZOH, kReadout,
                                    MODE == kSegAgg ? SSM_SEGAGG_POLY_PAIRS : SSM_POLY_PAIRS>(
                        dl, du, fBq + r0 * NSP, fCq + r0 * NSP, NSP, A2, h2, y, invA2);
                }
                if (MODE == kCkpt) {
                    // no readout
                } else if (MODE == kSegAgg) {
#pragma unroll
                    for (int j = 0; j < KG; ++j)
#pragma unroll
                        for (int cc = 0; cc < CPL; ++cc) dsum[cc] += (double)dlo[j][cc];
                } else {
                    float yo[KG][CPL];
                    reduce_scatter_steps_cpl<KSTEP, G, CPL, LS>(y, yo, q);
#pragma unroll
                    for (int j = 0; j < KG; ++j) {
                        const int rr = r0 + j * G;
                        if (rr + q < nrows) {
                            float yy[CPL], zz[CPL];
#pragma unroll
                            for (int cc = 0; cc < CPL; ++cc) yy[cc] = fmaf(dskip[cc], uvo[j][cc], yo[j][cc]);
                            if (pz) {
                                load_vals<IO, CPL>(sz + rr * ROW, zz);
#pragma unroll
                                for (int cc = 0; cc < CPL; ++cc) yy[cc] *= silu<PRECISE>(zz[cc]);
                            }
                            store_vals<IO, CPL>(poq + (int64_t)rr * Dm, yy);
                        }
                    }
                }
            };
            if (rows == T) {
                SSM_UNROLL_N(SSM_R0_UNROLL)
                for (int r0 = 0; r0 < T; r0 += KSTEP) step_block(r0, T);
            } else {
                for (int r0 = 0; r0 < rows; r0 += KSTEP) step_block(r0, rows);
            }
        }
        vblock_sync<TPB, MODE>(vb);  // stage c % S and the fp32 B/C buffers are free again
    }
    cp_async_wait<0>();
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const double ds = MODE == kSegAgg ? group_sum_d<G, LS>(dsum[c]) : 0.0;
        float h[NS];
#pragma unroll
        for (int p = 0; p < NS / 2; ++p) {
            h[2 * p] = h2[c][p].x;
            h[2 * p + 1] = h2[c][p].y;
        }
        lane_finish<NS, MODE>(args, LaneRef{b, dfirst + c, q, active}, seg, t_end, h, ds);
    }
}

// Threads of a virtual block of the one-pass scan, by lanes per channel.
// Measured on B200 (Gelem/s; 1.4B layer = 32,768 channels, 130M layer =
// 12,288 channels): two lanes per channel in 64-thread virtual blocks, seven
// per CTA, 164.6 at the 1.4B layer with 16-step blocks, 167.5-167.9 with
// 8-step blocks (one lane: 156.7 in one-warp virtual blocks, 155.9 in
// 128-thread blocks); four lanes in 128-thread blocks, one per CTA, 122.6 at
// the 130M layer, 125-130 once a channel's lanes sat 8 apart (packed three per
// CTA: 113.6; 32- or 64-thread virtual blocks: 104-108, each re-widening the
// B/C rows for fewer channels).
#ifndef SSM_VB_THREADS_G1
#define SSM_VB_THREADS_G1 128
#endif
#ifndef SSM_VB_THREADS_G2
#define SSM_VB_THREADS_G2 64
#endif
#ifndef SSM_VB_THREADS_G4
#define SSM_VB_THREADS_G4 128
#endif
template <int G>
struct SlabTPB {
    static constexpr int value = G == 1 ? SSM_VB_THREADS_G1 : (G == 2 ? SSM_VB_THREADS_G2 : SSM_VB_THREADS_G4);
};

// SM count and opt-in shared memory of the current device (cached per device).
inline cudaError_t staged_device_limits(int *sms, int *smem_optin) {
    static std::atomic<int> cache_sms[64], cache_smem[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int slot = dev & 63;
    int s = cache_sms[slot].load(std::memory_order_relaxed), m = cache_smem[slot].load(std::memory_order_relaxed);
    if (s <= 0 || m <= 0) {
        e = cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&m, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        cache_sms[slot].store(s, std::memory_order_relaxed);
        cache_smem[slot].store(m, std::memory_order_relaxed);
    }
    *sms = s;
    *smem_optin = m;
    return cudaSuccess;
}

// Launches the staged kernel over `units` (batch row, channel tile) units and
// `nseg` sequence segments (grid y).  The one-pass mode (kFull) packs
// ceil(units / SMs) virtual blocks into each CTA (as far as threads, shared
// memory and hardware barriers allow), so that every SM receives the same
// number of units up to one; the other modes run one virtual block per CTA.
template <typename IO, int NS, int G, int CPL, int MODE, bool ZOH, int TPB>
inline cudaError_t launch_mode(ScanArgs a, int64_t units, unsigned nseg, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    using Lay = StagedLayout<IO, NS, G, CPL, TPB>;
    auto kern = scan_fwd_staged_kernel<IO, NS, G, CPL, P, MODE, ZOH, TPB>;
    int sms = 0, optin = 0;
    cudaError_t e = staged_device_limits(&sms, &optin);
    if (e != cudaSuccess) return e;
    int vmax = StagedMaxThreads<G, NS, CPL, MODE>::value / TPB;
#ifdef SSM_VPB_MAX
    if (vmax > SSM_VPB_MAX) vmax = SSM_VPB_MAX;
#endif
    if (G == 4) vmax = 1;  // one block per unit measured faster for four lanes (see SSM_VB_THREADS_G*)
    if (TPB > 32 && vmax > 15) vmax = 15;  // hardware barriers 1..15
    if ((size_t)vmax * Lay::SMEM > (size_t)optin) vmax = (int)((size_t)optin / Lay::SMEM);
    if (MODE != kFull && MODE != kCkpt) vmax = 1;
    if (vmax < 1) return cudaErrorInvalidConfiguration;
    // the shared-memory opt-in is a per-device function attribute: set it once per device
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(vmax * Lay::SMEM));
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return e;
        }
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    // one CTA per SM with all units resident at once; when the units do not
    // fit that way, CTAs of several units would spread unevenly over the SMs,
    // so one unit per CTA is launched instead
    int64_t vpb = (units + sms - 1) / sms;
    if (vpb > vmax) vpb = 1;
    if (vpb < 1) vpb = 1;
    const int64_t gx = (units + vpb - 1) / vpb;
    if (gx > 2147483647LL) return cudaErrorInvalidConfiguration;
    a.units = units;
    // An ordinary launch: as a programmatic dependent (launch overlapping the
    // previous kernel's end) the 130M layer's 384 blocks, which leave free
    // block slots, were placed unevenly over the SMs and ran 18 % slower
    // (106 against 130 Gelem/s); the 1.4B layer gained 0.3 %.
    kern<<<dim3((unsigned)gx, nseg), (unsigned)(vpb * TPB), vpb * Lay::SMEM, st>>>(a);
    return cudaGetLastError();
}

template <typename IO, int NS, int G, int CPL, bool ZOH>
inline cudaError_t launch_z(const ScanArgs &a, int variant, cudaStream_t st) {
    constexpr int TPBS = SlabTPB<G>::value;
    constexpr int CPBS = StagedLayout<IO, NS, G, CPL, TPBS>::CPB;
    constexpr int CPB = StagedLayout<IO, NS, G, CPL>::CPB;
    const int64_t units = a.batch * ((a.dim + CPB - 1) / CPB);
    if (variant == kVariantSlab)
        return launch_mode<IO, NS, G, CPL, kFull, ZOH, TPBS>(a, a.batch * ((a.dim + CPBS - 1) / CPBS), 1, st);
    if (variant == kVariantCkpt) {
        if (CPL != 1 || ZOH) return cudaErrorInvalidConfiguration;
        constexpr int CPBC = StagedLayout<IO, NS, G, 1, TPBS>::CPB;
        return launch_mode<IO, NS, G, 1, kCkpt, false, TPBS>(a, a.batch * ((a.dim + CPBC - 1) / CPBC), 1, st);
    }
    cudaError_t e = launch_mode<IO, NS, G, CPL, kSegAgg, ZOH, kBlock>(a, units, (unsigned)(a.nseg - 1), st);
    if (e != cudaSuccess) return e;
    return launch_mode<IO, NS, G, CPL, kSegFinal, ZOH, kBlock>(a, units, (unsigned)a.nseg, st);
}

// Exact ZOH on B is built for one channel per lane only.
template <typename IO, int NS, int G, int CPL>
inline cudaError_t launch_t(const ScanArgs &a, int variant, cudaStream_t st) {
    if (!a.zoh_b) return launch_z<IO, NS, G, CPL, false>(a, variant, st);
    if (CPL != 1) return cudaErrorInvalidConfiguration;
    return launch_z<IO, NS, G, 1, true>(a, variant, st);
}

// Launchers of the staged kernel for one lane count G (all state slices NS
// of that G, one or two channels per lane), one translation unit per (I/O
// type, G) so that the kernel's many instantiations compile in parallel.
cudaError_t launch_staged_g1_bf16(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);
cudaError_t launch_staged_g1_f32(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);
cudaError_t launch_staged_g2_bf16(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);
cudaError_t launch_staged_g2_f32(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);
cudaError_t launch_staged_g4_bf16(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);
cudaError_t launch_staged_g4_f32(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st);

// The (NS, G) layouts with lane count G, for one channel-per-lane count.
template <typename IO, int G, int CPL>
cudaError_t launch_layouts(const ScanArgs &a, int ns, int variant, cudaStream_t st) {
    if constexpr (G == 1) {
        if (ns == 4) return launch_t<IO, 4, 1, CPL>(a, variant, st);
        if (ns == 8) return launch_t<IO, 8, 1, CPL>(a, variant, st);
        if (ns == 16) return launch_t<IO, 16, 1, CPL>(a, variant, st);
    } else if constexpr (G == 2) {
        if (ns == 8) return launch_t<IO, 8, 2, CPL>(a, variant, st);
        if (ns == 16) return launch_t<IO, 16, 2, CPL>(a, variant, st);
    } else if constexpr (G == 4) {
        if (ns == 4) return launch_t<IO, 4, 4, CPL>(a, variant, st);
        if (ns == 8) return launch_t<IO, 8, 4, CPL>(a, variant, st);
        if (ns == 16) return launch_t<IO, 16, 4, CPL>(a, variant, st);
    }
    return cudaErrorInvalidConfiguration;
}

}  // namespace ssm
