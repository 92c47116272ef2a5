// scan_common.cuh -- per-lane pieces shared by the scan kernels: the lane's
// slice of A and D, the initial state (h_0, or the carry folded from earlier
// segments), and the final write of the state or the segment aggregate.
#pragma once

#include "scan_kernels.cuh"

namespace ssm {

// Cooperative-group geometry of a scan block: G lanes per channel.
template <int G>
struct LaneGeom {
    static constexpr int CPB = kBlock / G;  // channels per block
    int q;                                   // lane within the channel group
    int ch;                                  // channel within the block
    int64_t b, d;                            // batch row, channel
    bool active;
    __device__ LaneGeom(const ScanArgs &a) {
        q = threadIdx.x % G;
        ch = threadIdx.x / G;
        const int64_t tiles = (a.dim + CPB - 1) / CPB;
        b = blockIdx.x / tiles;
        d = (blockIdx.x % tiles) * CPB + ch;
        active = d < a.dim;
    }
};

// One lane's share of one channel: batch row b, channel d, state slice q.
struct LaneRef {
    int64_t b, d;
    int q;
    bool active;
};

template <int G>
__device__ __forceinline__ LaneRef lane_ref(const LaneGeom<G> &g) {
    return LaneRef{g.b, g.d, g.q, g.active};
}

// A (pre-scaled for the decay tier) and the initial state of this lane.
template <int NS, bool PRECISE, int MODE>
__device__ __forceinline__ void lane_init(const ScanArgs &a, const LaneRef &g, int seg,
                                          float (&Aw)[NS], float (&h)[NS]) {
    const int N = a.dstate;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int n = g.q * NS + i;
        const bool ok = g.active && n < N;
        Aw[i] = ok ? scale_A<PRECISE>(a.A[g.d * N + n]) : 0.f;
        h[i] = 0.f;
    }
    if (!g.active) return;
    const int64_t soff = (g.b * a.dim + g.d) * N;
    if ((MODE == kFull || MODE == kCkpt) && a.last_state) {
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int n = g.q * NS + i;
            if (n < N) h[i] = a.last_state[soff + n];
        }
    }
    // The split passes read h_0 from last_state only in segment 0 of the first
    // pass, which copies it to the workspace: the last segment of the second
    // pass overwrites last_state while other segments may still be starting.
    if (MODE == kSegAgg && seg == 0 && a.last_state) {
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int n = g.q * NS + i;
            if (n < N) a.seg_h0[soff + n] = a.last_state[soff + n];
        }
    }
    if (MODE == kSegFinal) {
        if (a.last_state) {
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const int n = g.q * NS + i;
                if (n < N) h[i] = a.seg_h0[soff + n];
            }
        }
        // carry-in: left fold of the earlier segments' (P, h_loc) with
        // (P1, h1) o (P2, h2) = (P1 P2, P2 h1 + h2), applied to h_0
        for (int s = 0; s < seg; ++s) {
            const int64_t agg = (g.b * a.nseg + s) * a.dim + g.d;
            const float dsum = a.seg_dsum[agg];
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const int n = g.q * NS + i;
                if (n < N) h[i] = fmaf(decay<PRECISE>(dsum, Aw[i]), h[i], a.seg_h[agg * N + n]);
            }
        }
    }
}

// Final state (one pass, or the last segment) or the segment aggregate.
template <int NS, int MODE>
__device__ __forceinline__ void lane_finish(const ScanArgs &a, const LaneRef &g, int seg,
                                            int64_t t_end, const float (&h)[NS], double dsum) {
    if (!g.active || MODE == kCkpt) return;
    const int N = a.dstate;
    if (MODE == kSegAgg) {
        const int64_t agg = (g.b * a.nseg + seg) * a.dim + g.d;
        if (g.q == 0) a.seg_dsum[agg] = (float)dsum;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int n = g.q * NS + i;
            if (n < N) a.seg_h[agg * N + n] = h[i];
        }
    } else if (a.last_state && t_end == a.seqlen) {
        const int64_t soff = (g.b * a.dim + g.d) * N;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int n = g.q * NS + i;
            if (n < N) a.last_state[soff + n] = h[i];
        }
    }
}

// One time step of one channel: discretise, recur, read out.  Returns this
// lane's partial y (its states only).  du = Delta * u.
template <int NS, bool PRECISE, bool ZOH = false>
__device__ __forceinline__ float lane_step(float dl, float du, const float *Bs, const float *Cs,
                                           const float (&Aw)[NS], float (&h)[NS]) {
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int i = 0; i < NS; i += 4) {
        const float4 bv = *reinterpret_cast<const float4 *>(Bs + i);
        const float4 cv = *reinterpret_cast<const float4 *>(Cs + i);
        const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
        const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float a = decay<PRECISE>(dl, Aw[i + k]);
            float bu = du * bb[k];
            if (ZOH) {
                // Aw is A (precise tier) or A log2(e) (fast tier)
                const float z = PRECISE ? dl * Aw[i + k] : dl * Aw[i + k] * kLn2;
                bu *= PRECISE ? zoh_phi_precise(z)
                              : (fabsf(z) < 0.0625f
                                     ? fmaf(fmaf(fmaf(fmaf(1.f / 120.f, z, 1.f / 24.f), z, 1.f / 6.f), z, 0.5f), z, 1.f)
                                     : (a - 1.f) / z);
            }
            h[i + k] = fmaf(a, h[i + k], bu);
            if (k & 1) y1 = fmaf(cc[k], h[i + k], y1);
            else y0 = fmaf(cc[k], h[i + k], y0);
        }
    }
    return y0 + y1;
}

// K consecutive time steps of one channel (this lane's NS states, NS a
// multiple of 4), with the per-step scalars Delta (dl) and Delta * u (du)
// already computed.  Step k reads B/C row k at Bs + k * stride and
// Cs + k * stride.  The states are handled in pairs (n, n + 1); in the fast
// tier the pair's products and fused multiply-adds are single f32x2
// instructions.  Returns this lane's partial y of each step.
template <int K, int NS, bool PRECISE>
__device__ __forceinline__ void recur_block(const float (&dl)[K], const float (&du)[K],
                                            const float *Bs, const float *Cs, int stride,
                                            const float2 (&A2)[NS / 2], float2 (&h2)[NS / 2],
                                            float (&y)[K]) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const float2 d2 = make_float2(dl[k], dl[k]);
        const float2 u2 = make_float2(du[k], du[k]);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NS / 4; ++j) {
            const float4 bv = *reinterpret_cast<const float4 *>(Bs + k * stride + 4 * j);
            const float4 cv = *reinterpret_cast<const float4 *>(Cs + k * stride + 4 * j);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int p = 2 * j + hlf;
                const float2 b2 = hlf ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y);
                const float2 c2 = hlf ? make_float2(cv.z, cv.w) : make_float2(cv.x, cv.y);
                if (!PRECISE) {
                    // fast tier: the state pairs on f32x2 (half the issue slots)
                    const float2 x2 = mul2(d2, A2[p]);
                    const float2 a2 = make_float2(decay_of<PRECISE>(x2.x), decay_of<PRECISE>(x2.y));
                    h2[p] = fma2(a2, h2[p], mul2(u2, b2));
                    acc = fma2(c2, h2[p], acc);
                } else {
                    const float ax = decay_of<PRECISE>(d2.x * A2[p].x), ay = decay_of<PRECISE>(d2.y * A2[p].y);
                    h2[p].x = fmaf(ax, h2[p].x, u2.x * b2.x);
                    h2[p].y = fmaf(ay, h2[p].y, u2.y * b2.y);
                    acc.x = fmaf(c2.x, h2[p].x, acc.x);
                    acc.y = fmaf(c2.y, h2[p].y, acc.y);
                }
            }
        }
        y[k] = acc.x + acc.y;
    }
}

// The same for a lane that holds NS states of each of CPL channels: step k's
// B and C values are read once and used for every channel.
template <int K, int NS, int CPL, bool PRECISE, bool ZOH = false, bool READOUT = true,
          int POLY = SSM_POLY_PAIRS>
__device__ __forceinline__ void recur_block_cpl(const float (&dl)[K][CPL], const float (&du)[K][CPL],
                                                const float *Bs, const float *Cs, int stride,
                                                const float2 (&A2)[CPL][NS / 2],
                                                float2 (&h2)[CPL][NS / 2], float (&y)[K][CPL],
                                                const float2 (*invA2)[NS / 2] = nullptr) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
        float2 d2[CPL], u2[CPL], acc[CPL], id2[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            d2[c] = make_float2(dl[k][c], dl[k][c]);
            u2[c] = make_float2(du[k][c], du[k][c]);
            acc[c] = make_float2(0.f, 0.f);
            if (ZOH && !PRECISE) {
                const float inv = rcp_approx(dl[k][c]);
                id2[c] = make_float2(inv, inv);
            }
        }
#pragma unroll
        for (int j = 0; j < NS / 4; ++j) {
            const float4 bv = *reinterpret_cast<const float4 *>(Bs + k * stride + 4 * j);
            const float4 cv = READOUT ? *reinterpret_cast<const float4 *>(Cs + k * stride + 4 * j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const int p = 2 * j + hlf;
                const float2 b2 = hlf ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y);
                const float2 c2 = hlf ? make_float2(cv.z, cv.w) : make_float2(cv.x, cv.y);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    if (!PRECISE) {
                        const float2 x2 = mul2(d2[c], A2[c][p]);
                        const float2 a2 = poly_pair<POLY>(p) ? exp2_poly2(x2)
                                                       : make_float2(decay_of<PRECISE>(x2.x), decay_of<PRECISE>(x2.y));
                        float2 bu = mul2(u2[c], b2);
                        if (ZOH)
                            bu = mul2(bu, zoh_phi2(mul2(x2, make_float2(kLn2, kLn2)), a2, invA2[c][p], id2[c]));
                        h2[c][p] = fma2(a2, h2[c][p], bu);
                        if (READOUT) acc[c] = fma2(c2, h2[c][p], acc[c]);
                    } else {
                        const float zx = d2[c].x * A2[c][p].x, zy = d2[c].y * A2[c][p].y;
                        const float ax = decay_of<PRECISE>(zx), ay = decay_of<PRECISE>(zy);
                        float bx = u2[c].x * b2.x, by = u2[c].y * b2.y;
                        if (ZOH) {
                            bx *= zoh_phi_precise(zx);
                            by *= zoh_phi_precise(zy);
                        }
                        h2[c][p].x = fmaf(ax, h2[c][p].x, bx);
                        h2[c][p].y = fmaf(ay, h2[c][p].y, by);
                        if (READOUT) {
                            acc[c].x = fmaf(c2.x, h2[c][p].x, acc[c].x);
                            acc[c].y = fmaf(c2.y, h2[c][p].y, acc[c].y);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) y[k][c] = acc[c].x + acc[c].y;
    }
}

// exchange_steps / reduce_scatter_steps for CPL channels per lane.
template <int K, int G, int CPL, int STRIDE = 1>
__device__ __forceinline__ void exchange_steps_cpl(const float (&dlo)[K / G][CPL],
                                                   const float (&duo)[K / G][CPL],
                                                   float (&dl)[K][CPL], float (&du)[K][CPL]) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        float a[K / G], bo[K / G], x[K], z[K];
#pragma unroll
        for (int j = 0; j < K / G; ++j) { a[j] = dlo[j][c]; bo[j] = duo[j][c]; }
        exchange_steps<K, G, STRIDE>(a, bo, x, z);
#pragma unroll
        for (int k = 0; k < K; ++k) { dl[k][c] = x[k]; du[k][c] = z[k]; }
    }
}

template <int K, int G, int CPL, int STRIDE = 1>
__device__ __forceinline__ void reduce_scatter_steps_cpl(const float (&y)[K][CPL], float (&yo)[K / G][CPL],
                                                         int q) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        float a[K], o[K / G];
#pragma unroll
        for (int k = 0; k < K; ++k) a[k] = y[k][c];
        reduce_scatter_steps<K, G, STRIDE>(a, o, q);
#pragma unroll
        for (int j = 0; j < K / G; ++j) yo[j][c] = o[j];
    }
}

}  // namespace ssm
