// ssd_fwd.cu -- Mamba-2's SSD layer (structured state space duality) on the
// sm_100a tensor cores.
//
// What it computes ("Transformers are SSMs" review, nubint.ai, 提案手法): the
// selective SSM with one scalar A per head, so that the sequence map is a
// semiseparable matrix; for every (batch b, head h), with chunks of Q = 128
// tokens and the head's Delta_t = softplus(dt + dt_bias):
//   * the quadratic (attention-like) form inside a chunk:
//       Y_diag = (Lmask o (C B^T)) diag(Delta) X,
//       Lmask[t, s] = exp(A (S_t - S_s)) for s <= t, else 0,  S = cumsum(Delta);
//   * the linear (recurrent) form between chunks, through the state H
//     (headdim x dstate) carried in registers from chunk to chunk:
//       Y_off = diag(exp(A S_t)) C H_prev^T,
//       H     = exp(A S_end) H_prev + X^T diag(w) B,  w_s = exp(A (S_end - S_s)) Delta_s
//   * out = (Y_diag + Y_off + D_h X) * silu(Z).
// This is the review's block decomposition of the semiseparable matrix:
// diagonal blocks by the quadratic form, off-diagonal blocks by the carried
// state.  Four GEMMs per chunk and head run as tcgen05.mma with bf16
// operands in shared memory and fp32 accumulators in tensor memory:
//   C B^T      (128 x 128, K = dstate)    -> masked in registers
//   M X        (128 x headdim, K = 128)
//   C H^T      (128 x headdim, K = dstate)
//   B^T Xw     (dstate x headdim, K = 128)
// Three of them take two-term operands -- a bf16 high part plus the bf16
// rounding of the rest -- so that the result keeps fp32-level accuracy:
// Xw = w o X (one bf16 term would leave ~3e-3 relative error in the state),
// the carried state H in C H^T, and the masked matrix M (one bf16 term each
// measured 2.4e-2 output error on the full workload, above the 2e-2 bound).
// Tiles of C, B, X come in by TMA (cp.async.bulk.tensor, 128-byte swizzle,
// no multicast), two chunks deep.  One CTA of 512 threads per (b, h):
// thread (warp w, lane l) owns TMEM lane / tile row r = 32 (w % 4) + l and the
// quarter w / 4 of the columns; thread 0 issues the copies and the MMAs.
// Every wait is bounded; a wait that runs out sets bit 1 of the device
// status word and the CTA stops after its in-flight work.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "scan_kernels.cuh"
#include "ssm_device.cuh"
#include "umma.cuh"

namespace ssm {

namespace {

using namespace umma;

constexpr int kQ = 128;         // tokens per chunk
constexpr int kP = 64;          // head dimension (one 128-byte swizzled row of bf16)
constexpr uint32_t kTileBytes = kQ * 128;  // 128 rows x 128 bytes
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

// TMEM columns (fp32): C B^T, Y_diag, Y_off, chunk state
constexpr uint32_t kColCB = 0, kColY = 128, kColYoff = 192, kColS = 256, kTmemCols = 512;

struct SsdArgs {
    const void *dt;
    const float *A, *D, *dt_bias;
    float *state;  // (batch, heads, headdim, dstate) in/out, or null
    int64_t batch, seqlen, heads, groups;
    int dstate;    // 64 or 128
    int softplus;
    int has_z;
    unsigned int *status;
};


// Eight bf16 values of one 16-byte piece of a swizzled tile row.
__device__ __forceinline__ void load_piece(const unsigned char *tile, int row, int piece, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4 *>(tile + sw128_offset(row, piece));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}
__device__ __forceinline__ void store_piece(unsigned char *tile, int row, int piece, const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + sw128_offset(row, piece)) = w;
}

// ---------------------------------------------------------------------------
// The tiles of chunk c + 1 (C, B, X; two stages) are copied while chunk c
// computes, the masked intra-chunk matrix M stays in tensor memory as the A
// operand of M X (no shared-memory round trip), and z / out move between
// registers and global memory directly, so that the double buffers fit in
// shared memory.  Inside a chunk the products and the element-wise phases
// overlap: C B^T and C H^T run while the threads form w o X; B^T (w o X)
// runs while they mask C B^T; M X runs while they update the carried state.
enum Tile2 { kC0s0, kC1s0, kB0s0, kB1s0, kXs0, kC0s1, kC1s1, kB0s1, kB1s1, kXs1, kXh2, kXl2, kH2, kHl2,
             kNumTiles2 };
constexpr uint32_t kSmemBytes2 = kNumTiles2 * kTileBytes + 1024;
constexpr int kThreads2 = 512;   // 16 warps: four per scheduler to hide latency
constexpr uint32_t kColM = 320;  // M as the A operand, high part: 64 columns (two bf16 per column)
constexpr uint32_t kColMl = 384; // low part

// The carried state's two-term copy (this thread's 16 of the 64 channels of
// state row r): pieces 2 part and 2 part + 1 of the row.
__device__ __forceinline__ void store_state_split16(unsigned char *hi, unsigned char *lo, int r, int part,
                                                    const float (&H)[16]) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        float vh[8], vl[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            vh[i] = __bfloat162float(__float2bfloat16_rn(H[8 * j + i]));
            vl[i] = H[8 * j + i] - vh[i];
        }
        store_piece(hi, r, 2 * part + j, vh);
        store_piece(lo, r, 2 * part + j, vl);
    }
}

// Thread (warp w, lane l) owns TMEM lane / tile row r = 32 (w % 4) + l and
// the quarter part = w / 4 of the columns: channels [16 part, 16 part + 16)
// of the head, mask columns [32 part, 32 part + 32).
__global__ void __launch_bounds__(kThreads2, 1)
ssd_fwd_pipelined_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                         const __grid_constant__ CUtensorMap mapC, const __nv_bfloat16 *__restrict__ zg,
                         __nv_bfloat16 *__restrict__ og, const SsdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~static_cast<uintptr_t>(1023));
    auto tile = [&](int i) { return sm + (uint32_t)i * kTileBytes; };
    __shared__ uint64_t bar_ld[2], bar_mma1, bar_mma2, bar_mma3;
    __shared__ uint32_t s_tmem;
    __shared__ float s_dl[kQ], s_cum[kQ], s_wsum[16];
    __shared__ __align__(16) float s_q[kQ];  // A S_s - log2(Delta_s), log2 units (+inf where Delta_s = 0)
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const int64_t b = blockIdx.x / a.heads, h = blockIdx.x % a.heads;
    const int g = (int)(h / (a.heads / a.groups));
    const int N = a.dstate;
    const int ntiles = N / 64, ksteps = N / 16;
    const int64_t L = a.seqlen;
    const float Ah = a.A[h] * kLog2e;
    const float Dh = a.D ? a.D[h] : 0.f;
    const float bias = a.dt_bias ? a.dt_bias[h] : 0.f;
    const __nv_bfloat16 *dt = static_cast<const __nv_bfloat16 *>(a.dt);

    if (tid == 0) {
        mbar_init(&bar_ld[0], 1);
        mbar_init(&bar_ld[1], 1);
        mbar_init(&bar_mma1, 1);
        mbar_init(&bar_mma2, 1);
        mbar_init(&bar_mma3, 1);
        mbar_fence_init();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = s_tmem;
    const uint32_t tlane = tm + ((uint32_t)(quad * 32) << 16);
    const int nchunks = (int)((L + kQ - 1) / kQ);

    auto issue = [&](int cc) {  // thread 0: the tiles of chunk cc into stage cc & 1
        const int st = cc & 1;
        const int base = st ? kC0s1 : kC0s0;
        mbar_expect_tx(&bar_ld[st], (uint32_t)(2 * ntiles + 1) * kTileBytes);
        const int32_t t0 = cc * kQ;
        for (int kt = 0; kt < ntiles; ++kt) {
            tma_load_3d(tile(base + kt), &mapC, g * N + 64 * kt, t0, (int32_t)b, &bar_ld[st]);
            tma_load_3d(tile(base + 2 + kt), &mapB, g * N + 64 * kt, t0, (int32_t)b, &bar_ld[st]);
        }
        tma_load_3d(tile(base + 4), &mapX, (int32_t)(h * kP), t0, (int32_t)b, &bar_ld[st]);
    };
    if (tid == 0 && nchunks > 0) issue(0);

    // carried state H[n = r][p = 16 part + i], fp32
    float H[16];
    const bool nrow = r < N;
    const int64_t sbase = ((b * a.heads + h) * kP + 16 * part) * N + r;
#pragma unroll
    for (int i = 0; i < 16; ++i) H[i] = (a.state && nrow) ? a.state[sbase + (int64_t)i * N] : 0.f;
    store_state_split16(tile(kH2), tile(kHl2), r, part, H);
    fence_proxy_async();
    __syncthreads();

    auto wait = [&](uint64_t *bar, uint32_t par) {
        if (!mbar_wait(bar, par, kWaitNs)) {
            atomicOr(a.status, 2u);
            s_abort = 1;
        }
    };

    // z (this thread's 16 channels of row r) and dt of chunk cc, into registers
    uint4 zn[2];
    float dtn = 0.f;
    auto prefetch = [&](int cc) {
        const int64_t t = (int64_t)cc * kQ + r;
        const bool ok = cc < nchunks && t < L;
        const int64_t gr = ((b * L + t) * a.heads + h) * kP + 16 * part;
#pragma unroll
        for (int j = 0; j < 2; ++j)
            zn[j] = (zg && ok) ? __ldg(reinterpret_cast<const uint4 *>(zg + gr) + j) : make_uint4(0, 0, 0, 0);
        dtn = ok ? __bfloat162float(dt[(b * L + t) * a.heads + h]) : 0.f;
    };
    prefetch(0);

    int c = 0;
    for (; c < nchunks; ++c) {
        const int st = c & 1;
        const int64_t t0 = (int64_t)c * kQ;
        const int64_t trow = t0 + r;
        const bool valid = trow < L;
        const int tC0 = st ? kC0s1 : kC0s0, tB0 = tC0 + 2, tX = tC0 + 4;
        // 1. the next chunk's tiles into the other stage (its last readers,
        // the previous chunk's products and threads, are done)
        if (tid == 0 && c + 1 < nchunks) issue(c + 1);
        // 2. this chunk's z and dt (prefetched a chunk ahead); Delta and its
        // running sum over the chunk
        const uint4 zr0 = zn[0], zr1 = zn[1];
        const float dt_raw = dtn;
        const int64_t grow = ((b * L + trow) * a.heads + h) * kP + 16 * part;
        prefetch(c + 1);
        float dl = 0.f;
        if (valid) {
            const float sv = dt_raw + bias;
            dl = a.softplus ? softplus<false>(sv) : sv;
        }
        float cum = dl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, cum, o);
            if (lane >= o) cum += v;
        }
        if (lane == 31) s_wsum[warp] = cum;
        __syncthreads();
        for (int w2 = 0; w2 < quad; ++w2) cum += s_wsum[4 * part + w2];
        if (part == 0) {
            s_dl[r] = dl;
            s_cum[r] = cum;
            s_q[r] = dl > 0.f ? fmaf(Ah, cum, -lg2_approx(dl)) : __int_as_float(0x7f800000);
        }
        wait(&bar_ld[st], (uint32_t)(c >> 1) & 1u);
        __syncthreads();
        if (s_abort) break;
        const float cum_end = s_cum[kQ - 1];

        // 3. C B^T and C H_prev^T (two-term state copy)
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_cb = idesc_bf16(128, 128, kMajorK, kMajorK);
            const uint32_t id_yo = idesc_bf16(128, kP, kMajorK, kMajorMN);
            for (int k = 0; k < ksteps; ++k) {
                const uint64_t ad = desc_sw128(smem_u32(tile(tC0 + k / 4)) + (k % 4) * 32, 16, 1024);
                const uint64_t bd = desc_sw128(smem_u32(tile(tB0 + k / 4)) + (k % 4) * 32, 16, 1024);
                mma_bf16(tm + kColCB, ad, bd, id_cb, k > 0);
            }
            for (int hp = 0; hp < 2; ++hp)
                for (int k = 0; k < ksteps; ++k) {
                    const uint64_t ad = desc_sw128(smem_u32(tile(tC0 + k / 4)) + (k % 4) * 32, 16, 1024);
                    const uint64_t bd = desc_sw128(smem_u32(tile(hp ? kHl2 : kH2)) + k * 2048, 16, 1024);
                    mma_bf16(tm + kColYoff, ad, bd, id_yo, hp > 0 || k > 0);
                }
            mma_commit(&bar_mma1);
        }
        // 4. w o X as bf16 high and low parts, w_s = exp(A (S_end - S_s)) Delta_s
        {
            const float w = ex2_approx(Ah * (cum_end - cum)) * dl;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float x8[8], hi[8], lo[8];
                load_piece(tile(tX), r, 2 * part + j, x8);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float xw = w * x8[i];
                    hi[i] = __bfloat162float(__float2bfloat16_rn(xw));
                    lo[i] = xw - hi[i];
                }
                store_piece(tile(kXh2), r, 2 * part + j, hi);
                store_piece(tile(kXl2), r, 2 * part + j, lo);
            }
        }
        fence_proxy_async();
        __syncthreads();
        // 5. chunk state B^T (w o X)
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_s = idesc_bf16(128, kP, kMajorMN, kMajorMN);
            for (int xp = 0; xp < 2; ++xp)
                for (int k = 0; k < kQ / 16; ++k) {
                    const uint64_t ad = desc_sw128(smem_u32(tile(tB0)) + k * 2048, kTileBytes, 1024);
                    const uint64_t bd = desc_sw128(smem_u32(tile(xp ? kXl2 : kXh2)) + k * 2048, 16, 1024);
                    mma_bf16(tm + kColS, ad, bd, id_s, xp > 0 || k > 0);
                }
            mma_commit(&bar_mma2);
        }
        // 6. M[t, s] = CB[t, s] exp(A (S_t - S_s)) Delta_s for row t = r and the
        // 32 columns of this part, as bf16 high and low parts in tensor memory:
        // CB 2^(p_t - q_s), p_t = A S_t, q_s = A S_s - log2(Delta_s) when Delta
        // is a softplus (>= 0), the product form otherwise; a block of columns
        // above the diagonal for the whole warp is zero without arithmetic.
        wait(&bar_mma1, (uint32_t)c & 1u);
        fence_after_sync();
        {
            const int sb = 32 * part;
            uint32_t mh[16], ml[16];
            if (sb > quad * 32 + 31) {
#pragma unroll
                for (int i = 0; i < 16; ++i) mh[i] = ml[i] = 0u;
            } else {
                const float pt = Ah * cum;
                float cb[32];
                tmem_ld32(tlane + kColCB + sb, cb);
                tmem_wait_ld();
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    const float4 q4 = *reinterpret_cast<const float4 *>(s_q + sb + 4 * i4);
                    const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
                    float m[4], mhf[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s0 = sb + 4 * i4 + e;
                        const float f = a.softplus ? ex2_approx(pt - qv[e])
                                                   : ex2_approx(Ah * (cum - s_cum[s0])) * s_dl[s0];
                        m[e] = s0 <= r ? cb[4 * i4 + e] * f : 0.f;
                        mhf[e] = __bfloat162float(__float2bfloat16_rn(m[e]));
                    }
                    mh[2 * i4] = pack_bf16x2(mhf[0], mhf[1]);
                    mh[2 * i4 + 1] = pack_bf16x2(mhf[2], mhf[3]);
                    ml[2 * i4] = pack_bf16x2(m[0] - mhf[0], m[1] - mhf[1]);
                    ml[2 * i4 + 1] = pack_bf16x2(m[2] - mhf[2], m[3] - mhf[3]);
                }
            }
            tmem_st16(tlane + kColM + 16 * part, mh);
            tmem_st16(tlane + kColMl + 16 * part, ml);
            tmem_wait_st();
        }
        fence_before_sync();
        __syncthreads();
        if (s_abort) break;
        // 7. Y_diag = M X with both parts of M read from tensor memory
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_y = idesc_bf16(128, kP, kMajorK, kMajorMN);
            for (int mp = 0; mp < 2; ++mp)
                for (int k = 0; k < kQ / 16; ++k) {
                    const uint64_t bd = desc_sw128(smem_u32(tile(tX)) + k * 2048, 16, 1024);
                    mma_bf16_ts(tm + kColY, tm + (mp ? kColMl : kColM) + 8 * k, bd, id_y, mp > 0 || k > 0);
                }
            mma_commit(&bar_mma3);
        }
        // 8. carried state: H = exp(A S_end) H + B^T (w o X), and its copy for the next chunk
        wait(&bar_mma2, (uint32_t)c & 1u);
        fence_after_sync();
        {
            float sv[16];
            tmem_ld16(tlane + kColS + 16 * part, sv);
            tmem_wait_ld();
            const float gdec = ex2_approx(Ah * cum_end);
#pragma unroll
            for (int i = 0; i < 16; ++i) H[i] = fmaf(gdec, H[i], sv[i]);
            store_state_split16(tile(kH2), tile(kHl2), r, part, H);
        }
        // 9. out = (Y_diag + exp(A S_t) Y_off + D X) silu(z), straight to global memory
        wait(&bar_mma3, (uint32_t)c & 1u);
        fence_after_sync();
        {
            float yd[16], yo[16];
            tmem_ld16(tlane + kColY + 16 * part, yd);
            tmem_ld16(tlane + kColYoff + 16 * part, yo);
            tmem_wait_ld();
            const float et = ex2_approx(Ah * cum);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float x8[8];
                load_piece(tile(tX), r, 2 * part + j, x8);
                const uint4 zq = j ? zr1 : zr0;
                const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
                uint32_t ow[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float y0 = fmaf(Dh, x8[2 * i], fmaf(et, yo[8 * j + 2 * i], yd[8 * j + 2 * i]));
                    float y1 = fmaf(Dh, x8[2 * i + 1], fmaf(et, yo[8 * j + 2 * i + 1], yd[8 * j + 2 * i + 1]));
                    if (zg) {
                        y0 *= silu<false>(__uint_as_float(zw[i] << 16));
                        y1 *= silu<false>(__uint_as_float(zw[i] & 0xffff0000u));
                    }
                    ow[i] = pack_bf16x2(y0, y1);
                }
                if (valid) reinterpret_cast<uint4 *>(og + grow)[j] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (s_abort) break;
    }
    if (s_abort) {
        // let whatever was issued finish (bounded) before the memory goes away
        (void)mbar_wait(&bar_ld[c & 1], (uint32_t)(c >> 1) & 1u, kWaitNs);
        if (c + 1 < nchunks) (void)mbar_wait(&bar_ld[(c + 1) & 1], (uint32_t)((c + 1) >> 1) & 1u, kWaitNs);
        (void)mbar_wait(&bar_mma1, (uint32_t)c & 1u, kWaitNs);
        (void)mbar_wait(&bar_mma2, (uint32_t)c & 1u, kWaitNs);
        (void)mbar_wait(&bar_mma3, (uint32_t)c & 1u, kWaitNs);
    } else if (a.state && nrow) {
#pragma unroll
        for (int i = 0; i < 16; ++i) a.state[sbase + (int64_t)i * N] = H[i];
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, kTmemCols);
}

}  // namespace
}  // namespace ssm

namespace ssm {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, fetched through the runtime (no link-time
// dependency on the driver library).
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            return (EncodeTiledFn) nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// A (batch, seqlen, width) bf16 tensor as a 3-D tiled map: boxes of 64
// elements of the width x 128 steps x 1 row, 128-byte swizzle; steps past
// the sequence read as zeros and are not written by stores.
bool encode_btw(CUtensorMap *m, const void *p, int64_t batch, int64_t seqlen, int64_t width) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)seqlen, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)(width * seqlen) * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kQ, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(p), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool ssd_fwd_supported(const SsdFwdArgs &a) {
    auto al = [](const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) % 16) == 0; };
    return a.headdim == kP && (a.dstate == 64 || a.dstate == 128) && a.groups >= 1 && a.heads % a.groups == 0 &&
           al(a.x) && al(a.z) && al(a.B) && al(a.C) && al(a.out) && encode_fn() != nullptr;
}

cudaError_t launch_ssd_fwd(const SsdFwdArgs &a, cudaStream_t st) {
    if (!ssd_fwd_supported(a)) return cudaErrorNotSupported;
    CUtensorMap mx, mb, mc;
    const int64_t hp = a.heads * a.headdim, gn = a.groups * a.dstate;
    if (!encode_btw(&mx, a.x, a.batch, a.seqlen, hp) || !encode_btw(&mb, a.B, a.batch, a.seqlen, gn) ||
        !encode_btw(&mc, a.C, a.batch, a.seqlen, gn))
        return cudaErrorInvalidValue;
    SsdArgs k{};
    k.dt = a.dt;
    k.A = a.A;
    k.D = a.D;
    k.dt_bias = a.dt_bias;
    k.state = a.state;
    k.batch = a.batch;
    k.seqlen = a.seqlen;
    k.heads = a.heads;
    k.groups = a.groups;
    k.dstate = (int)a.dstate;
    k.softplus = a.softplus;
    k.has_z = a.z != nullptr;
    cudaError_t e = device_status_address(&k.status);
    if (e != cudaSuccess) return e;
    static bool configured[64] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!configured[dev & 63]) {
        e = cudaFuncSetAttribute(ssd_fwd_pipelined_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes2);
        if (e != cudaSuccess) return e;
        configured[dev & 63] = true;
    }
    const int64_t grid = a.batch * a.heads;
    if (grid > 2147483647LL) return cudaErrorInvalidConfiguration;
    ssd_fwd_pipelined_kernel<<<(unsigned)grid, kThreads2, kSmemBytes2, st>>>(
        mx, mb, mc, static_cast<const __nv_bfloat16 *>(a.z), static_cast<__nv_bfloat16 *>(a.out), k);
    return cudaGetLastError();
}

}  // namespace ssm
