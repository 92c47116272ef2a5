// state_update_bulk.cu -- the decode step with the state moved by TMA bulk
// copies (sm_100a).
//
// Same arithmetic as state_update.cu (NL-345 Mamba translation, section 1
// "Fast training and inference": constant time and memory per generated
// token; section 2 eq. (2) for one t):
//     h_n <- exp(dt A_n) h_n + dt B_n x;   y = sum_n C_n h_n + D x;
//     out = y * silu(z)
// The step reads and writes the whole fp32 state and does little arithmetic,
// so what sets its speed is how many bytes are in flight.  With one 16-byte
// load per thread, a fully occupied SM keeps 32 KB in flight, short of what
// HBM needs.  Here the work moves in units: the 16 KB of state of 4096 / N
// consecutive channels of one batch row, with those channels' x, dt, z and
// the row's B and C.
//   * One thread per CTA issues the unit's cp.async.bulk copies (TMA, one
//     per array) into a ring of kStages shared-memory buffers, kAhead units
//     ahead; they complete on the buffer's mbarrier (transaction bytes).
//   * Each thread updates its 4-state slices of the unit in registers and
//     writes them straight back to global memory (16-byte streaming stores;
//     a warp's 32 slices are 512 contiguous bytes); the lanes of a channel
//     sum their partial y with shuffles and the first writes out.  A warp
//     arrives on the buffer's "empty" mbarrier once it has read the buffer,
//     and the refill waits for all warps' arrivals: no CTA-wide barrier per
//     unit.
//   * A CTA takes a contiguous run of units in chunk-major order (consecutive
//     units cover the same channels of successive batch rows), so A and D stay
//     in registers and are reloaded only when the channel chunk changes.
//   * The kernel is launched as a programmatic dependent of the stream's
//     previous kernel (griddepcontrol): one decode step's launch and set-up
//     overlap the end of the step before it, and its global accesses wait
//     for that step's writes.
// The grid is persistent: up to three 256-thread CTAs per SM.  Every wait on
// an mbarrier gives up after 200 ms (read from the global timer) and sets bit
// 0 of a device status word; the warp that saw it (the answer is made
// warp-uniform) leaves its loop, and the thread that issues the loads first
// lets the loads it issued land (each wait again bounded); the host reads
// the word with ssm_get_device_status.
#include <atomic>
#include <utility>

#include "scan_kernels.cuh"

namespace ssm {

__device__ unsigned int g_device_status;

namespace {

// Programmatic dependent launch (sm_90 and later): the kernel may be launched
// before the stream's previous kernel has finished, so that its launch and
// CTA set-up overlap that kernel's end.  grid_dependency_wait() returns once
// the previous kernel has completed and its writes are visible, and then lets
// the next dependent launch begin.
#ifndef SSM_PDL
#define SSM_PDL 1
#endif
__device__ __forceinline__ void grid_dependency_wait() {
#if SSM_PDL
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
#endif
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = SSM_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#ifndef SSM_DECODE_STAGES
#define SSM_DECODE_STAGES 4
#endif
#ifndef SSM_DECODE_AHEAD
#define SSM_DECODE_AHEAD 2
#endif
#ifndef SSM_DECODE_UNIT_FLOATS
#define SSM_DECODE_UNIT_FLOATS 4096
#endif
#ifndef SSM_DECODE_CTAS
#define SSM_DECODE_CTAS 3
#endif
constexpr int kThreads = 256;
constexpr int kStages = SSM_DECODE_STAGES;
constexpr int kAhead = SSM_DECODE_AHEAD;          // units loaded ahead of the one being updated
constexpr int kUnitFloats = SSM_DECODE_UNIT_FLOATS;  // 16 KB of state per unit
constexpr int kSlices = kUnitFloats / 4;
constexpr int kPerThread = kSlices / kThreads;
constexpr int kCtasPerSm = SSM_DECODE_CTAS;
constexpr unsigned long long kWaitNs = 200000000ull;  // a wait gives up after 200 ms
static_assert(kAhead < kStages, "a buffer must be free before it is refilled");

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}
// Waits for the phase with the given parity to complete; false after kWaitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0 && global_ns() - t0 > kWaitNs) return false;
    }
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Shared-memory layout of one stage: the unit's state, then x, dt and z
// for its channels, then the batch row's B and C.
template <typename IO, int N>
struct BulkStage {
    static constexpr int CH = kUnitFloats / N;                       // channels per unit
    static constexpr size_t STATE = (size_t)kUnitFloats * 4;
    static constexpr size_t VEC = (size_t)CH * sizeof(IO);           // one per-channel array
    static constexpr size_t ROW = (size_t)N * sizeof(IO);            // one B or C row
    static constexpr size_t X = STATE, DT = X + VEC, Z = DT + VEC, B = Z + VEC, C = B + ROW;
    static constexpr size_t BYTES = (C + ROW + 127) / 128 * 128;
    static_assert(VEC % 16 == 0 && ROW % 16 == 0, "bulk copies move multiples of 16 bytes");
};

template <typename IO, int G4, bool PRECISE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
state_update_bulk_kernel(const DecodeArgs args, int64_t chunks, int64_t total_units, uint32_t missing_bytes) {
    using io = io_traits<IO>;
    constexpr int N = 4 * G4;                 // states per channel
    constexpr int kWarps = kThreads / 32;
    using SL = BulkStage<IO, N>;
    constexpr int CH = SL::CH;
    extern __shared__ __align__(128) unsigned char smem[];  // [kStages][SL::BYTES]
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];

    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t Dm = args.dim, Bt = args.batch;
    const IO *pz = static_cast<const IO *>(args.z);
    IO *pout = static_cast<IO *>(args.out);
    // this CTA's units: a contiguous run, chunk-major (unit u = chunk u / batch,
    // batch row u % batch), so that consecutive units share A and D
    const int64_t per = (total_units + gridDim.x - 1) / gridDim.x;
    const int64_t u0 = (int64_t)blockIdx.x * per;
    const int64_t mine = u0 < total_units ? (total_units - u0 < per ? total_units - u0 : per) : 0;

    if (tid == 0) {
#pragma unroll
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], kWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    // Launched as a programmatic dependent of the stream's previous kernel:
    // the set-up above may overlap that kernel's end, but nothing in global
    // memory is read or written before it has completed and its writes are
    // visible (the previous decode step's state, for one).  Once every CTA of
    // this grid runs, the next step's launch may begin (its CTAs take the
    // SMs as these exit and wait in turn).
    grid_dependency_wait();

    auto geom = [&](int64_t k, int64_t &b, int64_t &c0, int &nch) {
        const int64_t u = u0 + k;
        b = u % Bt;
        c0 = (u / Bt) * CH;
        nch = (int)(Dm - c0 < CH ? Dm - c0 : CH);
    };
    auto issue = [&](int64_t k) {  // thread 0
        int64_t b, c0;
        int nch;
        geom(k, b, c0, nch);
        unsigned char *stg = smem + (size_t)(k % kStages) * SL::BYTES;
        uint64_t *bar = &full[k % kStages];
        const uint32_t sb = (uint32_t)nch * N * 4, vb = (uint32_t)nch * sizeof(IO), rb = (uint32_t)SL::ROW;
        const int64_t ch = b * Dm + c0;
        mbar_arrive_expect_tx(bar, sb + vb * (pz ? 3 : 2) + 2 * rb + missing_bytes);
        bulk_load(stg, args.state + ch * N, sb, bar);
        bulk_load(stg + SL::X, static_cast<const IO *>(args.x) + ch, vb, bar);
        bulk_load(stg + SL::DT, static_cast<const IO *>(args.dt) + ch, vb, bar);
        if (pz) bulk_load(stg + SL::Z, pz + ch, vb, bar);
        bulk_load(stg + SL::B, static_cast<const IO *>(args.B) + b * N, rb, bar);
        bulk_load(stg + SL::C, static_cast<const IO *>(args.C) + b * N, rb, bar);
    };
    int64_t issued = 0;  // thread 0: units whose loads were issued
    if (tid == 0)
        for (; issued < kAhead && issued < mine; ++issued) issue(issued);

    float4 av[kPerThread];
    float dv[kPerThread];
    int64_t a_chunk = -1;
    bool abort = false;
    int64_t k = 0;
    for (; k < mine; ++k) {
        if (tid == 0 && k + kAhead < mine) {
            // the buffer being refilled last held unit k + kAhead - kStages:
            // every warp has arrived once it had read that unit
            const int64_t j = k + kAhead;
            if (j >= kStages && !mbar_wait_bounded(&empty[j % kStages], (uint32_t)((j / kStages - 1) & 1))) {
                atomicOr(&g_device_status, 1u);
                abort = true;
            } else {
                issue(j);
                issued = j + 1;
            }
        }
        int64_t b, c0;
        int nch;
        geom(k, b, c0, nch);
        if (c0 != a_chunk) {  // A and D of this chunk's channels
            a_chunk = c0;
#pragma unroll
            for (int i = 0; i < kPerThread; ++i) {
                const int sl = tid + i * kThreads;
                const int c = sl / G4, q = sl % G4;
                const bool ok = c < nch;
                av[i] = ok ? __ldg(reinterpret_cast<const float4 *>(args.A + (c0 + c) * N + q * 4))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
                dv[i] = (ok && args.Dskip) ? __ldg(args.Dskip + c0 + c) : 0.f;
            }
        }
        const int st = (int)(k % kStages);
        if (!abort && !mbar_wait_bounded(&full[st], (uint32_t)((k / kStages) & 1))) {
            atomicOr(&g_device_status, 1u);
            abort = true;
        }
        if (__any_sync(0xffffffffu, abort)) {  // the whole warp leaves together
            abort = true;
            break;
        }
        unsigned char *stg = smem + (size_t)st * SL::BYTES;
        float4 *unit = reinterpret_cast<float4 *>(stg);
        const IO *sx = reinterpret_cast<const IO *>(stg + SL::X);
        const IO *sdt = reinterpret_cast<const IO *>(stg + SL::DT);
        const IO *szz = reinterpret_cast<const IO *>(stg + SL::Z);
        const IO *sB = reinterpret_cast<const IO *>(stg + SL::B);
        const IO *sC = reinterpret_cast<const IO *>(stg + SL::C);
        const int64_t ch = b * Dm + c0;
#pragma unroll
        for (int i = 0; i < kPerThread; ++i) {
            const int sl = tid + i * kThreads;
            const int c = sl / G4, q = sl % G4;
            const bool ok = c < nch;
            const int cc = ok ? c : 0;
            float bv[4], cv[4];
            io::load4_smem(sB + q * 4, bv);
            io::load4_smem(sC + q * 4, cv);
            const float4 h4 = unit[sl];
            float h[4] = {h4.x, h4.y, h4.z, h4.w};
            const float a[4] = {av[i].x, av[i].y, av[i].z, av[i].w};
            const float xv = io::load_smem(sx + cc), dl = io::load_smem(sdt + cc), dx = dl * xv;
            float y = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                h[e] = fmaf(decay<PRECISE>(dl, scale_A<PRECISE>(a[e])), h[e], dx * bv[e]);
                y = fmaf(cv[e], h[e], y);
            }
            y = group_sum<G4>(y);
            if (ok) {
                __stcs(reinterpret_cast<float4 *>(args.state + (ch + c) * N + q * 4), make_float4(h[0], h[1], h[2], h[3]));
                if (q == 0) {
                    y = fmaf(dv[i], xv, y);
                    if (pz) y *= silu<PRECISE>(io::load_smem(szz + c));
                    io::store(pout + ch + c, y);
                }
            }
        }
        // this warp is done reading the buffer
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (tid == 0 && abort) {
        // let the loads already issued land before the buffers go away
        for (int64_t j = k; j < issued; ++j)
            (void)mbar_wait_bounded(&full[j % kStages], (uint32_t)((j / kStages) & 1));
    }
    // no warp leaves while loads it did not wait for may still be landing
    __syncthreads();
}

template <typename IO, int G4>
cudaError_t launch_g(const DecodeArgs &a, uint32_t missing_bytes, cudaStream_t st) {
    constexpr bool P = std::is_same<IO, float>::value;
    using SL = BulkStage<IO, 4 * G4>;
    constexpr size_t smem = (size_t)kStages * SL::BYTES;
    auto kern = state_update_bulk_kernel<IO, G4, P>;
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    const int64_t chunks = (a.dim + SL::CH - 1) / SL::CH;
    const int64_t total = a.batch * chunks;
    const int64_t grid = total < (int64_t)sms * kCtasPerSm ? total : (int64_t)sms * kCtasPerSm;
    return launch_dependent(kern, dim3((unsigned)grid), dim3(kThreads), smem, st, a, chunks, total, missing_bytes);
}

template <typename IO>
cudaError_t launch_io(const DecodeArgs &a, uint32_t missing_bytes, cudaStream_t st) {
    switch (a.dstate) {
        case 4:  // a 4-state row of B or C is 8 bytes in bf16: not a bulk-copy size
            if constexpr (sizeof(IO) == 4) return launch_g<IO, 1>(a, missing_bytes, st);
            return cudaErrorInvalidConfiguration;
        case 8: return launch_g<IO, 2>(a, missing_bytes, st);
        case 16: return launch_g<IO, 4>(a, missing_bytes, st);
        case 32: return launch_g<IO, 8>(a, missing_bytes, st);
        case 64: return launch_g<IO, 16>(a, missing_bytes, st);
    }
    return cudaErrorInvalidConfiguration;
}

}  // namespace

unsigned int read_and_clear_device_status(cudaStream_t st, cudaError_t *err) {
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *err = e;
    return v;
}

cudaError_t device_status_address(unsigned int **p) {
    return cudaGetSymbolAddress(reinterpret_cast<void **>(p), g_device_status);
}

bool state_update_bulk_eligible(const DecodeArgs &a, bool bf16) {
    const size_t es = bf16 ? 2 : 4;
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) % 16) == 0; };
    const int n = a.dstate;
    // every bulk copy starts on a 16-byte boundary and moves a multiple of 16
    // bytes: the per-channel rows (dim elements) and the B/C rows (dstate
    // elements) must be multiples of 16 bytes
    return (n == 4 || n == 8 || n == 16 || n == 32 || n == 64) && (a.dim * es) % 16 == 0 &&
           (n * es) % 16 == 0 && al(a.state) && al(a.A) && al(a.x) && al(a.dt) && al(a.B) && al(a.C) &&
           al(a.out) && (a.z == nullptr || al(a.z));
}

cudaError_t launch_state_update_bulk(const DecodeArgs &a, bool bf16, uint32_t missing_bytes, cudaStream_t st) {
    return bf16 ? launch_io<__nv_bfloat16>(a, missing_bytes, st) : launch_io<float>(a, missing_bytes, st);
}

}  // namespace ssm
