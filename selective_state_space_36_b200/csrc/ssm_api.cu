// ssm_api.cu -- the C ABI declared in include/ssm.h: argument validation,
// choice of kernel variant and thread layout, launch, error reporting.
#include <cuda_runtime.h>
#include <stdarg.h>

#include <atomic>
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "../../include/ssm.h"
#include "scan_kernels.cuh"

namespace {

thread_local char g_last_error[512] = "";

// Decode kernel: 1 = bulk-copy kernel where eligible, 0 = per-slice loads only.
#ifndef SSM_DECODE_BULK
#define SSM_DECODE_BULK 1
#endif
constexpr bool kDecodeBulk = SSM_DECODE_BULK != 0;

// test hook: extra bytes every decode unit's wait expects (0 = none)
std::atomic<uint32_t> g_inject_wait_bytes{0};

ssm_status fail(ssm_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

ssm_status cuda_fail(cudaError_t e, const char *what) {
    // The CUDA runtime is shared with the caller (torch, for instance): leave
    // no error of ours behind for its next status check to trip over.
    (void)cudaGetLastError();
    return fail(SSM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool misaligned(const void *p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) != 0; }

constexpr int64_t kMaxDstate = 64;
constexpr int64_t kMaxGridX = 2147483647LL;

// 128-thread blocks per SM the sequence split aims for.
constexpr int kTargetBlocksPerSm = 8;

// Channels per lane of the staged kernel when the caller does not choose.
#ifndef SSM_DEFAULT_CPL
#define SSM_DEFAULT_CPL 1
#endif
constexpr int kDefaultStagedCpl = SSM_DEFAULT_CPL;

// Lanes per channel of the backward's checkpoint pass (0: the forward's choice).
#ifndef SSM_BWD_CKPT_LANES
#define SSM_BWD_CKPT_LANES 4
#endif

struct DeviceInfo {
    int sms = 148;
    int smem_optin = 227 * 1024;  // dynamic shared memory a block may opt in to
};

DeviceInfo device_info() {
    DeviceInfo di;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            di.sms = v;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && v > 0)
            di.smem_optin = v;
    }
    (void)cudaGetLastError();  // no device here is not an error of the caller's
    return di;
}

// Lanes per channel (G) and states per lane (NS) for the scan.  lanes_req
// (0 = automatic) is honoured where a kernel exists for it.
void scan_layout(int64_t dstate, int64_t channels, int sms, int lanes_req, int *ns, int *g) {
    if (dstate <= 4) { *ns = 4; *g = 1; return; }
    if (dstate <= 8) { *ns = 8; *g = 1; return; }
    if (dstate <= 16) {
        int G = lanes_req;
        if (G != 1 && G != 2 && G != 4) {
            // Below 1.5 blocks of 128 channels per SM, four lanes per channel
            // (4 states each) give the warps that hide latency.  From there
            // up to what one CTA per SM holds in 64-thread virtual blocks of
            // two lanes per channel (8 per CTA: 256 channels per SM), two
            // lanes: the 1.4B layer (32,768 channels) measured 165.3 Gelem/s
            // against 161.5 with one lane and 163.6 with four (the same box,
            // 16-step blocks; two lanes 167.9 with their 8-step blocks).
            // Beyond that, one lane per channel
            // (all 16 states, no shuffles) in 128-thread blocks.
            if (2 * channels < (int64_t)sms * ssm::kBlock * 3) G = 4;
            else if (channels <= (int64_t)sms * 256) G = 2;
            else G = 1;
        }
        *g = G;
        *ns = 16 / G;
        return;
    }
    if (dstate <= 32) {
        if (lanes_req == 4) { *ns = 8; *g = 4; } else { *ns = 16; *g = 2; }
        return;
    }
    *ns = 16;
    *g = 4;
}

// Workspaces (the split scan's carries, the backward's checkpoints) come from
// a stream-ordered pool per device that keeps freed memory (no release
// threshold): a repeated call reuses its workspace instead of having it
// mapped again after every synchronisation, as the device's default pool
// would.  The pool holds at most the largest workspace in use at once.
constexpr int kMaxPoolDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxPoolDevices] = {};

cudaError_t workspace_alloc(void **p, size_t bytes, cudaStream_t st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxPoolDevices) return cudaMallocAsync(p, bytes, st);
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_pool_mu);
        if (!g_pool[dev]) {
            cudaMemPoolProps props{};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t created = nullptr;
            e = cudaMemPoolCreate(&created, &props);
            if (e != cudaSuccess) return e;
            uint64_t keep = UINT64_MAX;
            e = cudaMemPoolSetAttribute(created, cudaMemPoolAttrReleaseThreshold, &keep);
            if (e != cudaSuccess) {
                (void)cudaMemPoolDestroy(created);
                return e;
            }
            g_pool[dev] = created;
        }
        pool = g_pool[dev];
    }
    return cudaMallocFromPoolAsync(p, bytes, pool, st);
}

ssm_status check_io(ssm_dtype io, size_t *elem) {
    if (io == SSM_F32) { *elem = 4; return SSM_OK; }
    if (io == SSM_BF16) { *elem = 2; return SSM_OK; }
    return fail(SSM_ERR_INVALID_ARG, "io dtype %d is not SSM_F32 or SSM_BF16", (int)io);
}

}  // namespace

extern "C" {

const char *ssm_status_string(ssm_status s) {
    switch (s) {
        case SSM_OK: return "ok";
        case SSM_ERR_INVALID_ARG: return "invalid argument";
        case SSM_ERR_UNSUPPORTED: return "unsupported";
        case SSM_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char *ssm_last_error(void) { return g_last_error; }

int ssm_version(void) { return 200; }

void ssm_get_build_info(ssm_build_info *info) {
    if (!info) return;
    memset(info, 0, sizeof(*info));
    info->sfu_decays_per_16 = 16 - 4 * SSM_POLY_PAIRS;
    info->split_pass1_sfu_decays_per_16 = 16 - 4 * SSM_SEGAGG_POLY_PAIRS;
}

}  // extern "C"

namespace {

// Everything a scan call decides before launching.
struct ScanPlan {
    int variant = SSM_VARIANT_SLAB;
    int ns = 16, g = 1, cpl = 1;
    int zoh_b = 0;
    int family = ssm::kFamilyGeneric;
    int nseg = 1;
    int64_t seg_len = 0;
    size_t ws_bytes = 0;
    int launches = 0;
};

// Validates sizes and options (not data pointers, which may be absent when
// only planning) and decides variant, layout, kernel family and segments.
ssm_status plan_scan(ssm_dims dims, ssm_dtype io, const void *u, const void *delta, const void *B,
                     const void *C, const void *z, const void *out, int delta_softplus,
                     const ssm_scan_opts *opts, ScanPlan *plan) {
    size_t es = 0;
    if (ssm_status s = check_io(io, &es)) return s;
    if (dims.batch < 0 || dims.seqlen < 0 || dims.dim < 0 || dims.dstate < 0)
        return fail(SSM_ERR_INVALID_ARG, "negative size (batch %lld, seqlen %lld, dim %lld, dstate %lld)",
                    (long long)dims.batch, (long long)dims.seqlen, (long long)dims.dim,
                    (long long)dims.dstate);
    if (dims.dstate < 1) return fail(SSM_ERR_INVALID_ARG, "dstate must be >= 1");
    if (dims.dstate > kMaxDstate)
        return fail(SSM_ERR_UNSUPPORTED, "dstate %lld > %lld", (long long)dims.dstate, (long long)kMaxDstate);
    if (delta_softplus != 0 && delta_softplus != 1)
        return fail(SSM_ERR_INVALID_ARG, "delta_softplus must be 0 or 1");
    int variant = opts ? opts->variant : SSM_VARIANT_AUTO;
    if (variant < SSM_VARIANT_AUTO || variant > SSM_VARIANT_SPLIT)
        return fail(SSM_ERR_INVALID_ARG, "unknown variant %d", variant);
    const int lanes_req = opts ? opts->lanes : 0;
    int family = opts ? opts->family : 0;
    const int cpl_req = opts ? opts->channels_per_lane : 0;
    const int disc = opts ? opts->discretization : SSM_DISCRETIZE_EULER_B;
    if (opts && (opts->reserved[0] || opts->reserved[1]))
        return fail(SSM_ERR_INVALID_ARG, "ssm_scan_opts.reserved must be zero");
    if (disc != SSM_DISCRETIZE_EULER_B && disc != SSM_DISCRETIZE_ZOH)
        return fail(SSM_ERR_INVALID_ARG, "discretization must be SSM_DISCRETIZE_EULER_B or SSM_DISCRETIZE_ZOH");
    if (disc == SSM_DISCRETIZE_ZOH && cpl_req == 2)
        return fail(SSM_ERR_UNSUPPORTED, "exact ZOH on B is built for one channel per lane");
    if (cpl_req != 0 && cpl_req != 1 && cpl_req != 2)
        return fail(SSM_ERR_INVALID_ARG, "channels per lane must be 0, 1 or 2");
    if (family < ssm::kFamilyAuto || family > ssm::kFamilyStaged)
        return fail(SSM_ERR_INVALID_ARG, "kernel family must be 0 (auto), 1 (generic) or 2 (staged)");
    if (lanes_req != 0 && lanes_req != 1 && lanes_req != 2 && lanes_req != 4)
        return fail(SSM_ERR_INVALID_ARG, "lanes per channel must be 0, 1, 2 or 4");
    if (opts && opts->segments < 0) return fail(SSM_ERR_INVALID_ARG, "segments must be >= 0");
    if (opts && opts->segments > 65535) return fail(SSM_ERR_INVALID_ARG, "at most 65535 segments");
    const int64_t channels = dims.batch * dims.dim;
    if (dims.batch != 0 && channels / dims.batch != dims.dim)
        return fail(SSM_ERR_INVALID_ARG, "batch * dim overflows");
    *plan = ScanPlan{};
    if (channels == 0 || dims.seqlen == 0) return SSM_OK;  // nothing to compute; state unchanged
    if (dims.seqlen > INT64_MAX / channels / dims.dstate)
        return fail(SSM_ERR_INVALID_ARG, "batch * seqlen * dim * dstate overflows");

    const DeviceInfo di = device_info();
    scan_layout(dims.dstate, channels, di.sms, lanes_req, &plan->ns, &plan->g);
    if (!ssm::scan_shape_supported(plan->ns, plan->g))
        return fail(SSM_ERR_UNSUPPORTED, "no kernel for %d states x %d lanes", plan->ns, plan->g);
    ssm::ScanArgs probe{};
    probe.u = u; probe.delta = delta; probe.z = z; probe.B = B; probe.C = C; probe.out = const_cast<void *>(out);
    probe.dim = dims.dim; probe.dstate = (int)dims.dstate;
    const bool eligible = ssm::staged_eligible(probe, (int)es);
    if (family == ssm::kFamilyStaged && !eligible)
        return fail(SSM_ERR_UNSUPPORTED, "staged kernel needs 16-byte aligned rows (dim and dstate "
                    "multiples of %d, 16-byte aligned u, delta, z, B, C, out)", (int)(16 / es));
    const int cpl_try = cpl_req ? cpl_req : (disc == SSM_DISCRETIZE_ZOH ? 1 : kDefaultStagedCpl);
    const bool fits = ssm::staged_smem_bytes(io == SSM_BF16, plan->ns, plan->g, cpl_try) <= (size_t)di.smem_optin;
    if (family == ssm::kFamilyStaged && !fits)
        return fail(SSM_ERR_UNSUPPORTED, "the staged kernel's shared memory for %d lanes x %d channels "
                    "exceeds the device's %d bytes", plan->g, cpl_try, di.smem_optin);
    if (family == ssm::kFamilyAuto) family = (eligible && fits) ? ssm::kFamilyStaged : ssm::kFamilyGeneric;
    plan->family = family;
    if (cpl_req == 2 && family != ssm::kFamilyStaged)
        return fail(SSM_ERR_UNSUPPORTED, "two channels per lane needs the staged kernel");
    plan->cpl = family == ssm::kFamilyStaged ? cpl_try : 1;
    plan->zoh_b = disc == SSM_DISCRETIZE_ZOH;
    const int64_t cpb = ssm::kBlock / plan->g * plan->cpl;
    const int64_t blocks = dims.batch * ((dims.dim + cpb - 1) / cpb);
    if (blocks > kMaxGridX) return fail(SSM_ERR_UNSUPPORTED, "grid too large");

    // Sequence split when the channel blocks alone leave SMs idle and the
    // sequence is long enough to amortise the second pass.
    int nseg = opts ? opts->segments : 0;
    const int64_t full = (int64_t)di.sms * kTargetBlocksPerSm;
    int64_t blocks_now = blocks;
    const int64_t blocks1 = dims.batch * ((dims.dim + ssm::kBlock * plan->cpl - 1) / (ssm::kBlock * plan->cpl));
    if (variant == SSM_VARIANT_AUTO)
        variant = (blocks1 < di.sms && dims.seqlen >= 4 * 1024) ? SSM_VARIANT_SPLIT : SSM_VARIANT_SLAB;
    // Segments, not extra lanes per channel, supply the parallelism of a
    // split, whether it was chosen or asked for (at L = 1,048,576, dim 1536:
    // one lane 15.21 ms per call, two lanes 15.48-16.03, four 19.83).
    if (variant == SSM_VARIANT_SPLIT && lanes_req == 0 && dims.dstate > 8 && dims.dstate <= 16) {
        plan->g = 1;
        plan->ns = 16;
        blocks_now = blocks1;
    }
    if (variant == SSM_VARIANT_SPLIT && nseg == 0) {
        int64_t sgm = (full + blocks_now - 1) / blocks_now;
        const int64_t max_by_len = (dims.seqlen + ssm::kChunk - 1) / ssm::kChunk;  // >= 1 chunk each
        if (sgm > max_by_len) sgm = max_by_len;
        if (sgm > 65535) sgm = 65535;
        nseg = (int)(sgm < 1 ? 1 : sgm);
    }
    plan->variant = SSM_VARIANT_SLAB;
    plan->nseg = 1;
    plan->seg_len = dims.seqlen;
    plan->launches = 1;
    if (variant == SSM_VARIANT_SPLIT && nseg > 1) {
        // even segments, each a whole number of chunks except the last
        int64_t seg_len = (dims.seqlen + nseg - 1) / nseg;
        seg_len = (seg_len + ssm::kChunk - 1) / ssm::kChunk * ssm::kChunk;
        nseg = (int)((dims.seqlen + seg_len - 1) / seg_len);
        if (nseg > 1) {
            plan->variant = SSM_VARIANT_SPLIT;
            plan->nseg = nseg;
            plan->seg_len = seg_len;
            plan->launches = 2;
            plan->ws_bytes = ((size_t)channels * dims.dstate * (1 + (size_t)nseg) +
                              (size_t)nseg * channels) * sizeof(float);
        }
    }
    return SSM_OK;
}

}  // namespace

extern "C" {

ssm_status ssm_scan_plan(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                         const void *B, const void *C, const void *z, const void *out,
                         const ssm_scan_opts *opts, ssm_scan_plan_info *info) {
    g_last_error[0] = 0;
    if (!info) return fail(SSM_ERR_INVALID_ARG, "info is required");
    ScanPlan p;
    if (ssm_status s = plan_scan(dims, io, u, delta, B, C, z, out, 0, opts, &p)) return s;
    memset(info, 0, sizeof(*info));
    info->variant = p.variant;
    info->segments = p.nseg;
    info->lanes = p.g;
    info->family = p.family;
    info->launches = p.launches;
    info->channels_per_lane = p.cpl;
    info->workspace_bytes = (int64_t)p.ws_bytes;
    return SSM_OK;
}

ssm_status ssm_selective_scan_fwd_ex(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, const float *delta_bias, int delta_softplus,
                                     void *out, float *last_state, const ssm_scan_opts *opts,
                                     ssm_stream stream) {
    g_last_error[0] = 0;
    ScanPlan p;
    if (ssm_status s = plan_scan(dims, io, u, delta, B, C, z, out, delta_softplus, opts, &p)) return s;
    if (p.launches == 0) return SSM_OK;  // empty problem
    const size_t es = io == SSM_BF16 ? 2 : 4;
    if (!u || !delta || !A || !B || !C || !out)
        return fail(SSM_ERR_INVALID_ARG, "u, delta, A, B, C and out are required");
    if (misaligned(u, es) || misaligned(delta, es) || misaligned(B, es) || misaligned(C, es) ||
        misaligned(z, es) || misaligned(out, es) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(delta_bias, 4) || misaligned(last_state, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");

    ssm::ScanArgs a{};
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.Dskip = D; a.bias = delta_bias;
    a.out = out; a.last_state = last_state;
    a.batch = dims.batch; a.seqlen = dims.seqlen; a.dim = dims.dim;
    a.dstate = (int)dims.dstate;
    a.softplus = delta_softplus;
    a.zoh_b = p.zoh_b;
    a.seg_len = p.seg_len;
    a.nseg = p.nseg;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    if (p.variant == SSM_VARIANT_SLAB) {
        cudaError_t e = ssm::launch_scan_fwd(a, io == SSM_BF16, p.ns, p.g, p.cpl, ssm::kVariantSlab, p.family, st);
        if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
        return SSM_OK;
    }
    void *ws = nullptr;
    cudaError_t e = workspace_alloc(&ws, p.ws_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    const size_t n_h0 = (size_t)dims.batch * dims.dim * dims.dstate;
    a.seg_h0 = static_cast<float *>(ws);
    a.seg_h = a.seg_h0 + n_h0;
    a.seg_dsum = a.seg_h + n_h0 * p.nseg;
    e = ssm::launch_scan_fwd(a, io == SSM_BF16, p.ns, p.g, p.cpl, ssm::kVariantSplit, p.family, st);
    cudaError_t ef = cudaFreeAsync(ws, st);
    if (e != cudaSuccess) return cuda_fail(e, "split scan launch");
    if (ef != cudaSuccess) return cuda_fail(ef, "workspace release");
    return SSM_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Sequence-split scan without any device allocation.
//
// The split scan needs a carry buffer (segment end states and Delta sums).
// ssm_selective_scan_fwd takes it from the workspace pool; this variant takes it
// from the fixed scratch array below, which the CUDA runtime places in device
// memory when the library's module is loaded on a GPU and keeps until the
// process exits.  Host code must not pass the array's name to a kernel (on the
// host it is only a shadow symbol): the device address is looked up with
// cudaGetSymbolAddress while the device is current, once per device and CUDA
// context -- a device reset (cudaDeviceReset) destroys the context and the
// module with it, so an address cached across it would be stale; the cache is
// keyed by the context's unique id and the lookup is repeated for a new one.
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)SSM_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct ScratchAddr {
    unsigned long long ctx_id = 0;  // 0: unknown (look up again)
    void *addr = nullptr;
};
ScratchAddr g_noalloc_addr[kMaxDevices];

// Unique id of the calling thread's current CUDA context (0 if there is none
// or the driver cannot say), through driver entry points fetched by the
// runtime, so the library needs no link-time dependency on the driver.
unsigned long long current_context_id() {
    using GetCurrent = int (*)(void **);
    using GetId = int (*)(void *, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
        (void)cudaGetLastError();
    });
    if (!get_current || !get_id) return 0;
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
    return id;
}

ssm_status noalloc_scratch_address(void **addr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(SSM_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    ScratchAddr &c = g_noalloc_addr[dev];
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || c.ctx_id != ctx || !c.addr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        c.addr = p;
        // the lookup makes the device's primary context current if it was not
        c.ctx_id = ctx ? ctx : current_context_id();
    }
    *addr = c.addr;
    return SSM_OK;
}

}  // namespace

extern "C" {

ssm_status ssm_selective_scan_fwd_noalloc(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                          const float *A, const void *B, const void *C, const float *D,
                                          const void *z, const float *delta_bias, int delta_softplus,
                                          void *out, float *last_state, int segments, ssm_stream stream) {
    g_last_error[0] = 0;
    if (segments < 0) return fail(SSM_ERR_INVALID_ARG, "segments must be >= 0");
    ssm_scan_opts o{};
    o.variant = SSM_VARIANT_SPLIT;
    o.segments = segments;
    ScanPlan p;
    if (ssm_status s = plan_scan(dims, io, u, delta, B, C, z, out, delta_softplus, &o, &p)) return s;
    if (p.launches == 0) return SSM_OK;  // empty problem
    if (p.ws_bytes > kNoAllocScratchBytes && segments == 0) {
        // Automatic segment count: the largest count whose carries fit the
        // scratch, found by bisection on the planner's own workspace size
        // (which grows with the count), so the two never disagree; when even
        // two segments do not fit, one pass runs, which needs no scratch.
        int lo = 1, hi = p.nseg;  // carries(lo) fit (one pass: none), carries(hi) do not
        while (hi - lo > 1) {
            const int mid = lo + (hi - lo) / 2;
            o.segments = mid;
            ScanPlan t;
            if (ssm_status s = plan_scan(dims, io, u, delta, B, C, z, out, delta_softplus, &o, &t)) return s;
            if (t.ws_bytes <= kNoAllocScratchBytes) lo = mid;
            else hi = mid;
        }
        if (lo >= 2) {
            o.segments = lo;
        } else {
            o.variant = SSM_VARIANT_SLAB;
            o.segments = 0;
        }
        if (ssm_status s = plan_scan(dims, io, u, delta, B, C, z, out, delta_softplus, &o, &p)) return s;
    }
    if (p.ws_bytes > kNoAllocScratchBytes)
        return fail(SSM_ERR_UNSUPPORTED, "the split needs %zu bytes of scratch but the static scratch holds %zu "
                    "(use fewer segments, a smaller batch * dim, or ssm_selective_scan_fwd)",
                    p.ws_bytes, kNoAllocScratchBytes);
    const size_t es = io == SSM_BF16 ? 2 : 4;
    if (!u || !delta || !A || !B || !C || !out)
        return fail(SSM_ERR_INVALID_ARG, "u, delta, A, B, C and out are required");
    if (misaligned(u, es) || misaligned(delta, es) || misaligned(B, es) || misaligned(C, es) ||
        misaligned(z, es) || misaligned(out, es) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(delta_bias, 4) || misaligned(last_state, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");

    ssm::ScanArgs a{};
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.Dskip = D; a.bias = delta_bias;
    a.out = out; a.last_state = last_state;
    a.batch = dims.batch; a.seqlen = dims.seqlen; a.dim = dims.dim;
    a.dstate = (int)dims.dstate;
    a.softplus = delta_softplus;
    a.seg_len = p.seg_len;
    a.nseg = p.nseg;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (p.variant == SSM_VARIANT_SLAB) {  // too short to split, or too wide for the scratch: one pass
        cudaError_t e = ssm::launch_scan_fwd(a, io == SSM_BF16, p.ns, p.g, p.cpl, ssm::kVariantSlab, p.family, st);
        if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
        return SSM_OK;
    }
    void *ws = nullptr;
    if (ssm_status s = noalloc_scratch_address(&ws)) return s;
    // Every scratch word the second pass reads is written by the first pass of
    // the same call (the h0 copy, and the aggregates of segments 0..nseg-2), so
    // nothing has to be cleared between calls.
    const size_t n_h0 = (size_t)dims.batch * dims.dim * dims.dstate;
    a.seg_h0 = static_cast<float *>(ws);
    a.seg_h = a.seg_h0 + n_h0;
    a.seg_dsum = a.seg_h + n_h0 * p.nseg;
    cudaError_t e = ssm::launch_scan_fwd(a, io == SSM_BF16, p.ns, p.g, p.cpl, ssm::kVariantSplit, p.family, st);
    if (e != cudaSuccess) return cuda_fail(e, "split scan launch");
    return SSM_OK;
}

ssm_status ssm_selective_scan_fwd(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                  const float *A, const void *B, const void *C, const float *D,
                                  const void *z, const float *delta_bias, int delta_softplus,
                                  void *out, float *last_state, ssm_stream stream) {
    return ssm_selective_scan_fwd_ex(dims, io, u, delta, A, B, C, D, z, delta_bias, delta_softplus,
                                     out, last_state, nullptr, stream);
}

ssm_status ssm_selective_scan_fwd_complex(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                          const float *A, const void *B, const void *C, const float *D,
                                          const void *z, const float *delta_bias, int delta_softplus,
                                          void *out, float *last_state, ssm_stream stream) {
    g_last_error[0] = 0;
    size_t es = 0;
    if (ssm_status s = check_io(io, &es)) return s;
    if (dims.batch < 0 || dims.seqlen < 0 || dims.dim < 0 || dims.dstate < 0)
        return fail(SSM_ERR_INVALID_ARG, "negative size (batch %lld, seqlen %lld, dim %lld, dstate %lld)",
                    (long long)dims.batch, (long long)dims.seqlen, (long long)dims.dim,
                    (long long)dims.dstate);
    if (dims.dstate < 1) return fail(SSM_ERR_INVALID_ARG, "dstate must be >= 1");
    if (dims.dstate > kMaxDstate)
        return fail(SSM_ERR_UNSUPPORTED, "dstate %lld > %lld", (long long)dims.dstate, (long long)kMaxDstate);
    if (delta_softplus != 0 && delta_softplus != 1)
        return fail(SSM_ERR_INVALID_ARG, "delta_softplus must be 0 or 1");
    const int64_t channels = dims.batch * dims.dim;
    if (dims.batch != 0 && channels / dims.batch != dims.dim)
        return fail(SSM_ERR_INVALID_ARG, "batch * dim overflows");
    if (channels != 0 && dims.seqlen > INT64_MAX / channels / (2 * dims.dstate))
        return fail(SSM_ERR_INVALID_ARG, "batch * seqlen * dim * dstate overflows");
    if (channels == 0 || dims.seqlen == 0) return SSM_OK;
    if (!u || !delta || !A || !B || !C || !out)
        return fail(SSM_ERR_INVALID_ARG, "u, delta, A, B, C and out are required");
    if (misaligned(u, es) || misaligned(delta, es) || misaligned(B, es) || misaligned(C, es) ||
        misaligned(z, es) || misaligned(out, es) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(delta_bias, 4) || misaligned(last_state, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
    const int64_t cpb = ssm::scan_complex_channels_per_block();
    if (dims.batch * ((dims.dim + cpb - 1) / cpb) > kMaxGridX)
        return fail(SSM_ERR_UNSUPPORTED, "grid too large");
    ssm::ScanArgs a{};
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.Dskip = D; a.bias = delta_bias;
    a.out = out; a.last_state = last_state;
    a.batch = dims.batch; a.seqlen = dims.seqlen; a.dim = dims.dim;
    a.dstate = (int)dims.dstate;
    a.softplus = delta_softplus;
    a.seg_len = dims.seqlen;
    a.nseg = 1;
    cudaError_t e = ssm::launch_scan_complex(a, io == SSM_BF16, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "complex scan launch");
    return SSM_OK;
}

ssm_status ssm_selective_scan_bwd_ex(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, const float *delta_bias, int delta_softplus,
                                     const float *h0, const void *dout, void *du, void *ddelta,
                                     void *dz, float *dA, float *dB, float *dC, float *dD,
                                     float *ddelta_bias, float *dh0, const ssm_scan_opts *opts,
                                     ssm_stream stream) {
    g_last_error[0] = 0;
    size_t es = 0;
    if (ssm_status s = check_io(io, &es)) return s;
    if (dims.batch < 0 || dims.seqlen < 0 || dims.dim < 0 || dims.dstate < 0)
        return fail(SSM_ERR_INVALID_ARG, "negative size (batch %lld, seqlen %lld, dim %lld, dstate %lld)",
                    (long long)dims.batch, (long long)dims.seqlen, (long long)dims.dim,
                    (long long)dims.dstate);
    if (dims.dstate < 1) return fail(SSM_ERR_INVALID_ARG, "dstate must be >= 1");
    if (dims.dstate > kMaxDstate)
        return fail(SSM_ERR_UNSUPPORTED, "dstate %lld > %lld", (long long)dims.dstate, (long long)kMaxDstate);
    if (delta_softplus != 0 && delta_softplus != 1)
        return fail(SSM_ERR_INVALID_ARG, "delta_softplus must be 0 or 1");
    int family = ssm::kFamilyAuto;
    if (opts) {
        if (opts->variant != SSM_VARIANT_AUTO || opts->segments != 0 || opts->lanes != 0 ||
            opts->channels_per_lane != 0 || opts->reserved[0] != 0 || opts->reserved[1] != 0)
            return fail(SSM_ERR_INVALID_ARG, "the backward scan takes only opts.family (other fields must be 0)");
        if (opts->discretization != SSM_DISCRETIZE_EULER_B)
            return fail(SSM_ERR_UNSUPPORTED, "the backward scan implements the Euler Bbar only");
        if (opts->family != SSM_KERNEL_AUTO && opts->family != SSM_KERNEL_GENERIC &&
            opts->family != SSM_KERNEL_STAGED)
            return fail(SSM_ERR_INVALID_ARG, "unknown kernel family %d", opts->family);
        family = opts->family;
    }
    const int64_t channels = dims.batch * dims.dim;
    if (dims.batch != 0 && channels / dims.batch != dims.dim)
        return fail(SSM_ERR_INVALID_ARG, "batch * dim overflows");
    if (dims.dim != 0 && dims.dstate != 0 && dims.dim > INT64_MAX / dims.dstate)
        return fail(SSM_ERR_INVALID_ARG, "dim * dstate overflows");
    if (channels != 0 && dims.seqlen > INT64_MAX / channels / dims.dstate)
        return fail(SSM_ERR_INVALID_ARG, "batch * seqlen * dim * dstate overflows");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool has_work = channels != 0 && dims.seqlen != 0;
    // Parameter gradients are sums: with no work they are zero.  dh0 of an
    // empty sequence is zero as well (the loss does not depend on h0).
    if (!has_work) {
        const size_t dn = (size_t)dims.dim * dims.dstate;
        const size_t hn = (size_t)channels * dims.dstate;
        struct Z { void *p; size_t n; } zs[] = {{dA, dn}, {dD, (size_t)dims.dim},
                                               {ddelta_bias, (size_t)dims.dim}, {dh0, hn}};
        for (const Z &zz : zs)
            if (zz.p && zz.n && misaligned(zz.p, 4))
                return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
        for (const Z &zz : zs) {
            if (!zz.p || zz.n == 0) continue;
            cudaError_t e = cudaMemsetAsync(zz.p, 0, zz.n * sizeof(float), st);
            if (e != cudaSuccess) return cuda_fail(e, "zeroing gradients");
        }
        return SSM_OK;
    }
    if (!u || !delta || !A || !B || !C || !dout || !du || !ddelta || !dA || !dB || !dC)
        return fail(SSM_ERR_INVALID_ARG, "u, delta, A, B, C, dout, du, ddelta, dA, dB and dC are required");
    if ((z != nullptr) != (dz != nullptr)) return fail(SSM_ERR_INVALID_ARG, "dz is required iff z is given");
    if ((D != nullptr) != (dD != nullptr)) return fail(SSM_ERR_INVALID_ARG, "dD is required iff D is given");
    if (misaligned(u, es) || misaligned(delta, es) || misaligned(B, es) || misaligned(C, es) ||
        misaligned(z, es) || misaligned(dout, es) || misaligned(du, es) || misaligned(ddelta, es) ||
        misaligned(dz, es) || misaligned(A, 4) || misaligned(D, 4) || misaligned(delta_bias, 4) ||
        misaligned(h0, 4) || misaligned(dA, 4) || misaligned(dB, 4) || misaligned(dC, 4) ||
        misaligned(dD, 4) || misaligned(ddelta_bias, 4) || misaligned(dh0, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
    const int64_t cpb = ssm::scan_bwd_channels_per_block();
    if (dims.batch * ((dims.dim + cpb - 1) / cpb) > kMaxGridX)
        return fail(SSM_ERR_UNSUPPORTED, "grid too large");

    ssm::ScanBwdArgs a{};
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z; a.dout = dout;
    a.A = A; a.Dskip = D; a.bias = delta_bias; a.h0 = h0;
    a.du = du; a.ddelta = ddelta; a.dz = dz;
    a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD; a.dbias = ddelta_bias; a.dh0 = dh0;
    a.batch = dims.batch; a.seqlen = dims.seqlen; a.dim = dims.dim;
    a.dstate = (int)dims.dstate;
    a.softplus = delta_softplus;
    a.vec_red = dims.dstate % 4 == 0 && !misaligned(dB, 16) && !misaligned(dC, 16);

    // staged pair (checkpointing forward pass + staged reverse pass) where
    // the rows allow it, else the generic single kernel
    const bool eligible = ssm::scan_bwd_staged_eligible(a, (int)es);
    if (family == ssm::kFamilyStaged && !eligible)
        return fail(SSM_ERR_UNSUPPORTED, "staged backward needs dstate <= 16 and 16-byte aligned rows "
                    "(dim and dstate times the element size multiples of 16, pointers 16-byte aligned)");
    const bool staged = eligible && family != ssm::kFamilyGeneric;
    int ns = 0, g = 0;
    if (staged) {
        const DeviceInfo di = device_info();
        // the checkpoint pass (8-step blocks, no readout) measured faster with
        // four lanes per channel than with one at the 1.4B-layer shape (a
        // whole backward call: 2.19 vs 2.49 ms)
        scan_layout(dims.dstate, channels, di.sms, SSM_BWD_CKPT_LANES, &ns, &g);
        if (ssm::staged_smem_bytes(io == SSM_BF16, ns, g, 1) > (size_t)di.smem_optin)
            return fail(SSM_ERR_UNSUPPORTED, "staged backward needs more shared memory than the device has");
    }

    const size_t bln = (size_t)dims.batch * dims.seqlen * dims.dstate;
    struct Z { void *p; size_t n; } zs[] = {{dA, (size_t)dims.dim * dims.dstate}, {dB, bln}, {dC, bln},
                                           {dD, (size_t)dims.dim}, {ddelta_bias, (size_t)dims.dim}};
    for (const Z &zz : zs) {
        if (!zz.p) continue;
        cudaError_t e = cudaMemsetAsync(zz.p, 0, zz.n * sizeof(float), st);
        if (e != cudaSuccess) return cuda_fail(e, "zeroing gradients");
    }
    const int64_t kc = staged ? ssm::scan_bwd_staged_chunk() : ssm::scan_bwd_chunk((int)dims.dstate);
    const size_t ws_bytes = (size_t)channels * ((dims.seqlen + kc - 1) / kc) * dims.dstate * sizeof(float);
    void *ws = nullptr;
    cudaError_t e = workspace_alloc(&ws, ws_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "checkpoint workspace allocation");
    a.ckpt = static_cast<float *>(ws);
    if (staged) {
        ssm::ScanArgs f{};
        f.u = u; f.delta = delta; f.B = B; f.C = C; f.z = nullptr;
        f.A = A; f.Dskip = nullptr; f.bias = delta_bias;
        f.out = nullptr;
        f.last_state = const_cast<float *>(h0);  // read as h_0, not written in checkpoint mode
        f.batch = dims.batch; f.seqlen = dims.seqlen; f.dim = dims.dim;
        f.dstate = (int)dims.dstate;
        f.softplus = delta_softplus;
        f.seg_len = dims.seqlen;
        f.nseg = 1;
        f.ckpt = a.ckpt;
        e = ssm::launch_scan_staged(f, io == SSM_BF16, ns, g, 1, ssm::kVariantCkpt, st);
        if (e == cudaSuccess) e = ssm::launch_scan_bwd_staged(a, io == SSM_BF16, st);
    } else {
        e = ssm::launch_scan_bwd(a, io == SSM_BF16, st);
    }
    cudaError_t ef = cudaFreeAsync(ws, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward scan launch");
    if (ef != cudaSuccess) return cuda_fail(ef, "workspace release");
    return SSM_OK;
}

ssm_status ssm_selective_scan_bwd(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                  const float *A, const void *B, const void *C, const float *D,
                                  const void *z, const float *delta_bias, int delta_softplus,
                                  const float *h0, const void *dout, void *du, void *ddelta,
                                  void *dz, float *dA, float *dB, float *dC, float *dD,
                                  float *ddelta_bias, float *dh0, ssm_stream stream) {
    return ssm_selective_scan_bwd_ex(dims, io, u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0,
                                     dout, du, ddelta, dz, dA, dB, dC, dD, ddelta_bias, dh0, nullptr,
                                     stream);
}

ssm_status ssm_selective_state_update(ssm_dims dims, ssm_dtype io, float *state, const void *x,
                                      const void *dt, const float *A, const void *B, const void *C,
                                      const float *D, const void *z, void *out, ssm_stream stream) {
    g_last_error[0] = 0;
    size_t es = 0;
    if (ssm_status s = check_io(io, &es)) return s;
    if (dims.batch < 0 || dims.dim < 0 || dims.dstate < 0)
        return fail(SSM_ERR_INVALID_ARG, "negative size");
    if (dims.dstate < 1) return fail(SSM_ERR_INVALID_ARG, "dstate must be >= 1");
    if (dims.dstate > kMaxDstate)
        return fail(SSM_ERR_UNSUPPORTED, "dstate %lld > %lld", (long long)dims.dstate, (long long)kMaxDstate);
    const int64_t channels = dims.batch * dims.dim;
    if (dims.batch != 0 && channels / dims.batch != dims.dim)
        return fail(SSM_ERR_INVALID_ARG, "batch * dim overflows");
    if (channels == 0) return SSM_OK;
    if (channels > INT64_MAX / dims.dstate) return fail(SSM_ERR_INVALID_ARG, "state size overflows");
    if (!state || !x || !dt || !A || !B || !C || !out)
        return fail(SSM_ERR_INVALID_ARG, "state, x, dt, A, B, C and out are required");
    if (misaligned(x, es) || misaligned(dt, es) || misaligned(B, es) || misaligned(C, es) ||
        misaligned(z, es) || misaligned(out, es) || misaligned(A, 4) || misaligned(D, 4) ||
        misaligned(state, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
    int g = 1;
    while (g * 4 < dims.dstate) g *= 2;
    const int64_t cpb = ssm::kBlock / g;
    if (dims.batch * ((dims.dim + cpb - 1) / cpb) > kMaxGridX)
        return fail(SSM_ERR_UNSUPPORTED, "grid too large");
    ssm::DecodeArgs a{};
    a.state = state; a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.A = A; a.Dskip = D; a.out = out;
    a.batch = dims.batch; a.dim = dims.dim; a.dstate = (int)dims.dstate;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (kDecodeBulk && ssm::state_update_bulk_eligible(a, io == SSM_BF16))
        e = ssm::launch_state_update_bulk(a, io == SSM_BF16, g_inject_wait_bytes.load(), st);
    else
        e = ssm::launch_state_update(a, io == SSM_BF16, 4, g, st);
    if (e != cudaSuccess) return cuda_fail(e, "state update launch");
    return SSM_OK;
}

ssm_status ssm_ssd_scan_fwd(ssm_ssd_dims dims, ssm_dtype io, const void *x, const void *dt, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int dt_softplus, void *out, float *last_state,
                            ssm_stream stream) {
    g_last_error[0] = 0;
    size_t es = 0;
    if (ssm_status s = check_io(io, &es)) return s;
    if (dims.batch < 0 || dims.seqlen < 0 || dims.heads < 0 || dims.headdim < 0 || dims.groups < 0 ||
        dims.dstate < 0)
        return fail(SSM_ERR_INVALID_ARG, "negative size");
    if (dims.groups < 1 || dims.heads % dims.groups != 0)
        return fail(SSM_ERR_INVALID_ARG, "heads (%lld) must be a multiple of groups (%lld >= 1)",
                    (long long)dims.heads, (long long)dims.groups);
    if (dt_softplus != 0 && dt_softplus != 1) return fail(SSM_ERR_INVALID_ARG, "dt_softplus must be 0 or 1");
    if (io != SSM_BF16) return fail(SSM_ERR_UNSUPPORTED, "the SSD layer runs on bf16 tensors only");
    if (dims.headdim != 64) return fail(SSM_ERR_UNSUPPORTED, "headdim %lld (64 is built)", (long long)dims.headdim);
    if (dims.dstate != 64 && dims.dstate != 128)
        return fail(SSM_ERR_UNSUPPORTED, "dstate %lld (64 or 128 are built)", (long long)dims.dstate);
    if (dims.batch == 0 || dims.heads == 0 || dims.seqlen == 0) return SSM_OK;  // state unchanged
    if (dims.seqlen > 0x7fffffffLL || dims.batch > 0x7fffffffLL || dims.heads * dims.headdim > 0x7fffffffLL ||
        dims.groups * dims.dstate > 0x7fffffffLL)
        return fail(SSM_ERR_UNSUPPORTED, "a tensor coordinate exceeds 32 bits");
    if (!x || !dt || !A || !B || !C || !out) return fail(SSM_ERR_INVALID_ARG, "x, dt, A, B, C and out are required");
    if (misaligned(dt, 2) || misaligned(A, 4) || misaligned(D, 4) || misaligned(dt_bias, 4) ||
        misaligned(last_state, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
    if (misaligned(x, 16) || misaligned(z, 16) || misaligned(B, 16) || misaligned(C, 16) || misaligned(out, 16))
        return fail(SSM_ERR_UNSUPPORTED, "x, z, B, C and out must be 16-byte aligned (tensor-memory copies)");
    ssm::SsdFwdArgs a{};
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.dt_bias = dt_bias; a.out = out; a.state = last_state;
    a.batch = dims.batch; a.seqlen = dims.seqlen; a.heads = dims.heads; a.headdim = dims.headdim;
    a.groups = dims.groups; a.dstate = dims.dstate; a.softplus = dt_softplus;
    if (!ssm::ssd_fwd_supported(a))
        return fail(SSM_ERR_UNSUPPORTED, "the driver offers no tensor-map encoder (cuTensorMapEncodeTiled)");
    cudaError_t e = ssm::launch_ssd_fwd(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "SSD kernel launch");
    return SSM_OK;
}

ssm_status ssm_get_device_status(ssm_stream stream, uint32_t *flags) {
    g_last_error[0] = 0;
    if (!flags) return fail(SSM_ERR_INVALID_ARG, "flags is required");
    cudaError_t e = cudaSuccess;
    *flags = ssm::read_and_clear_device_status(reinterpret_cast<cudaStream_t>(stream), &e);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    return SSM_OK;
}

ssm_status ssm_test_exp2_poly(const float *x, float *poly, float *sfu, int64_t n, ssm_stream stream) {
    g_last_error[0] = 0;
    if (n < 0) return fail(SSM_ERR_INVALID_ARG, "n must be >= 0");
    if (n > 0 && (!x || !poly || !sfu)) return fail(SSM_ERR_INVALID_ARG, "x, poly and sfu are required");
    if (misaligned(x, 4) || misaligned(poly, 4) || misaligned(sfu, 4))
        return fail(SSM_ERR_INVALID_ARG, "a pointer is not aligned to its element size");
    cudaError_t e = ssm::launch_exp2_poly_check(x, poly, sfu, n, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "exp2 check launch");
    return SSM_OK;
}

void ssm_test_inject_decode_wait_timeout(int32_t enable) { g_inject_wait_bytes.store(enable ? 16u : 0u); }

}  // extern "C"
