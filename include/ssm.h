/*
 * ssm.h -- C ABI of the B200 selective state-space (S6) library.
 *
 * The library computes the selective SSM of Mamba ("Mamba: Linear-Time
 * Sequence Modeling with Selective State Spaces") with hand-written sm_100a
 * CUDA kernels.  For every channel (b, d) independently (NL-345 Mamba
 * translation, section 2 "Structure and Dimensions"):
 *
 *   Delta_t = softplus(delta[b,t,d] + delta_bias[d])   (or the plain sum)
 *   Abar    = exp(Delta_t * A[d,n])                    (zero-order hold on A)
 *   Bbar    = Delta_t * B[b,t,n]                       (Euler form on B)
 *   h_t[n]  = Abar * h_{t-1}[n] + Bbar * u[b,t,d]      (section 2, eq. (2))
 *   y_t     = sum_n C[b,t,n] * h_t[n] + D[d] * u[b,t,d]
 *   out     = y_t * silu(z[b,t,d])                      (if z is given)
 *
 * Sources: NL-345 translation, section 2 "Discretization" and eq. (2)
 * (recurrence, readout after the update); 【論文要約】Mamba notes, 数式解説 3
 * (ZOH for Abar) and the "S6" section, Algorithm 2 (B, C per token, Delta =
 * softplus(parameter + projection)).  The pages give the exact ZOH form for
 * Bbar; this library uses the Euler form Delta * B by default and offers the
 * exact form through ssm_selective_scan_fwd_ex.  The D skip and the silu(z)
 * gate are the Mamba block's epilogue fused into the scan.
 *
 * Entry points: the scan (ssm_selective_scan_fwd, _ex with execution choices
 * and the exact ZOH form, _noalloc without device allocation), its gradient
 * (ssm_selective_scan_bwd, _ex), the scan with a complex diagonal A
 * (ssm_selective_scan_fwd_complex), Mamba-2's SSD layer (ssm_ssd_scan_fwd),
 * the one-token decode step
 * (ssm_selective_state_update), planning (ssm_scan_plan), the device status
 * word of the bounded waits (ssm_get_device_status) and error reporting.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers (cudaMalloc / cudaMallocAsync /
 *    torch CUDA memory) on the current device; the caller owns every buffer.
 *  - Layouts are dense and row-major:
 *      u, delta, z, out : (batch, seqlen, dim)     dim contiguous
 *      B, C             : (batch, seqlen, dstate)  dstate contiguous
 *      A                : (dim, dstate)            float32
 *      D, delta_bias    : (dim)                    float32
 *      state/last_state : (batch, dim, dstate)     float32
 *    "io" selects the element type of u, delta, z, B, C (and x, dt for the
 *    decode step) and out: SSM_F32 = float, SSM_BF16 = bfloat16 (out rounded
 *    to nearest even).  All arithmetic is fp32.
 *  - Every pointer must be aligned to its element size; no other alignment is
 *    required.  Sizes are arbitrary (ragged tails are masked); 1 <= dstate <= 64.
 *  - Work is enqueued on "stream" (a cudaStream_t; NULL is the legacy default
 *    stream).  No entry point synchronises the stream or the device, except
 *    ssm_get_device_status, which synchronises "stream" to read the word.
 *  - Argument errors return SSM_ERR_INVALID_ARG or SSM_ERR_UNSUPPORTED before
 *    anything is enqueued.  A failed launch returns SSM_ERR_CUDA.  The message
 *    of the last failure on the calling thread is ssm_last_error().
 *  - out must not overlap any input.  Calls are thread-safe.
 */
#ifndef SSM_B200_H
#define SSM_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad flag */
    SSM_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (dstate > 64) */
    SSM_ERR_CUDA = 3         /* a CUDA call failed; see ssm_last_error() */
} ssm_status;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

typedef struct {
    int64_t batch;  /* Bt */
    int64_t seqlen; /* L (ignored by the decode step) */
    int64_t dim;    /* D: channels */
    int64_t dstate; /* N: state size per channel */
} ssm_dims;

/* A cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st *ssm_stream;

/*
 * Selective scan, forward (one pass over the whole sequence).
 *
 *   u, delta       : (batch, seqlen, dim) io; delta is the raw Delta.
 *   A              : (dim, dstate) float32, used as given (no sign check).
 *   B, C           : (batch, seqlen, dstate) io, shared by all channels.
 *   D              : (dim) float32 or NULL (no skip term).
 *   z              : (batch, seqlen, dim) io or NULL (no gate).
 *   delta_bias     : (dim) float32 or NULL (zero bias).
 *   delta_softplus : 1 => Delta = softplus(delta + bias); 0 => delta + bias.
 *                    (Bbar is the Euler form Delta B; ssm_selective_scan_fwd_ex can select
 *                    the exact zero-order hold instead.)
 *   out            : (batch, seqlen, dim) io, written.
 *   last_state     : (batch, dim, dstate) float32 or NULL.  In: h_0 (the scan
 *                    resumes from it).  Out: h_L.  NULL => h_0 = 0, h_L not
 *                    returned.  With seqlen == 0 it is left unchanged.
 *
 * The expanded (batch, seqlen, dim, dstate) state never exists in memory; the
 * fp32 state lives in registers.  When batch * dim is too small to fill the
 * GPU, the sequence is split into segments scanned in parallel and joined
 * with the associative combine (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2); the
 * per-segment carries (8 bytes per (batch, segment, dim, dstate) plus 4 per
 * (batch, segment, dim)) are taken on "stream" from the library's workspace
 * pool and released on the same stream (see "Workspace memory" below).
 *
 * Workspace memory (the split scan's carries, the backward's checkpoints):
 * stream-ordered allocations (cudaMallocFromPoolAsync / cudaFreeAsync) from a
 * pool the library creates per device, which keeps freed memory for later
 * calls instead of returning it to the driver: a repeated call reuses its
 * workspace.  The pool holds at most the largest amount of workspace in use
 * at once, until the process exits.
 */
ssm_status ssm_selective_scan_fwd(ssm_dims dims, ssm_dtype io,
                                  const void *u, const void *delta, const float *A,
                                  const void *B, const void *C, const float *D,
                                  const void *z, const float *delta_bias, int delta_softplus,
                                  void *out, float *last_state, ssm_stream stream);

/* Execution choices for ssm_selective_scan_fwd_ex; zero-initialise for defaults. */
typedef enum {
    SSM_VARIANT_AUTO = 0,  /* pick by shape */
    SSM_VARIANT_SLAB = 1,  /* one pass: each thread group owns channels for all of L */
    SSM_VARIANT_SPLIT = 2  /* sequence split: segment carries, then a second pass */
} ssm_variant;

typedef enum {
    SSM_KERNEL_AUTO = 0,     /* staged when eligible, else generic */
    SSM_KERNEL_GENERIC = 1,  /* direct global loads; any size and element alignment */
    SSM_KERNEL_STAGED = 2    /* inputs staged through shared memory with 16-byte async
                                copies; needs dim and dstate rows of a multiple of 16
                                bytes and 16-byte aligned u, delta, z, B, C, out
                                (SSM_ERR_UNSUPPORTED otherwise) */
} ssm_kernel_family;

/* How B is discretised (A always uses the zero-order hold, Abar = exp(Delta A)). */
typedef enum {
    SSM_DISCRETIZE_EULER_B = 0, /* Bbar = Delta B (the default) */
    SSM_DISCRETIZE_ZOH = 1      /* exact zero-order hold: Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B
                                   = expm1(Delta A) / A * B, and Delta B where Delta A = 0
                                   (【論文要約】Mamba notes, 数式解説 3); one channel per lane only */
} ssm_discretization;

typedef struct {
    int32_t variant;  /* ssm_variant */
    int32_t segments; /* SPLIT only: number of sequence segments, 0 = automatic */
    int32_t lanes;    /* lanes sharing one channel: 0 = automatic, else 1, 2 or 4
                         (honoured for 9 <= dstate <= 32) */
    int32_t family;   /* ssm_kernel_family */
    int32_t channels_per_lane; /* staged kernel: 0 = automatic, 1, or 2 (one B/C load serves two
                                  adjacent channels) */
    int32_t discretization;    /* ssm_discretization of B */
    int32_t reserved[2];       /* must be zero */
} ssm_scan_opts;

/* ssm_selective_scan_fwd with explicit execution choices (opts may be NULL).
 * Every variant computes the same function; results agree to fp32 rounding. */
ssm_status ssm_selective_scan_fwd_ex(ssm_dims dims, ssm_dtype io,
                                     const void *u, const void *delta, const float *A,
                                     const void *B, const void *C, const float *D,
                                     const void *z, const float *delta_bias, int delta_softplus,
                                     void *out, float *last_state, const ssm_scan_opts *opts,
                                     ssm_stream stream);

/*
 * ssm_selective_scan_fwd for callers that cannot allocate device memory at
 * call time.  (The paper has no counterpart: this is a deployment option.)
 *
 * Who needs it: a serving runtime that reserved nearly all of the GPU's memory
 * for its own pool at start-up, so growing the library's workspace pool
 * would fail or fragment that reservation; a real-time or latency-budgeted
 * path that may not take the allocator's locks; an embedding where all device
 * memory is owned by the host application.  The only scratch the scan needs
 * is the carry buffer of the sequence split, and this entry point takes it
 * from a fixed static array inside the library instead of allocating.
 *
 * Same arguments and results as ssm_selective_scan_fwd, with the sequence
 * split always requested: segments = the number of segments, or 0 for the
 * automatic count, lowered to the largest count whose carries fit the scratch;
 * when not even two segments fit, one pass runs (it needs no scratch).  When
 * the sequence is too short to split, one pass runs and no scratch is used.
 *
 * Limits and behaviour:
 *  - The scratch holds SSM_NOALLOC_SCRATCH_BYTES (16 MiB).  A split needs
 *    4 * batch * dim * (dstate * (segments + 1) + segments) bytes; an explicit
 *    segment count that does not fit returns SSM_ERR_UNSUPPORTED before
 *    anything is enqueued.  Every GPU on which the library is loaded holds
 *    these 16 MiB until the process exits.
 *  - No cudaMalloc, cudaMallocAsync, cudaFree or allocating library routine is
 *    called.  The first call on each device (and the first after a
 *    cudaDeviceReset, which replaces the device's context) looks up the
 *    scratch's device address (cudaGetSymbolAddress) with that device
 *    current; make that first call before any stream capture.
 *  - All calls share the one scratch array, which keeps the last call's
 *    contents.  Nothing in it needs to start at zero (each call writes every
 *    word it later reads), but calls whose GPU work overlaps in time -- on
 *    different streams, or from different threads -- race on it: order them
 *    on one stream or synchronise between them.
 */
#define SSM_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

ssm_status ssm_selective_scan_fwd_noalloc(ssm_dims dims, ssm_dtype io,
                                          const void *u, const void *delta, const float *A,
                                          const void *B, const void *C, const float *D,
                                          const void *z, const float *delta_bias, int delta_softplus,
                                          void *out, float *last_state, int segments,
                                          ssm_stream stream);

/* What a scan call with these arguments would do (nothing is launched or
 * allocated; data pointers are only inspected for alignment and may be
 * fake).  Lets a caller size the workspace and count kernel launches. */
typedef struct {
    int32_t variant;         /* ssm_variant chosen: SLAB or SPLIT */
    int32_t segments;        /* sequence segments (1 for SLAB) */
    int32_t lanes;           /* lanes per channel */
    int32_t family;          /* ssm_kernel_family chosen: GENERIC or STAGED */
    int32_t launches;        /* kernels the call enqueues (0 for an empty problem) */
    int32_t channels_per_lane;
    int64_t workspace_bytes; /* device scratch the call allocates (SPLIT), else 0 */
} ssm_scan_plan_info;

ssm_status ssm_scan_plan(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                         const void *B, const void *C, const void *z, const void *out,
                         const ssm_scan_opts *opts, ssm_scan_plan_info *info);

/*
 * Selective scan with a complex diagonal A (and complex B, C), one pass over
 * the sequence: the complex parameterisation the Mamba notes single out for
 * audio (【論文要約】Mamba notes, Figure 10; Table 8), read as the real
 * recurrence carried out in complex numbers:
 *   Abar_n = exp(Delta A_n),  Bbar_n = Delta B_n (Euler),
 *   h_n <- Abar_n h_n + Bbar_n u,   y = Re(sum_n C_n h_n) + D u,
 *   out = y * silu(z).
 * Delta (softplus(delta + bias) or the plain sum), u, z, D, delta_bias and
 * out are real, with the layouts of ssm_selective_scan_fwd.  Complex arrays
 * hold (re, im) pairs:
 *   A          : (dim, dstate, 2) float32
 *   B, C       : (batch, seqlen, dstate, 2) io
 *   last_state : (batch, dim, dstate, 2) float32 or NULL; read as h_0 and
 *                overwritten with h_L (NULL: h_0 = 0, not written).
 * Returns the statuses of ssm_selective_scan_fwd.  No sequence split.
 */
ssm_status ssm_selective_scan_fwd_complex(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                          const float *A, const void *B, const void *C, const float *D,
                                          const void *z, const float *delta_bias, int delta_softplus,
                                          void *out, float *last_state, ssm_stream stream);

/*
 * Selective scan, backward: the gradients of the scalar loss sum(dout * out)
 * of one ssm_selective_scan_fwd pass (Euler Bbar) with respect to every input.
 * The states are recomputed from checkpoints instead of being kept by the
 * forward pass (【論文要約】Mamba notes, "3.ハードウェアを考慮した効率的な
 * アルゴリズム": recomputation keeps the stored intermediate states small;
 * NL-345 section 1, "Fast training and inference").
 *
 * Inputs are those of the forward call (same layouts and dtypes; h0 is the
 * state the forward pass started from, (batch, dim, dstate) float32, or NULL
 * for zero) plus
 *   dout           : (batch, seqlen, dim) io, the gradient of out.
 * Outputs (all written, none accumulated into):
 *   du, ddelta     : (batch, seqlen, dim) io.  ddelta is d/d(raw delta).
 *   dz             : (batch, seqlen, dim) io; required iff z is given.
 *   dA             : (dim, dstate) float32.
 *   dB, dC         : (batch, seqlen, dstate) float32.
 *   dD             : (dim) float32; required iff D is given.
 *   ddelta_bias    : (dim) float32 or NULL (not computed).
 *   dh0            : (batch, dim, dstate) float32 or NULL (not computed).
 * The float32 sums (dA, dB, dC, dD, ddelta_bias) are accumulated with
 * atomics, so their last bits depend on the order blocks finish in.
 * Workspace: (batch, ceil(seqlen / K), dim, dstate) float32 state checkpoints
 * (K = 8 on the staged path; 16, 8 or 4 on the generic one for dstate <= 16,
 * 32, 64), taken from the library's workspace pool on "stream" (see
 * ssm_selective_scan_fwd).  Output buffers must not overlap each other or any
 * input.
 */
ssm_status ssm_selective_scan_bwd(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                  const float *A, const void *B, const void *C, const float *D,
                                  const void *z, const float *delta_bias, int delta_softplus,
                                  const float *h0, const void *dout, void *du, void *ddelta,
                                  void *dz, float *dA, float *dB, float *dC, float *dD,
                                  float *ddelta_bias, float *dh0, ssm_stream stream);

/*
 * ssm_selective_scan_bwd with a forced kernel family (tests, tuning).  Only
 * opts->family is read; every other field of opts must be zero (the backward
 * has no sequence split and no lane choices, and implements the Euler Bbar
 * only).  SSM_KERNEL_STAGED -- a checkpointing pass of the staged forward
 * kernel (a state every 8 steps) and a staged reverse pass -- needs
 * dstate <= 16 and the staged forward kernel's row alignment (for du, ddelta,
 * dz and dout as well); SSM_KERNEL_GENERIC is one kernel with direct global
 * loads and a checkpoint every 64 / ceil(dstate / 4) steps.  opts may be NULL
 * (automatic: staged where eligible).
 */
ssm_status ssm_selective_scan_bwd_ex(ssm_dims dims, ssm_dtype io, const void *u, const void *delta,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, const float *delta_bias, int delta_softplus,
                                     const float *h0, const void *dout, void *du, void *ddelta,
                                     void *dz, float *dA, float *dB, float *dC, float *dD,
                                     float *ddelta_bias, float *dh0, const ssm_scan_opts *opts,
                                     ssm_stream stream);

/*
 * One recurrent (decode) step for every channel: constant time and memory per
 * generated token, no cache of past inputs (NL-345 section 1, "Fast training
 * and inference"; section 2 eq. (2) for a single t).
 *
 *   state : (batch, dim, dstate) float32, updated in place (h_{t-1} -> h_t).
 *   x, dt : (batch, dim) io; dt is the time step itself (already positive:
 *           no bias and no softplus are applied).
 *   A     : (dim, dstate) float32.     B, C : (batch, dstate) io.
 *   D     : (dim) float32 or NULL.     z    : (batch, dim) io or NULL.
 *   out   : (batch, dim) io.
 * dims.seqlen is ignored.  With dstate 4, 8, 16, 32 or 64, a 16-byte aligned
 * state and A, and B, C aligned to four elements, the state moves through
 * shared memory in 16 KB units by TMA bulk copies (a persistent kernel whose
 * waits are bounded, see ssm_get_device_status); otherwise each thread loads
 * its 4-state slice directly.
 */
ssm_status ssm_selective_state_update(ssm_dims dims, ssm_dtype io, float *state,
                                      const void *x, const void *dt, const float *A,
                                      const void *B, const void *C, const float *D,
                                      const void *z, void *out, ssm_stream stream);

/*
 * Mamba-2's SSD layer ("Transformers are SSMs: Generalized Models and
 * Efficient Algorithms Through Structured State Space Duality", review on
 * nubint.ai, 提案手法): the selective SSM with one scalar A per head, whose
 * sequence map is a semiseparable matrix, computed by its block
 * decomposition -- the quadratic (attention-like) form inside chunks of 128
 * tokens and the linear (recurrent) form between chunks -- on the tensor
 * cores.  For every batch row b, head h (of P = headdim channels) and time t:
 *
 *   Delta_t = softplus(dt[b,t,h] + dt_bias[h])      (or the plain sum)
 *   H_t     = exp(Delta_t A[h]) H_{t-1} + Delta_t x[b,t,h,:] B[b,t,g,:]^T
 *   y       = H_t C[b,t,g,:] + D[h] x[b,t,h,:],     out = y * silu(z[b,t,h,:])
 *
 * with H (headdim x dstate) per (b, h) and g = h / (heads / groups) the
 * group whose B, C the head reads.  Layouts (dense, row-major):
 *   x, z, out  : (batch, seqlen, heads, headdim) bf16; z may be NULL (no gate)
 *   dt         : (batch, seqlen, heads) bf16, the raw step
 *   A, D, dt_bias : (heads) float32; D and dt_bias may be NULL (zero)
 *   B, C       : (batch, seqlen, groups, dstate) bf16
 *   last_state : (batch, heads, headdim, dstate) float32 or NULL; read as H_0
 *                and overwritten with H_L (NULL: H_0 = 0, not returned).
 * Supported: io = SSM_BF16, headdim = 64, dstate = 64 or 128, heads a
 * multiple of groups, x, z, B, C, out 16-byte aligned (SSM_ERR_UNSUPPORTED
 * otherwise).  Arithmetic: products on the tensor cores with bf16 operands
 * and fp32 accumulation; the state is carried in fp32; three operands take
 * two terms, a bf16 high part plus the bf16 rounding of the rest: the masked
 * intra-chunk matrix, the weighted x of the chunk's state update, and the
 * carried state in the inter-chunk output.  A wait inside
 * the kernel that runs out (2 s) sets bit 1 of the device status word
 * (ssm_get_device_status); the outputs are then not valid.
 */
typedef struct {
    int64_t batch, seqlen, heads, headdim, groups, dstate;
} ssm_ssd_dims;

ssm_status ssm_ssd_scan_fwd(ssm_ssd_dims dims, ssm_dtype io, const void *x, const void *dt, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int dt_softplus, void *out, float *last_state,
                            ssm_stream stream);

/*
 * Reads and clears the device status word of the current device, after
 * synchronising "stream".  Bit 0: a bounded wait inside the decode kernel
 * (its state copies, see ssm_selective_state_update) gave up; the outputs of
 * the launches since the last read are then not valid.  Bit 1: a bounded
 * wait inside the SSD kernel (ssm_ssd_scan_fwd) gave up.  The word is shared by
 * every launch on the device.  Returns SSM_ERR_CUDA if the copies or the
 * synchronisation fail.
 */
ssm_status ssm_get_device_status(ssm_stream stream, uint32_t *flags);

/*
 * Test hook (no counterpart in the method): while enabled, every decode
 * launch that moves its state with bulk copies waits for 16 bytes per unit
 * that never arrive, so each of its waits runs out (200 ms) and sets bit 0 of
 * the device status word; the copies themselves complete normally.  Used to
 * test the bounded waits without a GPU fault.  Process-wide; 0 disables.
 */
void ssm_test_inject_decode_wait_timeout(int32_t enable);

/* Build parameters that set the arithmetic of the library's kernels (no
 * counterpart in the method; lets a benchmark state the ceiling of the code
 * it runs). */
typedef struct {
    int32_t sfu_decays_per_16; /* of every 16 decays exp(Delta A) of the bf16 (fast) scan
                                  tier, how many the SFU computes; the rest are computed
                                  on the FMA pipe by a polynomial */
    int32_t split_pass1_sfu_decays_per_16; /* the same for the first pass of the
                                  sequence split (segment aggregates) */
    int32_t reserved[6];
} ssm_build_info;

void ssm_get_build_info(ssm_build_info *info);

/*
 * Test hook (no counterpart in the method): evaluates, for n float32 inputs x,
 * the FMA-pipe exp2 that computes part of the decays of the bf16 scan tier
 * (poly[i]) and the SFU's ex2.approx (sfu[i]); device pointers, enqueued on
 * "stream".  Lets a test bound the polynomial's error on the GPU itself.
 */
ssm_status ssm_test_exp2_poly(const float *x, float *poly, float *sfu, int64_t n, ssm_stream stream);

/* Static description of a status code. */
const char *ssm_status_string(ssm_status status);

/* Detail of the last non-OK status returned on the calling thread ("" if none). */
const char *ssm_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_B200_H */
