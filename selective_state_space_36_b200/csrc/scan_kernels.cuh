// scan_kernels.cuh -- argument block and launch entry points of the scan and
// decode kernels (internal to the library; the public ABI is include/ssm.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "ssm_device.cuh"

namespace ssm {

constexpr int kBlock = 128;  // threads per block
constexpr int kChunk = 64;   // time steps of B/C staged in shared memory at once

// kCkpt: forward recurrence only (no readout), storing the state entering
// every kCkptEvery-th step -- the first pass of the backward scan.
enum ScanMode { kFull = 0, kSegAgg = 1, kSegFinal = 2, kCkpt = 3 };
constexpr int kCkptEvery = 8;  // kCkpt: steps between stored states
enum { kVariantSlab = 1, kVariantSplit = 2, kVariantCkpt = 3 };
// kernel family: generic (direct global loads, any alignment) or staged
// (cp.async pipeline through shared memory, 16-byte aligned rows)
enum { kFamilyAuto = 0, kFamilyGeneric = 1, kFamilyStaged = 2 };

struct ScanArgs {
    const void *u, *delta, *B, *C, *z;
    const float *A, *Dskip, *bias;
    void *out;
    float *last_state;
    // sequence-split workspace: h_0 copy (batch, dim, N), local end states
    // (batch, nseg, dim, N), Delta sums (batch, nseg, dim)
    float *seg_h0, *seg_h, *seg_dsum;
    int64_t batch, seqlen, dim;
    int dstate;
    int softplus;
    int zoh_b;        // 1: exact zero-order hold on B (Bbar = expm1(Delta A)/A B); 0: Euler (Delta B)
    int64_t seg_len;  // time steps per segment (== seqlen for one pass)
    int nseg;
    // kCkpt: states (batch, ceil(seqlen / kCkptEvery), dim, dstate); h_0 is
    // read from last_state, which is not written
    float *ckpt;
    // staged kernel: (batch row, channel tile) work units; set by its launcher
    int64_t units;
};

struct DecodeArgs {
    float *state;
    const void *x, *dt, *B, *C, *z;
    const float *A, *Dskip;
    void *out;
    int64_t batch, dim;
    int dstate;
};

// Gradient of the scan (Euler Bbar): inputs as in ScanArgs plus dout; the
// accumulated gradients (dA, dB, dC, dD, dbias) must be zero on entry.
struct ScanBwdArgs {
    const void *u, *delta, *B, *C, *z, *dout;
    const float *A, *Dskip, *bias, *h0;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *dbias, *dh0;
    float *ckpt;  // workspace: (batch, ceil(seqlen / chunk), dim, dstate) states
    int64_t batch, seqlen, dim;
    int dstate;
    int softplus;
    int vec_red;  // dB / dC rows take 16-byte vector atomics
};

cudaError_t launch_scan_fwd(const ScanArgs &a, bool bf16, int ns, int g, int cpl, int variant,
                            int family, cudaStream_t st);
cudaError_t launch_scan_staged(const ScanArgs &a, bool bf16, int ns, int g, int cpl, int variant,
                               cudaStream_t st);
bool staged_eligible(const ScanArgs &a, int es);
size_t staged_smem_bytes(bool bf16, int ns, int g, int cpl);
bool scan_shape_supported(int ns, int g);
cudaError_t launch_state_update(const DecodeArgs &a, bool bf16, int ns, int g, cudaStream_t st);
// decode step with the state moved by TMA bulk copies (dstate 4, 8, 16, 32 or
// 64; 16-byte aligned state and A); missing_bytes > 0 makes every unit's wait
// expect bytes that never arrive (a test of the bounded waits)
bool state_update_bulk_eligible(const DecodeArgs &a, bool bf16);
cudaError_t launch_state_update_bulk(const DecodeArgs &a, bool bf16, uint32_t missing_bytes, cudaStream_t st);
// the device status word the kernels' bounded waits report into (bit 0: a
// decode wait ran out; bit 1: an SSD scan wait ran out)
unsigned int read_and_clear_device_status(cudaStream_t st, cudaError_t *err);
cudaError_t device_status_address(unsigned int **p);
cudaError_t launch_scan_bwd(const ScanBwdArgs &a, bool bf16, cudaStream_t st);
// complex diagonal A: A, B, C and last_state hold (re, im) pairs
cudaError_t launch_scan_complex(const ScanArgs &a, bool bf16, cudaStream_t st);
int64_t scan_complex_channels_per_block();
// staged second pass (checkpoints every scan_bwd_staged_chunk() steps, from
// the staged forward kernel in kCkpt mode)
bool scan_bwd_staged_eligible(const ScanBwdArgs &a, int es);
int scan_bwd_staged_chunk();
cudaError_t launch_scan_bwd_staged(const ScanBwdArgs &a, bool bf16, cudaStream_t st);
int64_t scan_bwd_chunk(int dstate);              // time steps between checkpoints

// Mamba-2 SSD layer (bf16 x, dt, B, C, z, out; fp32 A, D, dt_bias, state):
// x, z, out (batch, seqlen, heads, headdim); dt (batch, seqlen, heads);
// B, C (batch, seqlen, groups, dstate); state (batch, heads, headdim, dstate)
struct SsdFwdArgs {
    const void *x, *dt, *B, *C, *z;
    const float *A, *D, *dt_bias;
    void *out;
    float *state;
    int64_t batch, seqlen, heads, headdim, groups, dstate;
    int softplus;
};
bool ssd_fwd_supported(const SsdFwdArgs &a);
// the fast tier's FMA-pipe exp2 (and the SFU's ex2) of n values, for tests
cudaError_t launch_exp2_poly_check(const float *x, float *poly, float *sfu, int64_t n, cudaStream_t st);  // headdim 64, dstate 64 or 128, 16-byte aligned tensors
cudaError_t launch_ssd_fwd(const SsdFwdArgs &a, cudaStream_t st);
int64_t scan_bwd_channels_per_block();

}  // namespace ssm
