// scan_fwd_staged.cu -- the staged forward kernel's host-side dispatch: the
// shared-memory size of each layout and the launch by (I/O type, lanes).
// The kernel itself is in scan_fwd_staged.cuh; its instantiations live in
// scan_fwd_staged_g{1,2,4}_{bf16,f32}.cu.
#include "scan_fwd_staged.cuh"

namespace ssm {

template <typename IO, int CPL>
static size_t smem_of(int ns, int g) {
    if (ns == 4 && g == 1) return StagedLayout<IO, 4, 1, CPL>::SMEM;
    if (ns == 8 && g == 1) return StagedLayout<IO, 8, 1, CPL>::SMEM;
    if (ns == 16 && g == 1) return StagedLayout<IO, 16, 1, CPL>::SMEM;
    if (ns == 8 && g == 2) return StagedLayout<IO, 8, 2, CPL>::SMEM;
    if (ns == 4 && g == 4) return StagedLayout<IO, 4, 4, CPL>::SMEM;
    if (ns == 16 && g == 2) return StagedLayout<IO, 16, 2, CPL>::SMEM;
    if (ns == 8 && g == 4) return StagedLayout<IO, 8, 4, CPL>::SMEM;
    if (ns == 16 && g == 4) return StagedLayout<IO, 16, 4, CPL>::SMEM;
    return ~(size_t)0;
}

size_t staged_smem_bytes(bool bf16, int ns, int g, int cpl) {
    if (cpl == 2) return bf16 ? smem_of<__nv_bfloat16, 2>(ns, g) : smem_of<float, 2>(ns, g);
    return bf16 ? smem_of<__nv_bfloat16, 1>(ns, g) : smem_of<float, 1>(ns, g);
}

cudaError_t launch_scan_staged(const ScanArgs &a, bool bf16, int ns, int g, int cpl, int variant,
                               cudaStream_t st) {
    if (cpl != 1 && cpl != 2) return cudaErrorInvalidConfiguration;
    if (g == 1) return bf16 ? launch_staged_g1_bf16(a, ns, cpl, variant, st) : launch_staged_g1_f32(a, ns, cpl, variant, st);
    if (g == 2) return bf16 ? launch_staged_g2_bf16(a, ns, cpl, variant, st) : launch_staged_g2_f32(a, ns, cpl, variant, st);
    if (g == 4) return bf16 ? launch_staged_g4_bf16(a, ns, cpl, variant, st) : launch_staged_g4_f32(a, ns, cpl, variant, st);
    return cudaErrorInvalidConfiguration;
}

}  // namespace ssm
