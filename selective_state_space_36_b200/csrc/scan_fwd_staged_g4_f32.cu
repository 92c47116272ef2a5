// scan_fwd_staged_g4_f32.cu -- instantiations of the staged forward kernel
// with 4 lane(s) per channel and fp32 I/O (see scan_fwd_staged.cuh).
#include "scan_fwd_staged.cuh"

namespace ssm {

cudaError_t launch_staged_g4_f32(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st) {
    return cpl == 2 ? launch_layouts<float, 4, 2>(a, ns, variant, st) : launch_layouts<float, 4, 1>(a, ns, variant, st);
}

}  // namespace ssm
