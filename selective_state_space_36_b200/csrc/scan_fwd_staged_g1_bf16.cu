// scan_fwd_staged_g1_bf16.cu -- instantiations of the staged forward kernel
// with 1 lane(s) per channel and bf16 I/O (see scan_fwd_staged.cuh).
#include "scan_fwd_staged.cuh"

namespace ssm {

cudaError_t launch_staged_g1_bf16(const ScanArgs &a, int ns, int cpl, int variant, cudaStream_t st) {
    return cpl == 2 ? launch_layouts<__nv_bfloat16, 1, 2>(a, ns, variant, st) : launch_layouts<__nv_bfloat16, 1, 1>(a, ns, variant, st);
}

}  // namespace ssm
