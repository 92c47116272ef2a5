// cp_async.cuh -- 16-byte global -> shared copies tracked by cp.async groups
// (shared by the staged scan kernels).
#pragma once

namespace ssm {

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool full) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = full ? 16 : 0;  // 0: no global read, destination zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace ssm
