// exp2_poly_check.cu -- evaluates the FMA-pipe exp2 of the fast scan tier
// (exp2_poly2 in ssm_device.cuh) over an array, so that a test can compare it
// with exp2 in fp64 and with the SFU's ex2.approx on the GPU itself.
#include "scan_kernels.cuh"

namespace ssm {

namespace {

__global__ void exp2_poly_check_kernel(const float *x, float *poly, float *sfu, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
    const float2 p = exp2_poly2(v);
    poly[i] = p.x;
    sfu[i] = ex2_approx(v.x);
    if (i + 1 < n) {
        poly[i + 1] = p.y;
        sfu[i + 1] = ex2_approx(v.y);
    }
}

}  // namespace

cudaError_t launch_exp2_poly_check(const float *x, float *poly, float *sfu, int64_t n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t pairs = (n + 1) / 2;
    const int64_t blocks = (pairs + 255) / 256;
    if (blocks > 2147483647LL) return cudaErrorInvalidValue;
    exp2_poly_check_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, poly, sfu, n);
    return cudaGetLastError();
}

}  // namespace ssm
