// pipe_rates.cu -- per-SM throughput of the instruction classes the scan is
// made of, measured with clock64 inside each block (all blocks co-resident,
// 64 warps per SM).  Not part of the library: a standalone probe whose numbers
// decide how the scan's exponentials are computed.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o pipe_rates pipe_rates.cu && ./pipe_rates
//
// Each kernel runs chains of "one transcendental followed by K other ops"; the
// transcendental rate and the other-op rate per SM clock tell how the SFU
// shares the issue slots with the FMA pipe.
#include <cuda_runtime.h>

#include <cstdio>

#define ITERS 1024

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float th(float x) {
    float y;
    asm volatile("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ unsigned ex2h2(unsigned x) {
    unsigned y;
    asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
    unsigned long long d;
    asm volatile("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// KIND: 0 ex2 + K ffma, 1 tanh + K ffma, 2 ex2.f16x2 + K ffma, 3 ex2 + K ffma2,
//       4 K ffma only, 5 K ffma2 only, 6 ex2 + K/2 ffma + K/2 integer xor-add,
//       7 K/2 ffma + K/2 integer xor-add (no transcendental)
template <int K, int KIND>
__global__ void chains(float *out, long long *cyc, float s) {
    float a[4], b[4];
    unsigned hh[4], iv[4];
    unsigned long long b2[4], s2, c2;
    {
        float2 v = make_float2(s, s);
        s2 = *reinterpret_cast<unsigned long long *>(&v);
        float2 w = make_float2(0.25f, 0.25f);
        c2 = *reinterpret_cast<unsigned long long *>(&w);
    }
    for (int i = 0; i < 4; ++i) {
        a[i] = -(threadIdx.x * 1e-4f + i * 0.01f);
        b[i] = i;
        hh[i] = 0x3c003c00u ^ threadIdx.x;
        iv[i] = threadIdx.x * 7u + i;
        float2 v = make_float2(i, i + 1);
        b2[i] = *reinterpret_cast<unsigned long long *>(&v);
    }
    const long long t0 = clock64();
    for (int it = 0; it < ITERS; ++it) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (KIND == 0 || KIND == 3 || KIND == 6) a[i] = ex2(a[i]);
            if (KIND == 1) a[i] = th(a[i]);
            if (KIND == 2) hh[i] = ex2h2(hh[i]);
#pragma unroll
            for (int k = 0; k < K; ++k) {
                if (KIND == 3 || KIND == 5) b2[i] = ffma2(b2[i], s2, c2);
                else if ((KIND == 6 || KIND == 7) && (k & 1)) iv[i] = (iv[i] ^ 0x9e3779b9u) + (unsigned)k;
                else b[i] = fmaf(b[i], s, 0.25f);
            }
        }
    }
    const long long t1 = clock64();
    float r = 0;
    for (int i = 0; i < 4; ++i) {
        float2 v = *reinterpret_cast<float2 *>(&b2[i]);
        r += a[i] + b[i] + (float)hh[i] + (float)iv[i] + v.x + v.y;
    }
    out[blockIdx.x * blockDim.x + threadIdx.x] = r;
    if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

typedef void (*Kern)(float *, long long *, float);

static void run(const char *name, Kern f, int K, int lanes_per_other, int has_transc, int sms) {
    const int bps = 8, threads = 256, nb = sms * bps;
    float *out;
    long long *cyc;
    cudaMalloc(&out, (size_t)nb * threads * 4);
    cudaMalloc(&cyc, nb * 8);
    f<<<nb, threads>>>(out, cyc, 0.999f);
    f<<<nb, threads>>>(out, cyc, 0.999f);
    cudaError_t e = cudaDeviceSynchronize();
    long long *h = new long long[nb];
    cudaMemcpy(h, cyc, nb * 8, cudaMemcpyDeviceToHost);
    double mx = 0;
    for (int i = 0; i < nb; ++i)
        if (h[i] > mx) mx = h[i];
    const double steps = 4.0 * ITERS * threads * bps;  // chain steps per SM
    printf("%-20s K=%2d  transcendental/clk/SM=%6.2f  other-op lanes/clk/SM=%7.2f  %s\n", name, K,
           has_transc ? steps / mx : 0.0, steps * K * lanes_per_other / mx, cudaGetErrorString(e));
    cudaFree(out);
    cudaFree(cyc);
    delete[] h;
}

int main() {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    cudaDeviceProp p;
    cudaGetDeviceProperties(&p, 0);
    printf("%s: %d SMs, L2 %d MB\n", p.name, sms, p.l2CacheSize >> 20);
    run("ffma", chains<8, 4>, 8, 1, 0, sms);
    run("ffma2 (2 lanes)", chains<8, 5>, 8, 2, 0, sms);
    run("ex2", chains<0, 0>, 0, 1, 1, sms);
    run("ex2 + ffma", chains<2, 0>, 2, 1, 1, sms);
    run("ex2 + ffma", chains<4, 0>, 4, 1, 1, sms);
    run("ex2 + ffma", chains<6, 0>, 6, 1, 1, sms);
    run("ex2 + ffma", chains<8, 0>, 8, 1, 1, sms);
    run("ex2 + ffma", chains<12, 0>, 12, 1, 1, sms);
    run("ex2 + ffma", chains<16, 0>, 16, 1, 1, sms);
    run("ex2 + ffma2", chains<4, 3>, 4, 2, 1, sms);
    run("ex2 + ffma2", chains<8, 3>, 8, 2, 1, sms);
    run("tanh", chains<0, 1>, 0, 1, 1, sms);
    run("tanh + ffma", chains<8, 1>, 8, 1, 1, sms);
    run("ex2.f16x2", chains<0, 2>, 0, 1, 1, sms);
    run("ex2.f16x2 + ffma", chains<8, 2>, 8, 1, 1, sms);
    run("ffma/int mix only", chains<8, 7>, 8, 1, 0, sms);
    run("ex2 + ffma/int mix", chains<8, 6>, 8, 1, 1, sms);
    run("ex2 + ffma/int mix", chains<16, 6>, 16, 1, 1, sms);

    const size_t n = (size_t)1 << 30;
    void *a, *b;
    cudaMalloc(&a, n);
    cudaMalloc(&b, n);
    cudaMemcpy(b, a, n, cudaMemcpyDeviceToDevice);
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    float best = 1e9f;
    for (int i = 0; i < 5; ++i) {
        cudaEventRecord(e0);
        cudaMemcpy(b, a, n, cudaMemcpyDeviceToDevice);
        cudaEventRecord(e1);
        cudaEventSynchronize(e1);
        float ms;
        cudaEventElapsedTime(&ms, e0, e1);
        if (ms < best) best = ms;
    }
    printf("device copy of 1 GiB: %.1f GB/s (bytes read + written)\n", 2.0 * n / best / 1e6);
    cudaFree(a);
    cudaFree(b);
    return 0;
}
