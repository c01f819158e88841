// probe.cu -- a measurement aid: the device's throughput of the hardware
// base-2 exponential (PTX ex2.approx, the MUFU pipe), which bounds the
// Mamba-1 selective scan (one exponential per state and token).  Every thread
// runs eight independent chains v <- 2^(-0.999 v), which settle near 0.64, so
// the pipe stays fed without overflow; the multiply goes to the FMA pipe.
#include <cuda_runtime.h>

#include "ssd.h"
#include "ssd_device.cuh"

namespace ssd {

constexpr int kEx2Chains = 8;

__global__ void __launch_bounds__(256) ex2_rate_kernel(int iters, float* sink)
{
    float v[kEx2Chains];
#pragma unroll
    for (int j = 0; j < kEx2Chains; j++) v[j] = 0.01f * (threadIdx.x & 31) + 0.1f * j;
    for (int i = 0; i < iters; i++) {
#pragma unroll
        for (int j = 0; j < kEx2Chains; j++) v[j] = ex2(-0.999f * v[j]);
    }
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < kEx2Chains; j++) acc += v[j];
    if (acc == -1.0f) sink[threadIdx.x] = acc;   // never true: keeps the chains live
}

}  // namespace ssd

extern "C" ssd_status ssd_ex2_throughput(double* results_per_second, struct CUstream_st* stream)
{
    if (!results_per_second) return SSD_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SSD_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    const int blocks = sms * 8, threads = 256, iters = 4096;
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess) return SSD_ERR_CUDA;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0);
        return SSD_ERR_CUDA;
    }
    ssd::ex2_rate_kernel<<<blocks, threads, 0, st>>>(iters, nullptr);   // warm-up
    cudaEventRecord(e0, st);
    ssd::ex2_rate_kernel<<<blocks, threads, 0, st>>>(iters, nullptr);
    cudaEventRecord(e1, st);
    const cudaError_t err = cudaEventSynchronize(e1);
    float ms = 0.0f;
    if (err == cudaSuccess) cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (err != cudaSuccess || cudaGetLastError() != cudaSuccess || ms <= 0.0f) return SSD_ERR_CUDA;
    *results_per_second = (double)blocks * threads * iters * ssd::kEx2Chains / (ms * 1e-3);
    return SSD_OK;
}
