// finite.cu -- the validate_finite check: raises a bit in the device status
// word when a result holds a NaN or an infinity.
//
// A value is non-finite when its exponent field is all ones (bf16: bits 7..14
// of each 16-bit half; fp32: bits 23..30).  The data is read as 16-byte
// vectors; every result buffer of the library is a multiple of 16 bytes long
// and 16-byte aligned.  One atomic per warp that saw a bad value.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

template <bool BF16>
__global__ void __launch_bounds__(256)
finite_check_kernel(const uint4* __restrict__ v, size_t nvec, int* __restrict__ status)
{
    bool bad = false;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        const uint4 w = v[i];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            if (BF16)
                bad |= ((ws[k] & 0x7F80u) == 0x7F80u) || ((ws[k] & 0x7F800000u) == 0x7F800000u);
            else
                bad |= (ws[k] & 0x7F800000u) == 0x7F800000u;
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kStatusNonFinite);
}

cudaError_t launch_finite_check(const void* data, size_t bytes, bool bf16, int* status, cudaStream_t st)
{
    if (bytes == 0) return cudaSuccess;
    if (bytes % 16 || ((uintptr_t)data % 16)) return cudaErrorInvalidValue;
    const size_t nvec = bytes / 16;
    size_t blocks = (nvec + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (bf16)
        finite_check_kernel<true><<<(unsigned)blocks, 256, 0, st>>>((const uint4*)data, nvec, status);
    else
        finite_check_kernel<false><<<(unsigned)blocks, 256, 0, st>>>((const uint4*)data, nvec, status);
    return cudaGetLastError();
}

}  // namespace ssd
