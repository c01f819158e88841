// gated_norm.cu -- the gated RMSNorm that follows the scan in the upstream
// Mamba-2 block: out <- norm(y * SiLU(z)) = g * w / sqrt(mean(g^2) + eps).
//
// codestral_mamba.ts header: the layer holds `mixer.norm.weight [d_inner]`,
// and reconciliation 3 names the upstream order, the norm applied to
// y * silu(z).  The gated product g is what the scan writes to `out`, so the
// norm rewrites `out` in place.  The mean runs over a group of `gs`
// consecutive channels (gs = d_inner: one norm per token; upstream's grouped
// variant uses d_inner / ngroups).
//
// Groups of up to 2048 channels take one warp each (gated_norm_warp_kernel, its
// register footprint sized to the group);
// wider ones one block per (token, group): each thread holds up to kVecPerThread
// 8-channel vectors of the group in registers, the sum of squares is reduced in a fixed
// order (warp shuffles, then the warps in turn), and every vector is scaled
// and written back.  Tokens past a ragged row's length are left untouched, so
// their +0.0 padding stays +0.0.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kVecPerThread = 8;

template <typename T>
__global__ void __launch_bounds__(256)
gated_norm_kernel(Shape s, void* out_, const float* __restrict__ weight, int gs, float eps,
                  const int32_t* __restrict__ lengths)
{
    __shared__ float red[8];
    const int HP = s.nheads * s.headdim, L = s.seqlen;
    const int64_t tok = blockIdx.x;
    const int grp = blockIdx.y;
    const int b = (int)(tok / L), t = (int)(tok % L);
    if (t >= row_length(lengths, b, L)) return;          // padding stays +0.0
    T* row = (T*)out_ + tok * HP + (int64_t)grp * gs;
    const float* wr = weight ? weight + (int64_t)grp * gs : nullptr;
    const int nvec = gs / 8;
    float v[kVecPerThread][8];
    float ss = 0.0f;
#pragma unroll
    for (int k = 0; k < kVecPerThread; k++) {
        const int i = threadIdx.x + k * blockDim.x;
        if (i < nvec) {
            load8(row + (int64_t)i * 8, v[k]);
#pragma unroll
            for (int j = 0; j < 8; j++) ss = fmaf(v[k][j], v[k][j], ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
    for (int i = 0; i < (int)(blockDim.x >> 5); i++) tot += red[i];
    const float r = rsqrtf(tot / gs + eps);
#pragma unroll
    for (int k = 0; k < kVecPerThread; k++) {
        const int i = threadIdx.x + k * blockDim.x;
        if (i < nvec) {
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; j++) o[j] = v[k][j] * r * (wr ? wr[i * 8 + j] : 1.0f);
            store8(row + (int64_t)i * 8, o);
        }
    }
}

// Groups of at most 2048 channels: one warp per (token, group), eight warps per
// block; each lane holds VPL 8-channel vectors (VPL = the group's vectors / 32,
// rounded up to a power of two, so a small group keeps few registers and many
// warps in flight), the warp reduces by xor shuffles (a fixed order) and writes
// the scaled group back.
template <typename T, int VPL>
__global__ void __launch_bounds__(256)
gated_norm_warp_kernel(Shape s, void* out_, const float* __restrict__ weight, int gs, float eps,
                       const int32_t* __restrict__ lengths)
{
    const int HP = s.nheads * s.headdim, L = s.seqlen, ngrp = HP / gs;
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= (int64_t)s.batch * L * ngrp) return;
    const int64_t tok = wid / ngrp;
    const int grp = (int)(wid % ngrp);
    const int b = (int)(tok / L), t = (int)(tok % L);
    if (t >= row_length(lengths, b, L)) return;          // padding stays +0.0
    T* row = (T*)out_ + tok * HP + (int64_t)grp * gs;
    const float* wr = weight ? weight + (int64_t)grp * gs : nullptr;
    const int nvec = gs / 8;
    float v[VPL][8];
    float ss = 0.0f;
#pragma unroll
    for (int k = 0; k < VPL; k++) {
        const int i = lane + 32 * k;
        if (i < nvec) {
            load8(row + (int64_t)i * 8, v[k]);
#pragma unroll
            for (int j = 0; j < 8; j++) ss = fmaf(v[k][j], v[k][j], ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / gs + eps);
#pragma unroll
    for (int k = 0; k < VPL; k++) {
        const int i = lane + 32 * k;
        if (i < nvec) {
            float wv[8];
            if (wr) load8(wr + (int64_t)i * 8, wv);
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; j++) o[j] = v[k][j] * r * (wr ? wv[j] : 1.0f);
            store8(row + (int64_t)i * 8, o);
        }
    }
}

bool gated_norm_group_ok(int d_inner, int gs)
{
    return gs >= 8 && gs % 8 == 0 && d_inner % gs == 0 && gs / 8 <= 256 * kVecPerThread;
}

cudaError_t launch_gated_norm(const Shape& s, void* out, const float* weight, int gs, float eps,
                              const int32_t* lengths, cudaStream_t st)
{
    const int HP = s.nheads * s.headdim;
    if (!gated_norm_group_ok(HP, gs)) return cudaErrorInvalidValue;
    const int nvec = gs / 8;
    if (nvec <= 32 * kVecPerThread) {
        const int64_t warps = (int64_t)s.batch * s.seqlen * (HP / gs);
        const unsigned blocks = (unsigned)((warps + 7) / 8);
        const int vpl = nvec <= 32 ? 1 : nvec <= 64 ? 2 : nvec <= 128 ? 4 : 8;
#define SSD_GN(TT, VV) gated_norm_warp_kernel<TT, VV><<<blocks, 256, 0, st>>>(s, out, weight, gs, eps, lengths)
        if (s.act_bf16) {
            switch (vpl) {
            case 1: SSD_GN(bf16, 1); break;
            case 2: SSD_GN(bf16, 2); break;
            case 4: SSD_GN(bf16, 4); break;
            default: SSD_GN(bf16, 8); break;
            }
        } else {
            switch (vpl) {
            case 1: SSD_GN(float, 1); break;
            case 2: SSD_GN(float, 2); break;
            case 4: SSD_GN(float, 4); break;
            default: SSD_GN(float, 8); break;
            }
        }
#undef SSD_GN
        return cudaGetLastError();
    }
    int threads = (nvec + kVecPerThread - 1) / kVecPerThread;
    threads = ((threads + 31) / 32) * 32;
    if (threads > 256) threads = 256;
    const dim3 grid((unsigned)((int64_t)s.batch * s.seqlen), (unsigned)(HP / gs));
    if (s.act_bf16)
        gated_norm_kernel<bf16><<<grid, threads, 0, st>>>(s, out, weight, gs, eps, lengths);
    else
        gated_norm_kernel<float><<<grid, threads, 0, st>>>(s, out, weight, gs, eps, lengths);
    return cudaGetLastError();
}

}  // namespace ssd
