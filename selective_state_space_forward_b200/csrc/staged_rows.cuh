// staged_rows.cuh -- per-chunk loads shared by the staged forward kernels and the
// backward kernels: chunk-local document segments and the (64-token) rows of
// x, B and C a block works on, in fp32.
#pragma once
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

// Chunk-local segment ids: seg[t] = boundaries at positions t0 .. t0+t (padding
// positions, at or after the row length Lb, hold none).
__device__ inline void chunk_segments(const int32_t* seq_row, int t0, int Lc, int Lb, int* seg, int* flag)
{
    const int tid = threadIdx.x;
    if (tid < kChunk) flag[tid] = (tid < Lc && t0 + tid < Lb) ? is_boundary(seq_row, t0 + tid) : 0;
    __syncthreads();
    if (tid < kChunk) {
        int acc = 0;
        for (int j = 0; j <= tid; j++) acc += flag[j];
        seg[tid] = acc;
    }
    __syncthreads();
}

// Load token rows [t0, t0+64) of the head's x (fp32 result, zero past the end).
template <typename T>
__device__ void load_x_rows(const Shape& s, const FwdArgs& a, const float* u, int b, int h,
                            int t0, int Lc, float* xs, int ld)
{
    const int P = s.headdim, HP = s.nheads * P, cd = s.conv_dim();
    for (int i = threadIdx.x; i < kChunk * P; i += blockDim.x) {
        const int r = i / P, p = i % P;
        float v = 0.0f;
        if (r < Lc) {
            const int64_t tok = (int64_t)b * s.seqlen + t0 + r;
            v = u ? u[tok * cd + h * P + p] : to_f(((const T*)a.x)[tok * a.ld_x + h * P + p]);
        }
        xs[r * ld + p] = v;
    }
}

// Load B (which = 0) or C (which = 1) rows of the head's group, then apply the
// B/C norm and the head's bias when enabled.
template <typename T>
__device__ void load_bc_rows(const Shape& s, const FwdArgs& a, const float* u, int b, int h,
                             int t0, int Lc, int which, float* dst, int ld)
{
    const int N = s.dstate, GN = s.ngroups * N, HP = s.nheads * s.headdim, cd = s.conv_dim();
    const int g = h / (s.nheads / s.ngroups);
    const T* raw = (const T*)(which ? a.C : a.B);
    for (int i = threadIdx.x; i < kChunk * N; i += blockDim.x) {
        const int r = i / N, n = i % N;
        float v = 0.0f;
        if (r < Lc) {
            const int64_t tok = (int64_t)b * s.seqlen + t0 + r;
            v = u ? u[tok * cd + HP + which * GN + g * N + n] : to_f(raw[tok * a.ld_bc + g * N + n]);
        }
        dst[r * ld + n] = v;
    }
    if (!s.bc_norm) return;
    __syncthreads();
    const float* wn = which ? a.cn_w : a.bn_w;
    const float* bias = which ? a.cn_bias : a.bn_bias;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int r = warp; r < Lc; r += nw) {
        float ss = 0.0f;
        for (int n = lane; n < N; n += 32) ss += dst[r * ld + n] * dst[r * ld + n];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = rsqrtf(ss / N + kNormEps);
        for (int n = lane; n < N; n += 32)
            dst[r * ld + n] = dst[r * ld + n] * rs * (wn ? wn[n] : 1.0f) +
                              (bias ? bias[(int64_t)h * N + n] : 0.0f);
    }
}

}  // namespace ssd
