// dt_cumsum.cu -- K2: dt = softplus(dt_raw + dt_bias), dA = dt * a, and the
// per-chunk (64-token) inclusive cumulative sum of dA.
//
// softplus(dt + bias) per head: falcon_mamba.ts header; no dt clamp:
// mojolearn Mamba3Block.  a = A[h] (A = -exp(A_log), codestral_mamba.ts
// reconciliation 2), or per token min(A[b,t,h], -1e-4) (Mamba3Block, "A floor
// 1e-4").  The per-chunk carry factor is exp(sum of the chunk's dA) when no
// document boundary (model card, "Checkpoint and training") falls inside the
// chunk -- including one between the chunk's first token and the previous
// chunk's last -- and 0 otherwise: the state entering such a chunk does not
// reach its end.
//
// One warp per (row, head, chunk): lane l owns tokens l and l+32 of the chunk;
// two shuffle scans give the inclusive sums.  Warps are ordered head-fastest,
// so the warps of one block read neighbouring dt_raw words of the same token
// rows (dt_raw is (batch, seqlen, H)).
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

__device__ __forceinline__ float warp_incl_scan(float v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__global__ void __launch_bounds__(256)
dt_cumsum_kernel(Shape s, const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                 const float* __restrict__ A, const int32_t* __restrict__ seq,
                 float* __restrict__ dt_out, float* __restrict__ acs_out, float* __restrict__ cdecay)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int H = s.nheads, nc = s.nchunks(), L = s.seqlen;
    if (warp >= (int64_t)s.batch * nc * H) return;
    const int h = (int)(warp % H);
    const int c = (int)((warp / H) % nc);
    const int b = (int)(warp / ((int64_t)H * nc));
    const int t0 = c * kChunk;
    const float bias = dt_bias[h];
    const float a_head = s.a_per_token ? 0.0f : A[h];

    float dtv[2], dA[2];
    int bd = 0;
#pragma unroll
    for (int half = 0; half < 2; half++) {
        const int t = t0 + half * 32 + lane;
        dtv[half] = 0.0f;
        dA[half] = 0.0f;
        if (t < L) {
            const int64_t i = ((int64_t)b * L + t) * H + h;
            dtv[half] = softplus_f(dt_raw[i] + bias);
            const float av = s.a_per_token ? fminf(A[i], -kAFloor) : a_head;
            dA[half] = dtv[half] * av;
            bd |= is_boundary(seq ? seq + (int64_t)b * L : nullptr, t);
        }
    }
    const float s0 = warp_incl_scan(dA[0], lane);
    const float tot0 = __shfl_sync(0xffffffffu, s0, 31);
    const float s1 = warp_incl_scan(dA[1], lane) + tot0;

    const int64_t row = ((int64_t)b * H + h) * L;
    if (t0 + lane < L) {
        dt_out[row + t0 + lane] = dtv[0];
        acs_out[row + t0 + lane] = s0;
    }
    if (t0 + 32 + lane < L) {
        dt_out[row + t0 + 32 + lane] = dtv[1];
        acs_out[row + t0 + 32 + lane] = s1;
    }
    if (cdecay != nullptr) {
        const int any_bd = __any_sync(0xffffffffu, bd);
        const int last = (L - t0 < kChunk ? L - t0 : kChunk) - 1;   // chunk-local index
        const float acs_last = __shfl_sync(0xffffffffu, last < 32 ? s0 : s1, last & 31);
        if (lane == 0) cdecay[((int64_t)b * H + h) * nc + c] = any_bd ? 0.0f : expf(acs_last);
    }
}

cudaError_t launch_dt_cumsum(const Shape& s, const FwdArgs& a, float* dt, float* acs,
                             float* cdecay, cudaStream_t st)
{
    const int64_t warps = (int64_t)s.batch * s.nchunks() * s.nheads;
    const int64_t blocks = (warps * 32 + 255) / 256;
    dt_cumsum_kernel<<<(unsigned)blocks, 256, 0, st>>>(s, a.dt_raw, a.dt_bias, a.A, a.seq_idx,
                                                       dt, acs, cdecay);
    return cudaGetLastError();
}

}  // namespace ssd
