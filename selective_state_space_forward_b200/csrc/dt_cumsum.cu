// dt_cumsum.cu -- K2: dt = softplus(dt_raw + dt_bias), dA = dt * a, and the
// per-chunk (64-token) segmented inclusive cumulative sum of dA.
//
// softplus(dt + bias) per head: falcon_mamba.ts header; no dt clamp:
// mojolearn Mamba3Block.  a = A[h] (A = -exp(A_log), codestral_mamba.ts
// reconciliation 2), or per token min(A[b,t,h], -1e-4) (Mamba3Block, "A floor
// 1e-4").
//
// The sum restarts at the chunk start and at every packed-document boundary
// inside the chunk (model card, "Checkpoint and training": state flow resets
// at every boundary), so acs_t - acs_s for two tokens of one document sums
// only that document's dA -- a changed document elsewhere in the row cannot
// even change the rounding of another document's decays.  The per-chunk carry
// factor is exp(acs of the chunk's last token) when no boundary falls in the
// chunk -- including one between the chunk's first token and the previous
// chunk's last -- and the reset marker -1 otherwise: the state entering such
// a chunk does not reach its end.
//
// One warp per (row, head, chunk): lane l owns tokens l and l+32 of the chunk;
// two segmented shuffle scans give the inclusive sums.  Warps are ordered
// head-fastest, so the warps of one block read neighbouring dt_raw words of
// the same token rows (dt_raw is (batch, seqlen, H)).
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

// Segmented inclusive scan across the warp: a lane with start = 1 begins a
// new segment.  Returns the sum from the lane's segment start to the lane;
// `start` becomes 1 when a segment start lies at or before the lane.
__device__ __forceinline__ float warp_seg_scan(float v, int& start, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float nv = __shfl_up_sync(0xffffffffu, v, o);
        const int nf = __shfl_up_sync(0xffffffffu, start, o);
        if (lane >= o) {
            if (!start) v = nv + v;
            start |= nf;
        }
    }
    return v;
}

__global__ void __launch_bounds__(256)
dt_cumsum_kernel(Shape s, const void* __restrict__ dt_raw, int64_t ld_dt, int dt_bf16,
                 const float* __restrict__ dt_bias,
                 const float* __restrict__ A, const int32_t* __restrict__ seq,
                 const int32_t* __restrict__ lengths, float* __restrict__ dt_out,
                 float* __restrict__ acs_out, float* __restrict__ cdecay)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int H = s.nheads, nc = s.nchunks(), L = s.seqlen;
    if (warp >= (int64_t)s.batch * nc * H) return;
    const int h = (int)(warp % H);
    const int c = (int)((warp / H) % nc);
    const int b = (int)(warp / ((int64_t)H * nc));
    const int t0 = c * kChunk;
    const int Lb = row_length(lengths, b, L);   // padding: dt = 0, no boundary
    const float bias = dt_bias[h];
    const float a_head = s.a_per_token ? 0.0f : A[h];

    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    float dtv[2], dA[2];
    int bd[2];
#pragma unroll
    for (int half = 0; half < 2; half++) {
        const int t = t0 + half * 32 + lane;
        dtv[half] = 0.0f;
        dA[half] = 0.0f;
        bd[half] = 0;
        if (t < Lb) {
            const int64_t i = ((int64_t)b * L + t) * H + h;
            const int64_t id = ((int64_t)b * L + t) * ld_dt + h;
            const float raw = dt_bf16 ? to_f(((const bf16*)dt_raw)[id]) : ((const float*)dt_raw)[id];
            dtv[half] = softplus_f(raw + bias);
            const float av = s.a_per_token ? fminf(A[i], -kAFloor) : a_head;
            dA[half] = dtv[half] * av;
            bd[half] = is_boundary(seq_row, t);
        }
    }
    const int any_bd = __any_sync(0xffffffffu, bd[0] | bd[1]);
    int f0 = bd[0] | (lane == 0);   // the chunk start opens a segment
    int f1 = bd[1];
    const float s0 = warp_seg_scan(dA[0], f0, lane);
    float s1 = warp_seg_scan(dA[1], f1, lane);
    const float tail0 = __shfl_sync(0xffffffffu, s0, 31);
    if (!f1) s1 = tail0 + s1;       // no segment start in tokens 32 .. lane+32

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
        const int last = (L - t0 < kChunk ? L - t0 : kChunk) - 1;   // chunk-local index
        const float acs_last = __shfl_sync(0xffffffffu, last < 32 ? s0 : s1, last & 31);
        if (lane == 0) cdecay[((int64_t)b * H + h) * nc + c] = any_bd ? kChunkReset : expf(acs_last);
    }
}

cudaError_t launch_dt_cumsum(const Shape& s, const FwdArgs& a, float* dt, float* acs,
                             float* cdecay, cudaStream_t st)
{
    const int64_t warps = (int64_t)s.batch * s.nchunks() * s.nheads;
    const int64_t blocks = (warps * 32 + 255) / 256;
    dt_cumsum_kernel<<<(unsigned)blocks, 256, 0, st>>>(s, a.dt_raw, a.ld_dt, a.dt_act, a.dt_bias, a.A, a.seq_idx,
                                                       a.lengths, dt, acs, cdecay);
    return cudaGetLastError();
}

}  // namespace ssd
