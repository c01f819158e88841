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

// One block per (row, chunk, block of kHeadBlk heads), 256 threads.  The chunk's
// dt_raw (and per-token A) rows are read coalesced -- consecutive threads take
// consecutive heads of a token row, every thread's loads issued before any is
// used -- turned into dt and dA in shared memory, and then each warp scans whole
// heads: lane l owns tokens l and l+32 of the chunk, and the two segmented
// shuffle scans give the inclusive sums.  dt and acs are written head-major, 64
// consecutive floats per head.
constexpr int kHeadBlk = 64;
constexpr int kPerThread = kChunk * kHeadBlk / 256;

__global__ void __launch_bounds__(256, 2)
dt_cumsum_kernel(Shape s, const void* __restrict__ dt_raw, int64_t ld_dt, int dt_bf16,
                 const float* __restrict__ dt_bias,
                 const float* __restrict__ A, const int32_t* __restrict__ seq,
                 const int32_t* __restrict__ lengths, float* __restrict__ dt_out,
                 float* __restrict__ acs_out, float* __restrict__ cdecay)
{
    __shared__ float s_dt[kChunk][kHeadBlk + 1], s_da[kChunk][kHeadBlk + 1];
    __shared__ int s_bd[kChunk];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = s.nheads, nc = s.nchunks(), L = s.seqlen;
    const int nhb = (H + kHeadBlk - 1) / kHeadBlk;
    const int hb = blockIdx.x % nhb, c = (blockIdx.x / nhb) % nc, b = blockIdx.x / (nhb * nc);
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0);
    const int Lb = row_length(lengths, b, L);   // padding: dt = 0, no boundary
    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    if (tid < kChunk) s_bd[tid] = (tid < Lc && t0 + tid < Lb) ? is_boundary(seq_row, t0 + tid) : 0;
    const int last = Lc - 1;
    const int h0 = hb * kHeadBlk, nh = min(kHeadBlk, H - h0);
    float raw[kPerThread], av[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; k++) {
        const int e = tid + k * 256;
        const int r = e / kHeadBlk, hh = e % kHeadBlk;
        const int t = t0 + r, h = h0 + hh;
        const bool ok = hh < nh && r < Lc && t < Lb;
        const int64_t tok = (int64_t)b * L + t;
        raw[k] = !ok ? 0.0f
                     : dt_bf16 ? to_f(((const bf16*)dt_raw)[tok * ld_dt + h]) : ((const float*)dt_raw)[tok * ld_dt + h];
        av[k] = !ok ? 0.0f : s.a_per_token ? A[tok * H + h] : A[h];
    }
#pragma unroll
    for (int k = 0; k < kPerThread; k++) {
        const int e = tid + k * 256;
        const int r = e / kHeadBlk, hh = e % kHeadBlk;
        const int t = t0 + r, h = h0 + hh;
        float dtv = 0.0f, dA = 0.0f;
        if (hh < nh && r < Lc && t < Lb) {
            dtv = softplus_f(raw[k] + dt_bias[h]);
            dA = dtv * (s.a_per_token ? fminf(av[k], -kAFloor) : av[k]);
        }
        s_dt[r][hh] = dtv;
        s_da[r][hh] = dA;
    }
    __syncthreads();
    for (int hh = warp; hh < nh; hh += (int)(blockDim.x >> 5)) {
        const int h = h0 + hh;
        const int bd0 = s_bd[lane], bd1 = s_bd[lane + 32];
        const int any_bd = __any_sync(0xffffffffu, bd0 | bd1);
        int f0 = bd0 | (lane == 0);         // the chunk start opens a segment
        int f1 = bd1;
        const float s0 = warp_seg_scan(s_da[lane][hh], f0, lane);
        float s1 = warp_seg_scan(s_da[lane + 32][hh], f1, lane);
        const float tail0 = __shfl_sync(0xffffffffu, s0, 31);
        if (!f1) s1 = tail0 + s1;           // no segment start in tokens 32 .. lane+32
        const int64_t row = ((int64_t)b * H + h) * L;
        if (lane < Lc) {
            dt_out[row + t0 + lane] = s_dt[lane][hh];
            acs_out[row + t0 + lane] = s0;
        }
        if (lane + 32 < Lc) {
            dt_out[row + t0 + 32 + lane] = s_dt[lane + 32][hh];
            acs_out[row + t0 + 32 + lane] = s1;
        }
        if (cdecay != nullptr) {
            const float acs_last = __shfl_sync(0xffffffffu, last < 32 ? s0 : s1, last & 31);
            if (lane == 0) cdecay[((int64_t)b * H + h) * nc + c] = any_bd ? kChunkReset : expf(acs_last);
        }
    }
}

cudaError_t launch_dt_cumsum(const Shape& s, const FwdArgs& a, float* dt, float* acs,
                             float* cdecay, cudaStream_t st)
{
    const int64_t blocks = (int64_t)s.batch * s.nchunks() * ((s.nheads + kHeadBlk - 1) / kHeadBlk);
    dt_cumsum_kernel<<<(unsigned)blocks, 256, 0, st>>>(s, a.dt_raw, a.ld_dt, a.dt_act, a.dt_bias, a.A,
                                                       a.seq_idx, a.lengths, dt, acs, cdecay);
    return cudaGetLastError();
}

}  // namespace ssd
