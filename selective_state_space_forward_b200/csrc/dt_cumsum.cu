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

// One block per (row, chunk, block of kHeadBlk heads), 256 threads.  The chunk's
// dt_raw (and per-token A) rows are read coalesced -- consecutive threads take
// consecutive heads of a token row, every thread's loads issued before any is
// used -- turned into dt and dA in shared memory.  Then thread (part q, head
// hh) sums dA over tokens 16q .. 16q+15 of head hh in token order, restarting
// at each boundary (a 64-bit mask of the chunk's boundaries, built by ballot),
// and adds the carry of the parts before it -- their tails back to and
// including the first part that holds a boundary -- to its tokens before its
// own first boundary.  dt and acs are written head-major, 16 consecutive
// floats per thread (four 16-byte stores when the row allows).
constexpr int kHeadBlk = 64;
constexpr int kPerThread = kChunk * kHeadBlk / 256;
constexpr int kParts = 256 / kHeadBlk;          // token parts per head
constexpr int kPartLen = kChunk / kParts;       // 16 tokens
static_assert(kPartLen == 16, "the part masks are 16 bits wide");

// Four blocks per SM (64 registers): the kernel is bound by the issue of its
// softplus and staging instructions, so it needs the resident warps.
__global__ void __launch_bounds__(256, 4)
dt_cumsum_kernel(Shape s, const void* __restrict__ dt_raw, int64_t ld_dt, int dt_bf16,
                 const float* __restrict__ dt_bias,
                 const float* __restrict__ A, const int32_t* __restrict__ seq,
                 const int32_t* __restrict__ lengths, float* __restrict__ dt_out,
                 float* __restrict__ acs_out, float* __restrict__ cdecay)
{
    __shared__ float s_dt[kChunk][kHeadBlk + 1], s_da[kChunk][kHeadBlk + 1];
    __shared__ float s_tail[kParts][kHeadBlk];
    __shared__ uint32_t s_bm[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = s.nheads, nc = s.nchunks(), L = s.seqlen;
    const int nhb = (H + kHeadBlk - 1) / kHeadBlk;
    const int hb = blockIdx.x % nhb, c = (blockIdx.x / nhb) % nc, b = blockIdx.x / (nhb * nc);
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0);
    const int Lb = row_length(lengths, b, L);   // padding: dt = 0, no boundary
    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    if (warp < 2) {
        const int r = warp * 32 + lane;
        const int bd = (r < Lc && t0 + r < Lb) ? is_boundary(seq_row, t0 + r) : 0;
        const uint32_t m = __ballot_sync(0xffffffffu, bd);
        if (lane == 0) s_bm[warp] = m;
    }
    // Every element a thread stages belongs to one head (its index mod 64), so
    // the head's bias and A are loaded once; rows are kRowStep tokens apart.
    const int h0 = hb * kHeadBlk, nh = min(kHeadBlk, H - h0);
    const int hs = tid % kHeadBlk, rs = tid / kHeadBlk;
    constexpr int kRowStep = 256 / kHeadBlk;
    const bool head_ok = hs < nh;
    const float bias = head_ok ? dt_bias[h0 + hs] : 0.0f;
    const float a_head = (head_ok && !s.a_per_token) ? A[h0 + hs] : 0.0f;
    const int64_t tok0 = (int64_t)b * L + t0 + rs;
    float raw[kPerThread], av[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; k++) {
        const int r = rs + k * kRowStep;
        const bool ok = head_ok && r < Lc && t0 + r < Lb;
        const int64_t tok = tok0 + k * kRowStep;
        raw[k] = !ok ? 0.0f
                     : dt_bf16 ? to_f(((const bf16*)dt_raw)[tok * ld_dt + h0 + hs])
                               : ((const float*)dt_raw)[tok * ld_dt + h0 + hs];
        av[k] = (ok && s.a_per_token) ? A[tok * H + h0 + hs] : a_head;
    }
#pragma unroll
    for (int k = 0; k < kPerThread; k++) {
        const int r = rs + k * kRowStep;
        float dtv = 0.0f, dA = 0.0f;
        if (head_ok && r < Lc && t0 + r < Lb) {
            dtv = softplus_f(raw[k] + bias);
            dA = dtv * (s.a_per_token ? fminf(av[k], -kAFloor) : av[k]);
        }
        s_dt[r][hs] = dtv;
        s_da[r][hs] = dA;
    }
    __syncthreads();

    const uint64_t bm = (uint64_t)s_bm[0] | ((uint64_t)s_bm[1] << 32);
    const int hh = tid % kHeadBlk, q = tid / kHeadBlk, r0 = q * kPartLen;
    const uint32_t pm = (uint32_t)(bm >> r0) & 0xffffu;      // boundaries in this part
    float v[kPartLen];
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < kPartLen; i++) {
        const float d = s_da[r0 + i][hh];
        acc = ((pm >> i) & 1u) ? d : acc + d;
        v[i] = acc;
    }
    s_tail[q][hh] = acc;
    __syncthreads();
    if (q > 0) {
        // the segment open at this part's first token began in an earlier part
        float carry = 0.0f;
        for (int p = q - 1; p >= 0; p--) {
            carry += s_tail[p][hh];
            if (p == 0 || ((bm >> (p * kPartLen)) & 0xffffu) != 0) break;
        }
        const int open = pm ? __ffs(pm) - 1 : kPartLen;      // tokens before the first boundary
#pragma unroll
        for (int i = 0; i < kPartLen; i++)
            if (i < open) v[i] = carry + v[i];
    }
    if (hh >= nh || r0 >= Lc) return;
    const int64_t row = ((int64_t)b * H + h0 + hh) * L + t0 + r0;
    float* dst_dt = dt_out + row;
    float* dst_acs = acs_out + row;
    if (r0 + kPartLen <= Lc && ((reinterpret_cast<uintptr_t>(dst_dt) | reinterpret_cast<uintptr_t>(dst_acs)) & 15) == 0) {
#pragma unroll
        for (int i = 0; i < kPartLen; i += 4) {
            *reinterpret_cast<float4*>(dst_dt + i) =
                make_float4(s_dt[r0 + i][hh], s_dt[r0 + i + 1][hh], s_dt[r0 + i + 2][hh], s_dt[r0 + i + 3][hh]);
            *reinterpret_cast<float4*>(dst_acs + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < kPartLen; i++) {
            if (r0 + i < Lc) {
                dst_dt[i] = s_dt[r0 + i][hh];
                dst_acs[i] = v[i];
            }
        }
    }
    if (cdecay != nullptr) {
        const int last = Lc - 1;
        if (last / kPartLen == q) {
            float acs_last = 0.0f;
#pragma unroll
            for (int i = 0; i < kPartLen; i++)
                if (i == last % kPartLen) acs_last = v[i];
            cdecay[((int64_t)b * H + h0 + hh) * nc + c] = bm ? kChunkReset : expf(acs_last);
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
