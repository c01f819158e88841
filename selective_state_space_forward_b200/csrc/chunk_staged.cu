// chunk_staged.cu -- the staged path's K3 (chunk states), K4 (state passing)
// and K5 (chunk outputs): fp32 accumulation throughout; the contractions of K3
// and K5 run on the tensor cores (tf32 operands) for bf16 activations and as
// register-tiled fp32 products for fp32 activations.
//
// The chunked evaluation of the selective scan (chunk 64; mojolearn
// Mamba3Block, "chunk size 64"): within a chunk c of tokens t0 .. t0+Lc-1,
// with acs_t the inclusive sum of dt*a from the start of t's segment (the
// chunk start or the last document boundary) and seg_t the number of document
// boundaries at positions t0 .. t (a boundary at t0 means the token before the
// chunk belongs to another document):
//
//   chunk state    S_c[p,n]  = sum_{s: seg_s = seg_last} exp(acs_last - acs_s) dt_s x_s[p] B_s[n]
//   state passing  Hin_0     = initial state;  Hin_{c+1} = k_c Hin_c + S_c,
//                  k_c = exp(acs_last) if the chunk holds no boundary, else Hin_c is
//                  dropped (Hin_{c+1} = S_c)
//   chunk output   y_t[p]    = sum_{s<=t, seg_s = seg_t} (C_t . B_s) exp(acs_t - acs_s) dt_s x_s[p]
//                            + [seg_t = 0] exp(acs_t) C_t . Hin_c[p, :]  +  D x_t[p]
//                  out_t     = y_t * SiLU(z_t)
//
// which is the recurrence h_t = exp(dt_t a_t) h_{t-1} + dt_t x_t B_t^T,
// y_t = C_t h_t + D x_t split at chunk boundaries, with the state restarting at
// every packed-document boundary (model card, "Checkpoint and training").
// x, B, C are the conv+SiLU outputs when the conv is on (u from K1, fp32),
// else the raw inputs; B and C are RMS-normalised and given the head's bias
// when the B/C norm is on (Mamba3Block class description).
#include "ssd_device.cuh"
#include "ssd_kernels.h"
#include "staged_rows.cuh"

namespace ssd {

template <typename T, int TC>
__global__ void __launch_bounds__(256)
chunk_state_kernel(Shape s, FwdArgs a, const float* __restrict__ u, const float* __restrict__ dt,
                   const float* __restrict__ acs, float* __restrict__ states)
{
    extern __shared__ float sm[];
    const int P = s.headdim, N = s.dstate, H = s.nheads, L = s.seqlen, nc = s.nchunks();
    const int XS = P + kPad, NB = N + kPad;  // padded row strides (bank spread)
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0);
    float* xs = sm;                    // [64][XS], pre-scaled by the token weight
    float* bs = xs + kChunk * XS;      // [64][NB]
    float* wv = bs + kChunk * NB;      // [64]
    int* seg = (int*)(wv + kChunk);    // [64]
    int* flag = seg + kChunk;          // [64]

    chunk_segments(a.seq_idx ? a.seq_idx + (int64_t)b * L : nullptr, t0, Lc,
                   row_length(a.lengths, b, L), seg, flag);
    const float* dtr = dt + ((int64_t)b * H + h) * L + t0;
    const float* acr = acs + ((int64_t)b * H + h) * L + t0;
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        wv[r] = (r < Lc && seg[r] == seg[Lc - 1]) ? expf(acr[Lc - 1] - acr[r]) * dtr[r] : 0.0f;
    }
    load_x_rows<T>(s, a, u, b, h, t0, Lc, xs, XS);
    load_bc_rows<T>(s, a, u, b, h, t0, Lc, 0, bs, NB);
    __syncthreads();
    for (int i = threadIdx.x; i < kChunk * P; i += blockDim.x) xs[(i / P) * XS + i % P] *= wv[i / P];
    __syncthreads();

    // S[p][n] = sum_r xs[r][p] B[r][n] in 64 x 16 TC output blocks (rows past the
    // chunk's end are zero in both operands)
    float* dst = states + (((int64_t)b * nc + c) * H + h) * P * N;
    const Prod<T, TC> pr(threadIdx.x);
    for (int p0 = 0; p0 < P; p0 += 64)
        for (int n0 = 0; n0 < N; n0 += 16 * TC) {
            float acc[4][TC];
            tile_zero(acc);
            pr.mm(acc, xs + p0, 1, XS, P - p0, bs + n0, NB, 1, N - n0, kChunk);
#pragma unroll
            for (int rr = 0; rr < 4; rr++)
#pragma unroll
                for (int cc = 0; cc < TC; cc++) {
                    const int pp = p0 + pr.row(rr, cc), n = n0 + pr.col(rr, cc);
                    if (pp < P && n < N) dst[pp * N + n] = acc[rr][cc];
                }
        }
}

// One thread per state element (row, head, p, n), walking the chunks in order.
// Reads the initial state before writing the final one, so they may alias.
__global__ void __launch_bounds__(256)
state_passing_kernel(Shape s, const float* __restrict__ cdecay, float* __restrict__ states,
                     const float* init, float* fin)
{
    const int PN = s.headdim * s.dstate, H = s.nheads, nc = s.nchunks();
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)s.batch * H * PN) return;
    const int e = (int)(gid % PN);
    const int h = (int)((gid / PN) % H);
    const int b = (int)(gid / ((int64_t)PN * H));
    float hv = init ? init[gid] : 0.0f;
    const float* kd = cdecay + ((int64_t)b * H + h) * nc;
    float* sp = states + ((int64_t)b * nc * H + h) * PN + e;     // chunk c at sp + c * cs
    const int64_t cs = (int64_t)H * PN;
    // the chunk states and carries of the next kAhead chunks are in flight while
    // the chain advances (each thread's loads are independent of its chain)
    constexpr int kAhead = 8;
    float pre[kAhead], kpre[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; i++) {
        pre[i] = i < nc ? sp[i * cs] : 0.0f;
        kpre[i] = i < nc ? kd[i] : 0.0f;
    }
    for (int c0 = 0; c0 < nc; c0 += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; i++) {
            const int c = c0 + i;
            if (c < nc) {
                const float sc = pre[i], k = kpre[i];
                if (c + kAhead < nc) {
                    pre[i] = sp[(c + kAhead) * cs];
                    kpre[i] = kd[c + kAhead];
                }
                sp[c * cs] = hv;
                hv = (k == kChunkReset) ? sc : k * hv + sc;   // select: a reset drops hv exactly
            }
        }
    }
    if (fin) fin[gid] = hv;
}

// Per (chunk, head): the three contractions of the chunk output go through the
// per-dtype product engine (tf32 tensor-core tiles for bf16 activations,
// register-tiled fp32 for fp32), 64 x 64 output blocks:
//   (C_t . B_s) on the causal same-segment mask, times exp(acs_t - acs_s);
//   sum_s [that] dt_s x_s[p]           (dt_s scales the reduction index);
//   C_t . Hin_c[p, :]                  (Hin_c takes B's tile once C B^T is done).
template <typename T>
__global__ void __launch_bounds__(256)
chunk_output_kernel(Shape s, FwdArgs a, const float* __restrict__ u, const float* __restrict__ dt,
                    const float* __restrict__ acs, const float* __restrict__ hin)
{
    extern __shared__ float sm[];
    const int P = s.headdim, N = s.dstate, H = s.nheads, L = s.seqlen, nc = s.nchunks();
    const int HP = H * P, NB = N + kPad, XS = P + kPad;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0);
    float* cs = sm;                             // [64][NB]          C
    float* bs = cs + kChunk * NB;               // [max(64, P)][NB]  B, then Hin_c ([P][NB])
    float* xs = bs + max(kChunk, P) * NB;       // [64][XS]          x
    float* cbe = xs + kChunk * XS;              // [64][kMS]         (C_t . B_s) E[t,s] on the mask
    float* ac = cbe + kChunk * kMS;             // [64]
    float* dv = ac + kChunk;                    // [64]
    float* ft = dv + kChunk;                    // [64] weight of the carried-state term
    int* seg = (int*)(ft + kChunk);             // [64]
    int* flag = seg + kChunk;                   // [64]

    const int Lb = row_length(a.lengths, b, L);
    chunk_segments(a.seq_idx ? a.seq_idx + (int64_t)b * L : nullptr, t0, Lc, Lb, seg, flag);
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        const int64_t o = ((int64_t)b * H + h) * L + t0 + r;
        ac[r] = r < Lc ? acs[o] : 0.0f;
        dv[r] = r < Lc ? dt[o] : 0.0f;
    }
    load_x_rows<T>(s, a, u, b, h, t0, Lc, xs, XS);
    load_bc_rows<T>(s, a, u, b, h, t0, Lc, 1, cs, NB);
    load_bc_rows<T>(s, a, u, b, h, t0, Lc, 0, bs, NB);
    __syncthreads();
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        ft[r] = (r < Lc && seg[r] == 0) ? expf(ac[r]) : 0.0f;
    }

    const Prod<T, 4> p4(threadIdx.x);
    {
        float acc[4][4];
        tile_zero(acc);
        p4.mm(acc, cs, NB, 1, kChunk, bs, 1, NB, kChunk, N);
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int t = p4.row(rr, cc), r = p4.col(rr, cc);
                cbe[t * kMS + r] = (r <= t && t < Lc && seg[r] == seg[t]) ? acc[rr][cc] * expf(ac[t] - ac[r]) : 0.0f;
            }
    }
    __syncthreads();                            // B's tile has been read
    load_rows8(hin + (((int64_t)b * nc + c) * H + h) * P * N, N, N, P, bs, NB, P);
    __syncthreads();

    const float Dh = a.D[h];
    for (int p0 = 0; p0 < P; p0 += 64) {
        float ys[4][4], off[4][4];
        tile_zero(ys);
        tile_zero(off);
        p4.mm(ys, cbe, kMS, 1, kChunk, xs + p0, XS, 1, P - p0, kChunk, dv);   // sum_s M[t,s] x_s
        p4.mm(off, cs, NB, 1, kChunk, bs + p0 * NB, 1, NB, P - p0, N);        // C_t . Hin[p]
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int t = p4.row(rr, cc), p = p0 + p4.col(rr, cc);
                if (t >= Lc || p >= P) continue;
                const int64_t o = ((int64_t)b * L + t0 + t) * HP + h * P + p;
                if (t0 + t >= Lb) {   // padding of a ragged row
                    ((T*)a.out)[o] = from_f<T>(0.0f);
                    continue;
                }
                float y = ys[rr][cc];
                if (seg[t] == 0) y += ft[t] * off[rr][cc];
                y += Dh * xs[t * XS + p];
                const float zv = to_f(((const T*)a.z)[((int64_t)b * L + t0 + t) * a.ld_z + h * P + p]);
                ((T*)a.out)[o] = from_f<T>(y * silu_f(zv));
            }
    }
}

size_t chunk_state_smem_bytes(const Shape& s)
{
    return sizeof(float) * ((size_t)kChunk * (s.headdim + kPad) + (size_t)kChunk * (s.dstate + kPad) + kChunk) +
           sizeof(int) * 2 * kChunk;
}

size_t chunk_output_smem_bytes(const Shape& s)
{
    const size_t N = s.dstate, P = s.headdim, NB = N + kPad, XS = P + kPad;
    const size_t rows_b = P > (size_t)kChunk ? P : (size_t)kChunk;
    return sizeof(float) * (kChunk * NB + rows_b * NB + kChunk * XS + kChunk * kMS + 3 * kChunk) +
           sizeof(int) * 2 * kChunk;
}

cudaError_t launch_chunk_state(const Shape& s, const FwdArgs& a, const float* u,
                               const float* dt, const float* acs, float* states, cudaStream_t st)
{
    const dim3 grid(s.nchunks(), s.nheads, s.batch);
    const size_t smem = chunk_state_smem_bytes(s);
    // output blocks of 64 x 64 for d_state <= 64, else 64 x 128
    void (*kern)(Shape, FwdArgs, const float*, const float*, const float*, float*) =
        s.act_bf16 ? (s.dstate > 64 ? chunk_state_kernel<bf16, 8> : chunk_state_kernel<bf16, 4>)
                   : (s.dstate > 64 ? chunk_state_kernel<float, 8> : chunk_state_kernel<float, 4>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 256, smem, st>>>(s, a, u, dt, acs, states);
    return cudaGetLastError();
}

cudaError_t launch_state_passing(const Shape& s, const FwdArgs& a, const float* cdecay,
                                 float* states, cudaStream_t st)
{
    const int64_t total = (int64_t)s.batch * s.nheads * s.headdim * s.dstate;
    state_passing_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        s, cdecay, states, a.init_ssm, a.final_ssm);
    return cudaGetLastError();
}

cudaError_t launch_chunk_output(const Shape& s, const FwdArgs& a, const float* u,
                                const float* dt, const float* acs, const float* hin,
                                cudaStream_t st)
{
    const dim3 grid(s.nchunks(), s.nheads, s.batch);
    const size_t smem = chunk_output_smem_bytes(s);
    cudaError_t e;
    if (s.act_bf16) {
        e = cudaFuncSetAttribute(chunk_output_kernel<bf16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        chunk_output_kernel<bf16><<<grid, 256, smem, st>>>(s, a, u, dt, acs, hin);
    } else {
        e = cudaFuncSetAttribute(chunk_output_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        chunk_output_kernel<float><<<grid, 256, smem, st>>>(s, a, u, dt, acs, hin);
    }
    return cudaGetLastError();
}

}  // namespace ssd
