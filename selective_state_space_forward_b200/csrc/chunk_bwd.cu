// chunk_bwd.cu -- the backward (vector-Jacobian product) of the chunked scan, fp32.
//
// mojolearn Mamba3Block, method "backward": given the gradient of the loss
// with respect to the output, the gradients with respect to the input and
// every weight of a zero-state prefill (no carried state, no final-state
// cotangent).  The model card ("Checkpoint and training") fixes what the
// gradients must respect: a loss on one packed document gives exactly zero
// gradient on every other document.
//
// The forward is the chunked form of the staged path (chunk_staged.cu): with
// E[t,s] = exp(acs_t - acs_s), M[t,s] = (C^_t . B^_s) E[t,s] dt_s on the
// causal same-segment mask of a chunk, f_t = [seg_t = 0] exp(acs_t),
// w_s = [seg_s = seg_last] exp(acs_last - acs_s) dt_s and k_c the chunk's carry,
//
//   y_t      = sum_s M[t,s] x_s + f_t C^_t . Hin_c + D x_t ,  out_t = y_t SiLU(z_t)
//   Hin_{c+1} = k_c Hin_c + S_c ,  S_c = sum_s w_s x_s (outer) B^_s .
//
// Its reverse, with gy = gout SiLU(z):
//
//   gHout_c  = sum_t f_t gy_t (outer) C^_t                 (bwd_state_out_kernel)
//   gHin_c   = gHout_c + k_c gHin_{c+1},  gS_c = gHin_{c+1}  (bwd_state_scan_kernel)
//   per chunk and head (bwd_chunk_kernel):
//     gz       = gout y SiLU'(z),           gD += gy . x
//     gM[t,s]  = gy_t . x_s                 gx_s += sum_t M[t,s] gy_t + D gy_s + w_s gS_c B^_s
//     gC^_t    = sum_s gM E dt_s B^_s + f_t gy_t Hin_c
//     gB^_s    = sum_t gM E dt_s C^_t + w_s x_s gS_c
//     gacs     from E (row sums minus column sums of gM M), f_t, w_s and k_c,
//     gdt      from M and w_s;  gdA = reverse segmented cumsum of gacs;
//     gdt += gdA a, ga = gdA dt;  gdt_raw = gdt sigmoid(dt_raw + dt_bias)
//   per group and token (bwd_bc_group_kernel): the heads' gB^, gC^ summed and
//     taken back through the B/C RMSNorm (weight and per-head bias gradients);
//   per channel (bwd_conv_kernel): back through SiLU and the 4-tap causal conv,
//     with the same document rule as the forward.
//
// Weight gradients are written as per-block partial sums and added up by
// bwd_reduce_kernel in a fixed order, so results repeat bit for bit.
#include "ssd_device.cuh"
#include "ssd_kernels.h"
#include "staged_rows.cuh"

namespace ssd {

constexpr int kBwdThreads = 256;
constexpr int kConvSeg = 128;          // tokens per thread of the conv backward

__device__ __forceinline__ float sigmoid_f(float v) { return 1.0f / (1.0f + expf(-v)); }
// d SiLU(v) / dv
__device__ __forceinline__ float silu_grad_f(float v)
{
    const float s = sigmoid_f(v);
    return s * (1.0f + v * (1.0f - s));
}

// Sum of v over the block (every thread gets the total); red holds >= 32 floats.
__device__ float block_sum(float v, float* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.0f;
    for (int i = 0; i < nw; i++) t += red[i];
    return t;
}

// ---------------------------------------------------------------------------------
// gHout_c[p,n] = sum_t f_t gy_t[p] C^_t[n]: the gradient of the state entering
// chunk c through the chunk's own outputs.  Written into gs.
template <typename T, int TCN>
__global__ void __launch_bounds__(kBwdThreads)
bwd_state_out_kernel(Shape s, FwdArgs a, BwdBufs w)
{
    extern __shared__ float sm[];
    const int P = s.headdim, N = s.dstate, H = s.nheads, L = s.seqlen, nc = s.nchunks();
    const int HP = H * P, NB = N + kPad, XS = P + kPad;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0);
    float* cs = sm;                    // [64][NB]
    float* gf = cs + kChunk * NB;      // [64][XS]  f_t gy_t
    float* ft = gf + kChunk * XS;      // [64]
    int* seg = (int*)(ft + kChunk);    // [64]
    int* flag = seg + kChunk;          // [64]

    const int Lb = row_length(a.lengths, b, L);
    chunk_segments(a.seq_idx ? a.seq_idx + (int64_t)b * L : nullptr, t0, Lc, Lb, seg, flag);
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        const int64_t o = ((int64_t)b * H + h) * L + t0 + r;
        ft[r] = (r < Lc && t0 + r < Lb && seg[r] == 0) ? expf(w.acs[o]) : 0.0f;
    }
    load_bc_rows<T>(s, a, w.u, b, h, t0, Lc, 1, cs, NB);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * P; e += blockDim.x) {
        const int t = e / P, p = e % P;
        float v = 0.0f;
        if (ft[t] != 0.0f) {
            const int64_t o = ((int64_t)b * L + t0 + t) * HP + h * P + p;
            v = ft[t] * to_f(((const T*)w.gout)[o]) * silu_f(to_f(((const T*)a.z)[o]));
        }
        gf[t * XS + p] = v;
    }
    __syncthreads();
    // [p][n] = sum_t gf[t][p] C^[t][n] (rows past the chunk's end are zero in both)
    const Prod<T, TCN> pr(threadIdx.x);
    float acc[4][TCN];
    tile_zero(acc);
    pr.mm(acc, gf, 1, XS, P, cs, NB, 1, N, kChunk);
    float* dst = w.gs + (((int64_t)b * nc + c) * H + h) * P * N;
#pragma unroll
    for (int rr = 0; rr < 4; rr++)
#pragma unroll
        for (int cc = 0; cc < TCN; cc++) {
            const int pp = pr.row(rr, cc), n = pr.col(rr, cc);
            if (pp < P && n < N) dst[pp * N + n] = acc[rr][cc];
        }
}

// Reverse state scan, one thread per state element: on entry gs holds gHout_c,
// on exit gS_c = gHin_{c+1} (zero for the last chunk: no final-state cotangent).
__global__ void __launch_bounds__(kBwdThreads)
bwd_state_scan_kernel(Shape s, const float* __restrict__ cdecay, float* __restrict__ gs)
{
    const int PN = s.headdim * s.dstate, H = s.nheads, nc = s.nchunks();
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)s.batch * H * PN) return;
    const int e = (int)(gid % PN);
    const int h = (int)((gid / PN) % H);
    const int b = (int)(gid / ((int64_t)PN * H));
    const float* kd = cdecay + ((int64_t)b * H + h) * nc;
    float* sp = gs + ((int64_t)b * nc * H + h) * PN + e;        // chunk c at sp + c * cs
    const int64_t cs = (int64_t)H * PN;
    // the next kAhead chunks (walking backwards) are in flight while the chain advances
    constexpr int kAhead = 8;
    float pre[kAhead], kpre[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; i++) {
        const int c = nc - 1 - i;
        pre[i] = c >= 0 ? sp[c * cs] : 0.0f;
        kpre[i] = c >= 0 ? kd[c] : 0.0f;
    }
    float g = 0.0f;                       // gHin_{c+1}
    for (int j0 = 0; j0 < nc; j0 += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; i++) {
            const int c = nc - 1 - (j0 + i);
            if (c >= 0) {
                const float gout_c = pre[i], k = kpre[i];
                if (c - kAhead >= 0) {
                    pre[i] = sp[(c - kAhead) * cs];
                    kpre[i] = kd[c - kAhead];
                }
                sp[c * cs] = g;
                g = (k == kChunkReset) ? gout_c : gout_c + k * g;
            }
        }
    }
}

// ---------------------------------------------------------------------------------
// The per-(chunk, head) gradients.  256 threads; P <= 64 and N <= 128 (TCN = 4
// column tiles for N <= 64, else 8).  Every contraction is a product of the
// kernel's engine (Prod: tensor-core tf32 tiles for bf16, fp32 SIMT tiles for
// fp32) over the chunk's operands in shared memory.
template <typename T, int TCN>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_chunk_kernel(Shape s, FwdArgs a, BwdBufs w)
{
    extern __shared__ float sm[];
    const int P = s.headdim, N = s.dstate, H = s.nheads, L = s.seqlen, nc = s.nchunks();
    const int HP = H * P, NB = N + kPad, XS = P + kPad, cd = s.conv_dim();
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * kChunk, Lc = min(kChunk, L - t0), last = Lc - 1;
    const int tid = threadIdx.x;
    const Prod<T, 4> p4(tid);                  // 64 x 64 products
    const Prod<T, TCN> pn(tid);                // 64 x N products
    float* cs = sm;                    // [64][NB]  C^
    float* bs = cs + kChunk * NB;      // [64][NB]  B^
    float* xs = bs + kChunk * NB;      // [64][XS]  x (conv output)
    float* gy = xs + kChunk * XS;      // [64][XS]  gradient of y
    float* hb = gy + kChunk * XS;      // [P][NB]   Hin_c, then gS_c
    float* cbe = hb + P * NB;          // [64][kMS] (C^_t . B^_s) E[t,s] on the mask
    float* gm = cbe + kChunk * kMS;    // [64][kMS] scratch; gM; then gM E dt_s
    float* ac = gm + kChunk * kMS;     // [64] acs
    float* dv = ac + kChunk;           // [64] dt
    float* ft = dv + kChunk;           // [64] weight of the carried-state term
    float* ws = ft + kChunk;           // [64] chunk-state weight
    float* gac = ws + kChunk;          // [64] gradient of acs
    float* gdv = gac + kChunk;         // [64] gradient of dt
    float* red = gdv + kChunk;         // [64] per-token scratch
    float* red2 = red + kChunk;        // [32] block reduction scratch
    int* seg = (int*)(red2 + 32);      // [64]
    int* flag = seg + kChunk;          // [64]

    const int Lb = row_length(a.lengths, b, L);
    chunk_segments(a.seq_idx ? a.seq_idx + (int64_t)b * L : nullptr, t0, Lc, Lb, seg, flag);
    const int64_t bh = (int64_t)b * H + h;
    if (tid < kChunk) {
        const int64_t o = bh * L + t0 + tid;
        ac[tid] = tid < Lc ? w.acs[o] : 0.0f;
        dv[tid] = tid < Lc ? w.dt[o] : 0.0f;
        gac[tid] = 0.0f;
        gdv[tid] = 0.0f;
    }
    __syncthreads();
    if (tid < kChunk) {
        ft[tid] = (tid < Lc && seg[tid] == 0) ? expf(ac[tid]) : 0.0f;
        ws[tid] = (tid < Lc && seg[tid] == seg[last]) ? expf(ac[last] - ac[tid]) * dv[tid] : 0.0f;
    }
    load_x_rows<T>(s, a, w.u, b, h, t0, Lc, xs, XS);
    load_bc_rows<T>(s, a, w.u, b, h, t0, Lc, 1, cs, NB);
    load_bc_rows<T>(s, a, w.u, b, h, t0, Lc, 0, bs, NB);
    load_rows8(w.hin + (((int64_t)b * nc + c) * H + h) * P * N, N, N, P, hb, NB, P);
    __syncthreads();

    // (C^_t . B^_s) E[t,s] on the causal same-segment mask
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
    __syncthreads();

    // y recomputed; gy, gz; the carried-state term's share of gacs; gD
    const float Dh = a.D[h];
    float dpart = 0.0f;
    {
        float ys[4][4], off[4][4];
        tile_zero(ys);
        tile_zero(off);
        // z and the output gradient of the thread's elements, requested before the
        // products so their latency overlaps them (and before any store of gz)
        float zr[4][4], gr[4][4];
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int t = p4.row(rr, cc), p = p4.col(rr, cc);
                const bool ok = p < P && t < Lc && t0 + t < Lb;
                const int64_t o = ((int64_t)b * L + t0 + t) * HP + h * P + p;
                zr[rr][cc] = ok ? to_f(((const T*)a.z)[o]) : 0.0f;
                gr[rr][cc] = ok ? to_f(((const T*)w.gout)[o]) : 0.0f;
            }
        p4.mm(ys, cbe, kMS, 1, kChunk, xs, XS, 1, P, kChunk, dv);   // sum_s M[t,s] x_s
        p4.mm(off, cs, NB, 1, kChunk, hb, 1, NB, P, N);           // C^_t . Hin[p]
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int t = p4.row(rr, cc), p = p4.col(rr, cc);
                if (p >= P) continue;
                float gyv = 0.0f, prod = 0.0f;
                if (t < Lc) {
                    const int64_t o = ((int64_t)b * L + t0 + t) * HP + h * P + p;
                    if (t0 + t < Lb) {
                        const float offv = ft[t] != 0.0f ? off[rr][cc] : 0.0f;
                        const float y = ys[rr][cc] + ft[t] * offv + Dh * xs[t * XS + p];
                        const float zv = zr[rr][cc];
                        const float go = gr[rr][cc];
                        gyv = go * silu_f(zv);
                        w.gz[o] = go * y * silu_grad_f(zv);
                        prod = ft[t] * gyv * offv;
                        dpart += gyv * xs[t * XS + p];
                    } else {
                        w.gz[o] = 0.0f;
                    }
                }
                gy[t * XS + p] = gyv;
                gm[t * kMS + p] = prod;
            }
    }
    __syncthreads();
    if (tid < kChunk) {
        float acc = 0.0f;
        for (int p = 0; p < P; p++) acc += gm[tid * kMS + p];
        gac[tid] += acc;
    }
    dpart = block_sum(dpart, red2);
    __syncthreads();

    // gM[t,s] = gy_t . x_s on the mask
    {
        float acc[4][4];
        tile_zero(acc);
        p4.mm(acc, gy, XS, 1, kChunk, xs, 1, XS, kChunk, P);
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int t = p4.row(rr, cc), r = p4.col(rr, cc);
                gm[t * kMS + r] = (r <= t && t < Lc && seg[r] == seg[t]) ? acc[rr][cc] : 0.0f;
            }
    }
    __syncthreads();
    // acs through E: + row sums, - column sums of gM M; dt through M
    if (tid < kChunk) {
        const int t = tid;
        float acc = 0.0f;
        for (int r = 0; r <= t; r++) acc += gm[t * kMS + r] * cbe[t * kMS + r] * dv[r];
        gac[t] += acc;
    } else if (tid < 2 * kChunk) {
        const int r = tid - kChunk;
        float acc = 0.0f, gd = 0.0f;
        for (int t = r; t < kChunk; t++) {
            const float g = gm[t * kMS + r] * cbe[t * kMS + r];
            acc += g * dv[r];
            gd += g;
        }
        red[r] = acc;
        gdv[r] += gd;
    }
    __syncthreads();
    if (tid < kChunk) gac[tid] -= red[tid];
    // gM -> gradient of (C^_t . B^_s): gM E dt_s
    for (int e = tid; e < kChunk * kChunk; e += blockDim.x) {
        const int t = e / kChunk, r = e % kChunk;
        const float g = gm[t * kMS + r];
        gm[t * kMS + r] = g != 0.0f ? g * expf(ac[t] - ac[r]) * dv[r] : 0.0f;
    }
    __syncthreads();

    // gx (intra-chunk and D), kept in registers until the chunk-state part is added
    float gx[4][4];
    tile_zero(gx);
    p4.mm(gx, cbe, 1, kMS, kChunk, gy, XS, 1, P, kChunk);        // sum_t M[t,s] gy_t
#pragma unroll
    for (int rr = 0; rr < 4; rr++)
#pragma unroll
        for (int cc = 0; cc < 4; cc++) {
            const int r = p4.row(rr, cc), p = min(p4.col(rr, cc), P - 1);
            gx[rr][cc] = r < Lc ? gx[rr][cc] * dv[r] + Dh * gy[r * XS + p] : 0.0f;
        }
    // gC^ (complete), written per head
    {
        float acc[4][TCN], acc2[4][TCN];
        tile_zero(acc);
        tile_zero(acc2);
        pn.mm(acc, gm, kMS, 1, kChunk, bs, NB, 1, N, kChunk);   // sum_s gM E dt_s B^_s
        pn.mm(acc2, gy, XS, 1, kChunk, hb, NB, 1, N, P);      // gy_t . Hin[:, n]
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < TCN; cc++) {
                const int t = pn.row(rr, cc), n = pn.col(rr, cc);
                if (t < Lc && n < N)
                    w.gch[(((int64_t)b * L + t0 + t) * H + h) * N + n] =
                        acc[rr][cc] + (ft[t] != 0.0f ? ft[t] * acc2[rr][cc] : 0.0f);
            }
    }
    // gB^ (intra-chunk part)
    float gb[4][TCN];
    tile_zero(gb);
    pn.mm(gb, gm, 1, kMS, kChunk, cs, NB, 1, N, kChunk);       // sum_t gM E dt_s C^_t
    __syncthreads();

    // gS_c replaces Hin_c; gk = <gS_c, Hin_c> is the carry's gradient
    const float* gsp = w.gs + (((int64_t)b * nc + c) * H + h) * P * N;
    float gk = 0.0f;
    {
        // four consecutive elements per task (N is a multiple of 8), two tasks' loads in flight
        const int ntask = P * N / 4;
        for (int i0 = tid; i0 < ntask; i0 += 2 * blockDim.x) {
            float4 g[2];
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const int i = i0 + k * blockDim.x;
                g[k] = i < ntask ? *reinterpret_cast<const float4*>(gsp + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const int i = i0 + k * blockDim.x;
                if (i < ntask) {
                    float* hr = hb + ((4 * i) / N) * NB + (4 * i) % N;
                    gk += g[k].x * hr[0] + g[k].y * hr[1] + g[k].z * hr[2] + g[k].w * hr[3];
                    *reinterpret_cast<float4*>(hr) = g[k];
                }
            }
        }
    }
    gk = block_sum(gk, red2);
    __syncthreads();

    // chunk state: gXs = gS B^_s -> gx += w_s gXs; gw_s = gXs . x_s; gB^_s += w_s x_s gS
    {
        float g7[4][4];
        tile_zero(g7);
        p4.mm(g7, bs, NB, 1, kChunk, hb, 1, NB, P, N);
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
                const int r = p4.row(rr, cc), p = p4.col(rr, cc);
                if (p >= P) continue;
                gx[rr][cc] += ws[r] * g7[rr][cc];
                gm[r * kMS + p] = g7[rr][cc] * xs[r * XS + p];
            }
    }
    {
        float g8[4][TCN];
        tile_zero(g8);
        pn.mm(g8, xs, XS, 1, kChunk, hb, NB, 1, N, P);
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < TCN; cc++) {
                const int r = pn.row(rr, cc), n = pn.col(rr, cc);
                if (r < Lc && n < N)
                    w.gbh[(((int64_t)b * L + t0 + r) * H + h) * N + n] = gb[rr][cc] + ws[r] * g8[rr][cc];
            }
    }
#pragma unroll
    for (int rr = 0; rr < 4; rr++)
#pragma unroll
        for (int cc = 0; cc < 4; cc++) {
            const int r = p4.row(rr, cc), p = p4.col(rr, cc);
            if (r < Lc && p < P) w.gu[((int64_t)b * L + t0 + r) * cd + h * P + p] = gx[rr][cc];
        }
    __syncthreads();
    if (tid < kChunk) {
        float acc = 0.0f;
        for (int p = 0; p < P; p++) acc += gm[tid * kMS + p];
        red[tid] = acc;                               // gradient of w_s
    }
    __syncthreads();
    if (tid < Lc && seg[tid] == seg[last]) {
        gac[tid] -= red[tid] * ws[tid];
        gdv[tid] += red[tid] * expf(ac[last] - ac[tid]);
    }
    __syncthreads();
    if (tid < kChunk) {
        // gl = sum_r red[r] ws[r] (ws is zero past the chunk's end): per warp, then in order
        float gl = red[tid] * ws[tid];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gl += __shfl_xor_sync(0xffffffffu, gl, o);
        if ((tid & 31) == 0) red2[1 + (tid >> 5)] = gl;
    }
    __syncthreads();
    if (tid == 0) {
        float gl = red2[1] + red2[2];
        const float kc = w.cdecay[bh * nc + c];
        if (kc != kChunkReset) gl += gk * kc;         // k_c = exp(acs_last)
        gac[last] += gl;
    }
    __syncthreads();

    // dA = dt a feeds acs through the segmented in-chunk cumsum: gdA is its reverse,
    // a suffix sum within each segment (warps 0 and 1, 32 tokens each, by shuffles;
    // segment ids never decrease along the chunk, so equal ids mean one run)
    if (tid < kChunk) {
        const int j = tid, lane = tid & 31;
        float v = j < Lc ? gac[j] : 0.0f;
        const int sj = seg[j];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float vo = __shfl_down_sync(0xffffffffu, v, o);
            const int so = __shfl_down_sync(0xffffffffu, sj, o);
            if (lane + o < 32 && so == sj) v += vo;
        }
        if (j == 32) red2[0] = v;                     // suffix of the second half
        red[j] = v;
    }
    __syncthreads();
    if (tid < kChunk) {
        float gv = 0.0f, ga = 0.0f;
        if (tid < Lc) {
            const int j = tid;
            const float gda = red[j] + ((j < 32 && Lc > 32 && seg[32] == seg[j]) ? red2[0] : 0.0f);
            const int64_t tok = (int64_t)b * L + t0 + j;
            const bool real = t0 + j < Lb;
            float av;
            bool floored = false;
            if (s.a_per_token) {
                const float Av = a.A[tok * H + h];
                av = fminf(Av, -kAFloor);
                floored = Av > -kAFloor;
            } else {
                av = a.A[h];
            }
            if (real) {
                gv = (gdv[j] + gda * av) * sigmoid_f(a.dt_raw[tok * H + h] + a.dt_bias[h]);
                ga = floored ? 0.0f : gda * dv[j];
            }
            w.gdt_raw[tok * H + h] = gv;
            if (s.a_per_token && w.gA) w.gA[tok * H + h] = ga;
        }
        // per-chunk sums of the dt_bias and A gradients: each warp in a fixed order,
        // then warp 0's before warp 1's
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gv += __shfl_xor_sync(0xffffffffu, gv, o);
            ga += __shfl_xor_sync(0xffffffffu, ga, o);
        }
        if ((tid & 31) == 0) {
            red2[3 + (tid >> 5)] = gv;
            red2[5 + (tid >> 5)] = ga;
        }
    }
    __syncthreads();
    if (tid == 0) {
        const int64_t pi = ((int64_t)b * nc + c) * H + h;
        w.p_dtb[pi] = red2[3] + red2[4];
        w.p_A[pi] = red2[5] + red2[6];
        w.p_D[pi] = dpart;
    }
}

// ---------------------------------------------------------------------------------
// Per (row, 64-token block, group): sum the group's heads' gB^ and gC^, then (with
// the B/C norm) go back through B^ = B r w + bias_h.  128 threads, n = tid (+128).
template <typename T>
__global__ void __launch_bounds__(128)
bwd_bc_group_kernel(Shape s, FwdArgs a, BwdBufs w)
{
    extern __shared__ float sm[];
    const int N = s.dstate, H = s.nheads, G = s.ngroups, L = s.seqlen, hg = H / G;
    const int HP = H * s.headdim, GN = G * N, cd = s.conv_dim();
    const int tb = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int ntb = gridDim.x;
    const int tid = threadIdx.x;
    float* acc = sm;                   // [2][hg][N] per-head bias gradient of this block
    float* red = acc + 2 * hg * N;     // [32]
    const bool norm = s.bc_norm != 0;
    if (norm)
        for (int i = tid; i < 2 * hg * N; i += blockDim.x) acc[i] = 0.0f;
    float wacc[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};   // [which][n slot] norm-weight gradient
    __syncthreads();
    for (int t = tb * kChunk; t < min(L, (tb + 1) * kChunk); t++) {
        const int64_t tok = (int64_t)b * L + t;
        for (int which = 0; which < 2; which++) {
            const float* gh = which ? w.gch : w.gbh;
            const float* wn = which ? a.cn_w : a.bn_w;
            float gsum[2] = {0.0f, 0.0f}, uv[2] = {0.0f, 0.0f};
            float ss = 0.0f, dot = 0.0f;
            for (int k = 0; k < 2; k++) {
                const int n = tid + 128 * k;
                if (n >= N) continue;
                for (int j = 0; j < hg; j++) {
                    const float v = gh[(tok * H + g * hg + j) * N + n];
                    gsum[k] += v;
                    if (norm) acc[(which * hg + j) * N + n] += v;
                }
                if (norm) {
                    const int64_t ch = HP + which * GN + g * N + n;
                    uv[k] = w.u ? w.u[tok * cd + ch]
                                : to_f(((const T*)(which ? a.C : a.B))[tok * GN + g * N + n]);
                    ss += uv[k] * uv[k];
                    dot += gsum[k] * (wn ? wn[n] : 1.0f) * uv[k];
                }
            }
            float r = 1.0f, r3n = 0.0f;
            if (norm) {
                ss = block_sum(ss, red);
                dot = block_sum(dot, red);
                r = rsqrtf(ss / N + kNormEps);
                r3n = r * r * r / N;
            }
            for (int k = 0; k < 2; k++) {
                const int n = tid + 128 * k;
                if (n >= N) continue;
                float gval = gsum[k];
                if (norm) {
                    const float wv = wn ? wn[n] : 1.0f;
                    gval = r * wv * gsum[k] - r3n * uv[k] * dot;
                    wacc[which][k] += gsum[k] * uv[k] * r;
                }
                w.gu[tok * cd + HP + which * GN + g * N + n] = gval;
            }
        }
    }
    if (!norm) return;
    __syncthreads();
    // partials: p_nw (B, ntb, G, 2, N), p_nb (B, ntb, 2, H, N)
    for (int which = 0; which < 2; which++)
        for (int k = 0; k < 2; k++) {
            const int n = tid + 128 * k;
            if (n < N) w.p_nw[((((int64_t)b * ntb + tb) * G + g) * 2 + which) * N + n] = wacc[which][k];
        }
    for (int i = tid; i < 2 * hg * N; i += blockDim.x) {
        const int which = i / (hg * N), j = (i / N) % hg, n = i % N;
        w.p_nb[((((int64_t)b * ntb + tb) * 2 + which) * H + g * hg + j) * N + n] = acc[i];
    }
}

// ---------------------------------------------------------------------------------
// Back through SiLU and the causal conv: one thread per (row, channel, segment of
// kConvSeg tokens); channels fastest, so a warp reads consecutive channels of a
// token row.  gconv partials (B, nseg, cd, 5): four taps, then the bias.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_conv_kernel(Shape s, FwdArgs a, BwdBufs w)
{
    const int cd = s.conv_dim(), L = s.seqlen;
    const int nseg = (L + kConvSeg - 1) / kConvSeg;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)s.batch * nseg * cd) return;
    const int ch = (int)(gid % cd);
    const int sg = (int)((gid / cd) % nseg);
    const int b = (int)(gid / ((int64_t)cd * nseg));
    const int HP = s.nheads * s.headdim, GN = s.ngroups * s.dstate;
    const T* src;
    float* dst;
    int64_t stride;
    int col;
    if (ch < HP) { src = (const T*)a.x; dst = w.gx; stride = HP; col = ch; }
    else if (ch < HP + GN) { src = (const T*)a.B; dst = w.gB; stride = GN; col = ch - HP; }
    else { src = (const T*)a.C; dst = w.gC; stride = GN; col = ch - HP - GN; }
    src += (int64_t)b * L * stride + col;
    dst += (int64_t)b * L * stride + col;
    const float* gu = w.gu + (int64_t)b * L * cd + ch;
    const int Lb = row_length(a.lengths, b, L);
    const int ts = sg * kConvSeg, te = min(L, ts + kConvSeg);

    if (s.dconv == 1) {       // no conv: the gradient of the raw input is gu itself
        for (int t = ts; t < te; t++) dst[(int64_t)t * stride] = t < Lb ? gu[(int64_t)t * cd] : 0.0f;
        return;
    }
    const int32_t* seq_row = a.seq_idx ? a.seq_idx + (int64_t)b * L : nullptr;
    float wk[4];
#pragma unroll
    for (int k = 0; k < 4; k++) wk[k] = to_f(((const T*)a.conv_w)[(int64_t)ch * 4 + k]);
    const float cb = to_f(((const T*)a.conv_b)[ch]);
    float gw[4] = {0.0f, 0.0f, 0.0f, 0.0f}, gbias = 0.0f;
    // window of raw inputs x[t-3 .. t] and boundary flags at t-2 .. t
    float xw[4];
#pragma unroll
    for (int k = 0; k < 3; k++) {
        const int tau = ts - 3 + k;
        xw[k] = (tau >= 0 && tau < Lb) ? to_f(src[(int64_t)tau * stride]) : 0.0f;
    }
    int bd1 = (ts - 2 >= 1 && ts - 2 < Lb) ? is_boundary(seq_row, ts - 2) : 0;   // at t-2
    int bd2 = (ts - 1 >= 1 && ts - 1 < Lb) ? is_boundary(seq_row, ts - 1) : 0;   // at t-1
    float gxw[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // pending gx at t-3 .. t
    const int tend = min(te + 3, Lb);
    for (int t = ts; t < tend; t++) {
        xw[3] = to_f(src[(int64_t)t * stride]);
        const int bd3 = is_boundary(seq_row, t);
        // tap k reads x[t-3+k]; valid while no boundary lies in (t-3+k, t]
        const bool ok3 = true;
        const bool ok2 = !bd3;
        const bool ok1 = ok2 && !bd2;
        const bool ok0 = ok1 && !bd1 && t - 3 >= 0;
        const bool okk[4] = {ok0, ok1 && t - 2 >= 0, ok2 && t - 1 >= 0, ok3};
        float pre = cb;
#pragma unroll
        for (int k = 0; k < 4; k++) pre += okk[k] ? wk[k] * xw[k] : 0.0f;
        const float gpre = gu[(int64_t)t * cd] * silu_grad_f(pre);
        if (t < te) {
            gbias += gpre;
#pragma unroll
            for (int k = 0; k < 4; k++) gw[k] += okk[k] ? gpre * xw[k] : 0.0f;
        }
#pragma unroll
        for (int k = 0; k < 4; k++) gxw[k] += okk[k] ? gpre * wk[k] : 0.0f;
        // x[t-3] has all its contributions (tokens t-3 .. t): emit it
        if (t - 3 >= ts && t - 3 < te) dst[(int64_t)(t - 3) * stride] = gxw[0];
        gxw[0] = gxw[1]; gxw[1] = gxw[2]; gxw[2] = gxw[3]; gxw[3] = 0.0f;
        xw[0] = xw[1]; xw[1] = xw[2]; xw[2] = xw[3];
        bd1 = bd2; bd2 = bd3;
    }
    // tokens whose later taps lie past the row's real end, and padding
    for (int tau = max(ts, tend - 3); tau < te; tau++) {
        const int k = tau - (tend - 3);      // gxw[k] holds x[tend-3+k]
        dst[(int64_t)tau * stride] = (tau < Lb && k >= 0 && k < 3) ? gxw[k] : 0.0f;
    }
    float* pc = w.p_conv + (((int64_t)b * nseg + sg) * cd + ch) * 5;
#pragma unroll
    for (int k = 0; k < 4; k++) pc[k] = gw[k];
    pc[4] = gbias;
}

// out[m] = sum over r of in[r * ld + m], r in order (weight-gradient partials).
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(const float* __restrict__ in, int64_t R, int64_t M, int64_t ld,
                  float* __restrict__ out)
{
    const int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    float acc = 0.0f;
    for (int64_t r = 0; r < R; r++) acc += in[r * ld + m];
    out[m] = acc;
}

// The conv partials (R, cd, 5) summed over r in order: taps to gconv_w (cd, 4),
// the fifth column to gconv_b (cd).
__global__ void __launch_bounds__(256)
bwd_conv_reduce_kernel(const float* __restrict__ in, int64_t R, int cd, float* __restrict__ gw,
                       float* __restrict__ gb)
{
    const int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= (int64_t)cd * 5) return;
    float acc = 0.0f;
    for (int64_t r = 0; r < R; r++) acc += in[r * cd * 5 + m];
    const int ch = (int)(m / 5), k = (int)(m % 5);
    if (k < 4) gw[(int64_t)ch * 4 + k] = acc;
    else gb[ch] = acc;
}

// ---------------------------------------------------------------------------------
// host side

size_t bwd_chunk_smem_bytes(const Shape& s)
{
    const size_t P = s.headdim, N = s.dstate, NB = N + kPad, XS = P + kPad;
    return sizeof(float) * (2 * kChunk * NB + 2 * kChunk * XS + P * NB + 2 * kChunk * kMS +
                            8 * kChunk + 32) + sizeof(int) * 2 * kChunk;
}

static size_t state_out_smem_bytes(const Shape& s)
{
    return sizeof(float) * (kChunk * ((size_t)s.dstate + kPad) + kChunk * ((size_t)s.headdim + kPad) + kChunk) +
           sizeof(int) * 2 * kChunk;
}

bool bwd_supported(const Shape& s)
{
    return s.headdim <= 64 && s.dstate <= 128 && bwd_chunk_smem_bytes(s) <= 227 * 1024;
}

template <typename K>
static cudaError_t set_smem(K kern, size_t bytes)
{
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T>
static cudaError_t launch_bwd_t(const Shape& s, const FwdArgs& a, const BwdBufs& w, int* launches,
                                cudaStream_t st)
{
    cudaError_t e;
    const dim3 cgrid(s.nchunks(), s.nheads, s.batch);
    const size_t so = state_out_smem_bytes(s);
    auto k_out = s.dstate > 64 ? bwd_state_out_kernel<T, 8> : bwd_state_out_kernel<T, 4>;
    if ((e = set_smem(k_out, so)) != cudaSuccess) return e;
    k_out<<<cgrid, kBwdThreads, so, st>>>(s, a, w);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const int64_t nel = (int64_t)s.batch * s.nheads * s.headdim * s.dstate;
    bwd_state_scan_kernel<<<(unsigned)((nel + 255) / 256), 256, 0, st>>>(s, w.cdecay, w.gs);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const size_t sc = bwd_chunk_smem_bytes(s);
    auto k_chunk = s.dstate > 64 ? bwd_chunk_kernel<T, 8> : bwd_chunk_kernel<T, 4>;
    if ((e = set_smem(k_chunk, sc)) != cudaSuccess) return e;
    k_chunk<<<cgrid, kBwdThreads, sc, st>>>(s, a, w);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const int ntb = s.nchunks();
    const int hg = s.nheads / s.ngroups;
    const size_t sg = sizeof(float) * (2 * (size_t)hg * s.dstate + 32);
    if ((e = set_smem(bwd_bc_group_kernel<T>, sg)) != cudaSuccess) return e;
    bwd_bc_group_kernel<T><<<dim3(ntb, s.ngroups, s.batch), 128, sg, st>>>(s, a, w);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const int nseg = (s.seqlen + kConvSeg - 1) / kConvSeg;
    const int64_t nth = (int64_t)s.batch * nseg * s.conv_dim();
    bwd_conv_kernel<T><<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(s, a, w);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // weight gradients: fixed-order sums of the partials
    auto reduce = [&](const float* in, int64_t R, int64_t M, int64_t ld, float* out) -> cudaError_t {
        if (!out || M == 0) return cudaSuccess;
        bwd_reduce_kernel<<<(unsigned)((M + 255) / 256), 256, 0, st>>>(in, R, M, ld, out);
        ++*launches;
        return cudaGetLastError();
    };
    const int64_t rc = (int64_t)s.batch * s.nchunks(), Hh = s.nheads;
    if ((e = reduce(w.p_dtb, rc, Hh, Hh, w.g_dt_bias)) != cudaSuccess) return e;
    if ((e = reduce(w.p_D, rc, Hh, Hh, w.g_D)) != cudaSuccess) return e;
    if (!s.a_per_token && (e = reduce(w.p_A, rc, Hh, Hh, w.gA)) != cudaSuccess) return e;
    if (s.dconv == 4) {
        const int cd = s.conv_dim();
        bwd_conv_reduce_kernel<<<(unsigned)(((int64_t)cd * 5 + 255) / 256), 256, 0, st>>>(
            w.p_conv, (int64_t)s.batch * nseg, cd, w.gconv_w, w.gconv_b);
        ++*launches;
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (s.bc_norm) {
        const int64_t N = s.dstate, HN = Hh * N;
        const int64_t rn = (int64_t)s.batch * ntb * s.ngroups, rb = (int64_t)s.batch * ntb;
        if ((e = reduce(w.p_nw, rn, N, 2 * N, w.g_bnw)) != cudaSuccess) return e;
        if ((e = reduce(w.p_nw + N, rn, N, 2 * N, w.g_cnw)) != cudaSuccess) return e;
        if ((e = reduce(w.p_nb, rb, HN, 2 * HN, w.g_bnb)) != cudaSuccess) return e;
        if ((e = reduce(w.p_nb + HN, rb, HN, 2 * HN, w.g_cnb)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_backward(const Shape& s, const FwdArgs& a, const BwdBufs& w, int* launches,
                            cudaStream_t st)
{
    return s.act_bf16 ? launch_bwd_t<bf16>(s, a, w, launches, st)
                      : launch_bwd_t<float>(s, a, w, launches, st);
}

}  // namespace ssd
