// conv.cu -- K1: causal depthwise conv (kernel 4) + SiLU over the x|B|C channels.
//
// u[b,t,c] = SiLU(conv_b[c] + sum_{k=0..3} conv_w[c,k] * xin[b, t-3+k, c])
//
// "Mini-K3-1H-mamba2-n64-g8" model card, Architecture (causal depthwise conv,
// kernel 4) and "Checkpoint and training" (the document ids reset the conv
// history at every boundary); x|B|C channel order and conv_dim from the
// codestral_mamba.ts weight-port header.  A tap at t-3+k is used only when no
// document boundary lies in (t-3+k, t]; taps before token 0 come from the
// caller's conv history (oldest first), which belongs to the row's first
// document.
//
// Layout: one thread owns 8 consecutive channels (one 16-byte bf16 vector, or
// two fp32 vectors) of 4 consecutive tokens, so its 7 input rows are loaded
// once and every load and store is a full 16-byte access; consecutive
// threads walk the channel axis, so a warp touches contiguous 512-byte
// (bf16) spans of a token row.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kTokPerThread = 4;

template <typename T>
__device__ __forceinline__ const T* channel_src(const Shape& s, const T* x, const T* B, const T* C,
                                               int c, int64_t& stride, int& col)
{
    const int HP = s.nheads * s.headdim, GN = s.ngroups * s.dstate;
    if (c < HP) { stride = HP; col = c; return x; }
    if (c < HP + GN) { stride = GN; col = c - HP; return B; }
    stride = GN; col = c - HP - GN; return C;
}

// One thread: channels [c, c+8) of tokens [t0, t0+4) of row b.
// OutT is float (staged path) or bf16 (fused path's shared B|C operand).
template <typename T, typename OutT>
__global__ void __launch_bounds__(256)
conv_silu_kernel(Shape s, const T* __restrict__ x, const T* __restrict__ Bm,
                 const T* __restrict__ Cm, const T* __restrict__ w, const T* __restrict__ bias,
                 const int32_t* __restrict__ seq, const T* __restrict__ hist0,
                 OutT* __restrict__ u, int cbase)
{
    const int cd = s.conv_dim();
    const int nvec = (cd - cbase) / 8;
    const int ntg = (s.seqlen + kTokPerThread - 1) / kTokPerThread;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)s.batch * ntg * nvec) return;
    const int v = (int)(gid % nvec);
    const int64_t r = gid / nvec;
    const int tg = (int)(r % ntg);
    const int b = (int)(r / ntg);
    const int c = cbase + v * 8;
    const int L = s.seqlen;

    int64_t stride;
    int col;
    const T* src = channel_src(s, x, Bm, Cm, c, stride, col);
    src += (int64_t)b * L * stride + col;

    float wk[8][4], bs[8];
    {
        float t8[8];
#pragma unroll
        for (int q = 0; q < 4; q++) {   // 32 weights: channels c..c+7, taps 0..3
            load8(w + (int64_t)c * 4 + q * 8, t8);
#pragma unroll
            for (int i = 0; i < 8; i++) wk[q * 2 + i / 4][i % 4] = t8[i];
        }
        load8(bias + c, bs);
    }

    const int t0 = tg * kTokPerThread;
    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    // bd[j] = boundary at position t0 - 2 + j  (j = 0 .. 5)
    int bd[kTokPerThread + 2];
#pragma unroll
    for (int j = 0; j < kTokPerThread + 2; j++) {
        const int64_t pos = (int64_t)t0 - 2 + j;
        bd[j] = (pos >= 1 && pos < L) ? is_boundary(seq_row, pos) : 0;
    }
    // rows t0-3 .. t0+3
    float win[kTokPerThread + 3][8];
#pragma unroll
    for (int j = 0; j < kTokPerThread + 3; j++) {
        const int64_t tau = (int64_t)t0 - 3 + j;
        if (tau >= 0 && tau < L) {
            load8(src + tau * stride, win[j]);
        } else if (tau < 0 && hist0 != nullptr) {
            load8(hist0 + ((int64_t)b * 3 + (tau + 3)) * cd + c, win[j]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) win[j][i] = 0.0f;
        }
    }

    OutT* dst = u + (int64_t)b * L * (cd - cbase) + (c - cbase);
#pragma unroll
    for (int q = 0; q < kTokPerThread; q++) {
        const int64_t t = t0 + q;
        if (t >= L) break;
        // tap k uses row t-3+k, i.e. win[q+k]; valid when no boundary at t-2+k .. t
        const int okk2 = !bd[q + 2];
        const int okk1 = okk2 && !bd[q + 1];
        const int okk0 = okk1 && !bd[q];
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            float acc = bs[i] + wk[i][3] * win[q + 3][i];
            acc += okk2 ? wk[i][2] * win[q + 2][i] : 0.0f;
            acc += okk1 ? wk[i][1] * win[q + 1][i] : 0.0f;
            acc += okk0 ? wk[i][0] * win[q][i] : 0.0f;
            o[i] = silu_f(acc);
        }
        store8(dst + t * (cd - cbase), o);
    }
}

// Final conv history: slot i holds the raw input at L-3+i when it lies in the
// last token's document, else 0.  Each thread reads its 3 slots before writing
// them, so the initial and final history may be the same buffer.
template <typename T>
__global__ void __launch_bounds__(256)
conv_state_kernel(Shape s, const T* __restrict__ x, const T* __restrict__ Bm,
                  const T* __restrict__ Cm, const int32_t* __restrict__ seq, const T* hist0,
                  T* hist1)
{
    const int cd = s.conv_dim();
    const int nvec = cd / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)s.batch * nvec) return;
    const int b = (int)(gid / nvec);
    const int c = (int)(gid % nvec) * 8;
    const int L = s.seqlen;
    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    int64_t stride;
    int col;
    const T* src = channel_src(s, x, Bm, Cm, c, stride, col);
    src += (int64_t)b * L * stride + col;

    float vals[3][8];
#pragma unroll
    for (int i = 0; i < 3; i++) {
        const int64_t tau = (int64_t)L - 3 + i;
        int ok = 1;
        for (int64_t pos = (tau + 1 > 1 ? tau + 1 : 1); pos <= L - 1; pos++)
            ok &= !is_boundary(seq_row, pos);
        if (ok && tau >= 0) {
            load8(src + tau * stride, vals[i]);
        } else if (ok && tau < 0 && hist0 != nullptr) {
            load8(hist0 + ((int64_t)b * 3 + (tau + 3)) * cd + c, vals[i]);
        } else {
#pragma unroll
            for (int k = 0; k < 8; k++) vals[i][k] = 0.0f;
        }
    }
#pragma unroll
    for (int i = 0; i < 3; i++) store8(hist1 + ((int64_t)b * 3 + i) * cd + c, vals[i]);
}

template <typename T, typename OutT>
static cudaError_t launch_conv(const Shape& s, const FwdArgs& a, OutT* u, int cbase, cudaStream_t st)
{
    const int nvec = (s.conv_dim() - cbase) / 8;
    const int ntg = (s.seqlen + kTokPerThread - 1) / kTokPerThread;
    const int64_t total = (int64_t)s.batch * ntg * nvec;
    const int64_t blocks = (total + 255) / 256;
    conv_silu_kernel<T, OutT><<<(unsigned)blocks, 256, 0, st>>>(
        s, (const T*)a.x, (const T*)a.B, (const T*)a.C, (const T*)a.conv_w, (const T*)a.conv_b,
        a.seq_idx, (const T*)a.init_conv, u, cbase);
    return cudaGetLastError();
}

cudaError_t launch_conv_silu_all(const Shape& s, const FwdArgs& a, float* u, cudaStream_t st)
{
    return s.act_bf16 ? launch_conv<bf16, float>(s, a, u, 0, st)
                      : launch_conv<float, float>(s, a, u, 0, st);
}

cudaError_t launch_conv_silu_bc(const Shape& s, const FwdArgs& a, void* ubc, cudaStream_t st)
{
    if (!s.act_bf16) return cudaErrorInvalidValue;
    return launch_conv<bf16, bf16>(s, a, (bf16*)ubc, s.nheads * s.headdim, st);
}

cudaError_t launch_conv_state(const Shape& s, const FwdArgs& a, cudaStream_t st)
{
    const int64_t total = (int64_t)s.batch * (s.conv_dim() / 8);
    const int64_t blocks = (total + 255) / 256;
    if (s.act_bf16)
        conv_state_kernel<bf16><<<(unsigned)blocks, 256, 0, st>>>(
            s, (const bf16*)a.x, (const bf16*)a.B, (const bf16*)a.C, a.seq_idx,
            (const bf16*)a.init_conv, (bf16*)a.final_conv);
    else
        conv_state_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            s, (const float*)a.x, (const float*)a.B, (const float*)a.C, a.seq_idx,
            (const float*)a.init_conv, (float*)a.final_conv);
    return cudaGetLastError();
}

}  // namespace ssd
