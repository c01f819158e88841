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
// two fp32 vectors) of 8 consecutive tokens and slides a 3-row window, so each
// input row is loaded once per thread and every load and store is a full
// 16-byte access; consecutive threads walk the channel axis, so a warp touches
// contiguous 512-byte (bf16) spans of a token row.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kTokPerThread = 8;

// Row strides (elements) of the raw x and B|C inputs.
struct RawStrides {
    int64_t x, bc;
};

template <typename T>
__device__ __forceinline__ const T* channel_src(const Shape& s, RawStrides ld, const T* x, const T* B,
                                               const T* C, int c, int64_t& stride, int& col)
{
    const int HP = s.nheads * s.headdim, GN = s.ngroups * s.dstate;
    if (c < HP) { stride = ld.x; col = c; return x; }
    if (c < HP + GN) { stride = ld.bc; col = c - HP; return B; }
    stride = ld.bc; col = c - HP - GN; return C;
}

// Eight consecutive elements kept in their storage form (fewer registers than
// eight floats for bf16) and widened on use.
template <typename T> struct Vec8;
template <> struct Vec8<bf16> {
    uint4 r;
    __device__ __forceinline__ void load(const bf16* p) { r = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void zero() { r = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ float operator[](int i) const
    {
        const uint32_t w = i < 2 ? r.x : i < 4 ? r.y : i < 6 ? r.z : r.w;
        return (i & 1) ? __uint_as_float(w & 0xFFFF0000u) : __uint_as_float(w << 16);
    }
};
template <> struct Vec8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p)
    {
        a = reinterpret_cast<const float4*>(p)[0];
        b = reinterpret_cast<const float4*>(p)[1];
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float operator[](int i) const
    {
        const float4& v = i < 4 ? a : b;
        const int j = i & 3;
        return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
    }
};

// One thread: channels [c, c+8) of tokens [t0, t0+8) of row b, with a rolling
// window of the three previous raw rows.  OutT is float (staged path, exact
// SiLU) or bf16 (fused path's shared B|C operand, hardware-tanh SiLU: the
// result is rounded to bf16 anyway).
template <typename T, typename OutT>
__global__ void __launch_bounds__(256, 3)
conv_silu_kernel(Shape s, const T* __restrict__ x, const T* __restrict__ Bm,
                 const T* __restrict__ Cm, const T* __restrict__ w, const T* __restrict__ bias,
                 const int32_t* __restrict__ seq, const T* __restrict__ hist0,
                 OutT* __restrict__ u, int cbase, RawStrides ld)
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
    const T* src = channel_src(s, ld, x, Bm, Cm, c, stride, col);
    src += (int64_t)b * L * stride + col;

    Vec8<T> wv[4], bv;          // weight (channel i, tap k) = element 4*i + k
#pragma unroll
    for (int q = 0; q < 4; q++) wv[q].load(w + (int64_t)c * 4 + q * 8);
    bv.load(bias + c);

    const int t0 = tg * kTokPerThread;
    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    uint32_t bdm = 0;           // bit j: boundary at position t0 - 2 + j
#pragma unroll
    for (int j = 0; j < kTokPerThread + 2; j++) {
        const int64_t pos = (int64_t)t0 - 2 + j;
        if (pos >= 1 && pos < L && is_boundary(seq_row, pos)) bdm |= 1u << j;
    }
    Vec8<T> win[3];             // rows t-3, t-2, t-1
#pragma unroll
    for (int j = 0; j < 3; j++) {
        const int64_t tau = (int64_t)t0 - 3 + j;
        if (tau >= 0 && tau < L) win[j].load(src + tau * stride);
        else if (tau < 0 && hist0 != nullptr) win[j].load(hist0 + ((int64_t)b * 3 + (tau + 3)) * cd + c);
        else win[j].zero();
    }

    OutT* dst = u + (int64_t)b * L * (cd - cbase) + (c - cbase);
#pragma unroll 1
    for (int q = 0; q < kTokPerThread; q++) {
        const int64_t t = t0 + q;
        if (t >= L) break;
        Vec8<T> cur;
        cur.load(src + t * stride);
        // tap k reads row t-3+k; valid when no boundary at positions t-2+k .. t
        const bool ok2 = !((bdm >> (q + 2)) & 1u);
        const bool ok1 = ok2 && !((bdm >> (q + 1)) & 1u);
        const bool ok0 = ok1 && !((bdm >> q) & 1u);
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int e = 4 * i;
            float acc = fmaf(wv[(e + 3) >> 3][(e + 3) & 7], cur[i], bv[i]);
            acc += ok2 ? wv[(e + 2) >> 3][(e + 2) & 7] * win[2][i] : 0.0f;
            acc += ok1 ? wv[(e + 1) >> 3][(e + 1) & 7] * win[1][i] : 0.0f;
            acc += ok0 ? wv[e >> 3][e & 7] * win[0][i] : 0.0f;
            o[i] = sizeof(OutT) == 2 ? silu_t(acc) : silu_f(acc);
        }
        store8(dst + t * (cd - cbase), o);
        win[0] = win[1];
        win[1] = win[2];
        win[2] = cur;
    }
}

// bf16 input: the same arithmetic with every input row of the thread (three
// history rows + its eight tokens) requested before any is used, so each thread
// keeps eleven 16-byte loads in flight -- enough bytes in flight per SM to run
// near HBM bandwidth at two resident blocks.  Rows stay packed (4 registers
// each) and are widened on use.
template <typename OutT>
__global__ void __launch_bounds__(256, 2)
conv_silu_bf16_kernel(Shape s, const bf16* __restrict__ x, const bf16* __restrict__ Bm,
                      const bf16* __restrict__ Cm, const bf16* __restrict__ w,
                      const bf16* __restrict__ bias, const int32_t* __restrict__ seq,
                      const bf16* __restrict__ hist0, OutT* __restrict__ u, int cbase,
                      RawStrides ld)
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
    const bf16* src = channel_src(s, ld, x, Bm, Cm, c, stride, col);
    src += (int64_t)b * L * stride + col;
    const int t0 = tg * kTokPerThread;

    Vec8<bf16> row[kTokPerThread + 3];      // rows t0-3 .. t0+7
#pragma unroll
    for (int j = 0; j < kTokPerThread + 3; j++) {
        const int64_t tau = (int64_t)t0 - 3 + j;
        if (tau >= 0 && tau < L) row[j].load(src + tau * stride);
        else if (tau < 0 && hist0 != nullptr) row[j].load(hist0 + ((int64_t)b * 3 + (tau + 3)) * cd + c);
        else row[j].zero();
    }
    Vec8<bf16> wv[4], bv;       // weight (channel i, tap k) = element 4*i + k
#pragma unroll
    for (int q = 0; q < 4; q++) wv[q].load(w + (int64_t)c * 4 + q * 8);
    bv.load(bias + c);

    const int32_t* seq_row = seq ? seq + (int64_t)b * L : nullptr;
    uint32_t bdm = 0;           // bit j: boundary at position t0 - 2 + j
#pragma unroll
    for (int j = 0; j < kTokPerThread + 2; j++) {
        const int64_t pos = (int64_t)t0 - 2 + j;
        if (pos >= 1 && pos < L && is_boundary(seq_row, pos)) bdm |= 1u << j;
    }

    OutT* dst = u + (int64_t)b * L * (cd - cbase) + (c - cbase);
    if (bdm == 0) {
        // no document boundary near these tokens: every tap is used
#pragma unroll
        for (int q = 0; q < kTokPerThread; q++) {
            const int64_t t = t0 + q;
            if (t >= L) break;
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int e = 4 * i;
                float acc = fmaf(wv[(e + 3) >> 3][(e + 3) & 7], row[q + 3][i], bv[i]);
                acc = fmaf(wv[(e + 2) >> 3][(e + 2) & 7], row[q + 2][i], acc);
                acc = fmaf(wv[(e + 1) >> 3][(e + 1) & 7], row[q + 1][i], acc);
                acc = fmaf(wv[e >> 3][e & 7], row[q][i], acc);
                o[i] = sizeof(OutT) == 2 ? silu_t(acc) : silu_f(acc);
            }
            store8(dst + t * (cd - cbase), o);
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < kTokPerThread; q++) {
        const int64_t t = t0 + q;
        if (t >= L) break;
        // tap k reads row t-3+k; valid when no boundary at positions t-2+k .. t
        const bool ok2 = !((bdm >> (q + 2)) & 1u);
        const bool ok1 = ok2 && !((bdm >> (q + 1)) & 1u);
        const bool ok0 = ok1 && !((bdm >> q) & 1u);
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int e = 4 * i;
            float acc = fmaf(wv[(e + 3) >> 3][(e + 3) & 7], row[q + 3][i], bv[i]);
            acc += ok2 ? wv[(e + 2) >> 3][(e + 2) & 7] * row[q + 2][i] : 0.0f;
            acc += ok1 ? wv[(e + 1) >> 3][(e + 1) & 7] * row[q + 1][i] : 0.0f;
            acc += ok0 ? wv[e >> 3][e & 7] * row[q][i] : 0.0f;
            o[i] = sizeof(OutT) == 2 ? silu_t(acc) : silu_f(acc);
        }
        store8(dst + t * (cd - cbase), o);
    }
}

// 1/rms of one N-long B or C row per thread: rinv[(b L + t) 2G + which G + g].
__global__ void __launch_bounds__(256)
bc_rms_kernel(Shape s, const bf16* __restrict__ Bm, const bf16* __restrict__ Cm,
              const bf16* __restrict__ ubc, float* __restrict__ rinv, int64_t ld_bc)
{
    const int G = s.ngroups, N = s.dstate;
    const int64_t rows = (int64_t)s.batch * s.seqlen * 2 * G;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows) return;
    const int64_t tok = gid / (2 * G);
    const int k = (int)(gid % (2 * G));          // which * G + g
    const bf16* src = ubc ? ubc + tok * (2 * G * N) + (int64_t)k * N
                          : (k < G ? Bm : Cm) + tok * ld_bc + (int64_t)(k % G) * N;
    float ss = 0.0f;
    for (int n = 0; n < N; n += 8) {
        Vec8<bf16> v;
        v.load(src + n);
#pragma unroll
        for (int j = 0; j < 8; j++) ss = fmaf(v[j], v[j], ss);
    }
    rinv[gid] = rsqrtf(ss / N + kNormEps);
}

cudaError_t launch_bc_rms(const Shape& s, const FwdArgs& a, const void* ubc, float* rinv, cudaStream_t st)
{
    if (!s.act_bf16 || s.dstate % 8) return cudaErrorInvalidValue;
    const int64_t rows = (int64_t)s.batch * s.seqlen * 2 * s.ngroups;
    bc_rms_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(
        s, (const bf16*)a.B, (const bf16*)a.C, (const bf16*)ubc, rinv, a.ld_bc);
    return cudaGetLastError();
}

// Final conv history: slot i holds the raw input at L-3+i when it lies in the
// last token's document, else 0.  Each thread reads its 3 slots before writing
// them, so the initial and final history may be the same buffer.
template <typename T>
__global__ void __launch_bounds__(256)
conv_state_kernel(Shape s, const T* __restrict__ x, const T* __restrict__ Bm,
                  const T* __restrict__ Cm, const int32_t* __restrict__ seq,
                  const int32_t* __restrict__ lengths, const T* hist0, T* hist1, RawStrides ld)
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
    const T* src = channel_src(s, ld, x, Bm, Cm, c, stride, col);
    src += (int64_t)b * L * stride + col;

    // the row's last real token is Lb - 1 (Lb = L unless the batch is ragged)
    const int Lb = row_length(lengths, b, L);
    float vals[3][8];
#pragma unroll
    for (int i = 0; i < 3; i++) {
        const int64_t tau = (int64_t)Lb - 3 + i;
        int ok = 1;
        for (int64_t pos = (tau + 1 > 1 ? tau + 1 : 1); pos <= Lb - 1; pos++)
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
    if constexpr (sizeof(T) == 2)
        conv_silu_bf16_kernel<OutT><<<(unsigned)blocks, 256, 0, st>>>(
            s, (const bf16*)a.x, (const bf16*)a.B, (const bf16*)a.C, (const bf16*)a.conv_w,
            (const bf16*)a.conv_b, a.seq_idx, (const bf16*)a.init_conv, u, cbase,
            RawStrides{a.ld_x, a.ld_bc});
    else
        conv_silu_kernel<T, OutT><<<(unsigned)blocks, 256, 0, st>>>(
            s, (const T*)a.x, (const T*)a.B, (const T*)a.C, (const T*)a.conv_w, (const T*)a.conv_b,
            a.seq_idx, (const T*)a.init_conv, u, cbase, RawStrides{a.ld_x, a.ld_bc});
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
            s, (const bf16*)a.x, (const bf16*)a.B, (const bf16*)a.C, a.seq_idx, a.lengths,
            (const bf16*)a.init_conv, (bf16*)a.final_conv, RawStrides{a.ld_x, a.ld_bc});
    else
        conv_state_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            s, (const float*)a.x, (const float*)a.B, (const float*)a.C, a.seq_idx, a.lengths,
            (const float*)a.init_conv, (float*)a.final_conv, RawStrides{a.ld_x, a.ld_bc});
    return cudaGetLastError();
}

}  // namespace ssd
