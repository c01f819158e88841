// staged_rows.cuh -- per-chunk pieces shared by the staged forward kernels and the
// backward kernels: chunk-local document segments, the (64-token) rows of x, B
// and C a block works on, in fp32, and a register-tiled product over them.
#pragma once
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

// Chunk-local segment ids: seg[t] = boundaries at positions t0 .. t0+t (padding
// positions, at or after the row length Lb, hold none).
// The inclusive prefix count runs on warps 0 and 1 by ballots.
__device__ inline void chunk_segments(const int32_t* seq_row, int t0, int Lc, int Lb, int* seg, int* flag)
{
    const int tid = threadIdx.x;
    if (tid < kChunk) flag[tid] = (tid < Lc && t0 + tid < Lb) ? is_boundary(seq_row, t0 + tid) : 0;
    __syncthreads();
    if (tid < kChunk) {
        const int lane = tid & 31;
        const uint32_t m0 = __ballot_sync(0xffffffffu, flag[lane] != 0);
        const uint32_t m1 = __ballot_sync(0xffffffffu, flag[32 + lane] != 0);
        const uint32_t le = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);
        seg[tid] = tid < 32 ? __popc(m0 & le) : __popc(m0) + __popc(m1 & le);
    }
    __syncthreads();
}

// Eight consecutive values as floats: two 16-byte loads (fp32) or one (bf16) when
// the address is 16-byte aligned, else element by element.
__device__ __forceinline__ void ld8(const float* p, bool vec, float (&v)[8])
{
    if (vec) {
        const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = p[e];
    }
}
__device__ __forceinline__ void ld8(const bf16* p, bool vec, float (&v)[8])
{
    if (vec) {
        load8(p, v);
    } else {
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = __bfloat162float(p[e]);
    }
}
__device__ __forceinline__ bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Rows [t0, t0+64) of width W (a multiple of 8) from src (row r at src + r * ld_src)
// into dst (row r at dst + r * ld_dst), zero past Lc.  Each task moves 8 values;
// a thread issues the loads of two tasks before storing.  Loads and stores are
// 16 bytes wide where both the base and the row stride keep 16-byte alignment.
template <typename S>
__device__ __forceinline__ void load_rows8(const S* src, int64_t ld_src, int W, int Lc, float* dst, int ld_dst,
                                           int rows = kChunk)
{
    const int per = W / 8, ntask = rows * per;
    const bool vec = aligned16(src) && (ld_src * (int64_t)sizeof(S)) % 16 == 0;
    const bool vst = aligned16(dst) && ld_dst % 4 == 0;
    for (int i0 = threadIdx.x; i0 < ntask; i0 += 2 * blockDim.x) {
        float v[2][8];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int i = i0 + k * blockDim.x;
            const int r = i / per, c = (i % per) * 8;
            if (i < ntask && r < Lc) {
                ld8(src + r * ld_src + c, vec, v[k]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; e++) v[k][e] = 0.0f;
            }
        }
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int i = i0 + k * blockDim.x;
            if (i < ntask) {
                float* d = dst + (i / per) * ld_dst + (i % per) * 8;
                if (vst) {
                    *reinterpret_cast<float4*>(d) = make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
                    *reinterpret_cast<float4*>(d + 4) = make_float4(v[k][4], v[k][5], v[k][6], v[k][7]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; e++) d[e] = v[k][e];
                }
            }
        }
    }
}

// Load token rows [t0, t0+64) of the head's x (fp32 result, zero past the end);
// ld is the destination row stride (a multiple of 4).
template <typename T>
__device__ void load_x_rows(const Shape& s, const FwdArgs& a, const float* u, int b, int h,
                            int t0, int Lc, float* xs, int ld)
{
    const int P = s.headdim, cd = s.conv_dim();
    const int64_t tok0 = (int64_t)b * s.seqlen + t0;
    if (u) load_rows8(u + tok0 * cd + h * P, cd, P, Lc, xs, ld);
    else load_rows8((const T*)a.x + tok0 * a.ld_x + h * P, a.ld_x, P, Lc, xs, ld);
}

// Load B (which = 0) or C (which = 1) rows of the head's group, then apply the
// B/C norm and the head's bias when enabled.
template <typename T>
__device__ void load_bc_rows(const Shape& s, const FwdArgs& a, const float* u, int b, int h,
                             int t0, int Lc, int which, float* dst, int ld)
{
    const int N = s.dstate, GN = s.ngroups * N, HP = s.nheads * s.headdim, cd = s.conv_dim();
    const int g = h / (s.nheads / s.ngroups);
    const int64_t tok0 = (int64_t)b * s.seqlen + t0;
    if (u) load_rows8(u + tok0 * cd + HP + which * GN + g * N, cd, N, Lc, dst, ld);
    else load_rows8((const T*)(which ? a.C : a.B) + tok0 * a.ld_bc + g * N, a.ld_bc, N, Lc, dst, ld);
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

// Register-tiled fp32 product over shared-memory operands.  Thread (it, jt) =
// (tid / 16, tid % 16) accumulates
//   acc[rr][cc] += sum_{k < K} A(i, k) B(k, j) [s_k],   i = it + 16 rr, j = jt + 16 cc,
// with A(i, k) = A[i a_si + k a_sk] and B(k, j) = B[k b_sk + j b_sj], k in order
// (so results repeat bit for bit); s_k scales A's column k when given.  Rows at or
// past R and columns at or past C read the last valid row / column: the caller
// discards those results.  The strides the kernels pass keep a warp's 16 columns
// on 16 banks and its 2 rows on different banks.
template <int TC>
__device__ __forceinline__ void tile_mm(float (&acc)[4][TC], const float* A, int a_si, int a_sk, int R,
                                        const float* B, int b_sk, int b_sj, int C, int K, int it, int jt,
                                        const float* sk = nullptr)
{
    const float* ap[4];
    const float* bp[TC];
#pragma unroll
    for (int rr = 0; rr < 4; rr++) ap[rr] = A + min(it + 16 * rr, R - 1) * a_si;
#pragma unroll
    for (int cc = 0; cc < TC; cc++) bp[cc] = B + min(jt + 16 * cc, C - 1) * b_sj;
#pragma unroll 4
    for (int k = 0; k < K; k++) {
        float av[4], bv[TC];
        const float sc = sk ? sk[k] : 1.0f;
#pragma unroll
        for (int rr = 0; rr < 4; rr++) av[rr] = sk ? ap[rr][k * a_sk] * sc : ap[rr][k * a_sk];
#pragma unroll
        for (int cc = 0; cc < TC; cc++) bv[cc] = bp[cc][k * b_sk];
#pragma unroll
        for (int rr = 0; rr < 4; rr++)
#pragma unroll
            for (int cc = 0; cc < TC; cc++) acc[rr][cc] = fmaf(av[rr], bv[cc], acc[rr][cc]);
    }
}

// The same product on the tensor cores (mma.sync m16n8k8, tf32 operands rounded
// to nearest, fp32 accumulation), for operands that tolerate tf32 rounding: a
// warp w owns rows 16 (w % 4) .. +15 and columns 8 TC (w / 4) .. +8 TC - 1 of
// the 64 x 16 TC output; accumulator element (rr, cc) is that of MmaMap below.
// K must be a multiple of 8 (rows of zeros pad a short chunk).
struct SimtMap {
    int it, jt;
    __device__ explicit SimtMap(int tid) : it(tid >> 4), jt(tid & 15) {}
    __device__ int row(int rr, int) const { return it + 16 * rr; }
    __device__ int col(int, int cc) const { return jt + 16 * cc; }
};
template <int TC>
struct MmaMap {
    int r0, c0;
    __device__ explicit MmaMap(int tid)
        : r0(16 * ((tid >> 5) & 3) + ((tid & 31) >> 2)), c0(8 * TC * (tid >> 7) + 2 * (tid & 3)) {}
    __device__ int row(int rr, int) const { return r0 + 8 * (rr >> 1); }
    __device__ int col(int rr, int cc) const { return c0 + 8 * cc + (rr & 1); }
};

__device__ __forceinline__ uint32_t to_tf32(float v)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
    return r;
}

template <int TC>
__device__ __forceinline__ void tile_mm_tc(float (&acc)[4][TC], const float* A, int a_si, int a_sk, int R,
                                           const float* B, int b_sk, int b_sj, int C, int K, int tid,
                                           const float* sk = nullptr)
{
    const int w = tid >> 5, g = (tid & 31) >> 2, t4 = tid & 3;
    const int row0 = 16 * (w & 3), col0 = 8 * TC * (w >> 2);
    const float* alo = A + min(row0 + g, R - 1) * a_si;
    const float* ahi = A + min(row0 + g + 8, R - 1) * a_si;
    const float* bp[TC];
#pragma unroll
    for (int cc = 0; cc < TC; cc++) bp[cc] = B + min(col0 + 8 * cc + g, C - 1) * b_sj;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        const int ka = k0 + t4, kb = ka + 4;
        float x0 = alo[ka * a_sk], x1 = ahi[ka * a_sk], x2 = alo[kb * a_sk], x3 = ahi[kb * a_sk];
        if (sk) {
            const float sa = sk[ka], sb = sk[kb];
            x0 *= sa; x1 *= sa; x2 *= sb; x3 *= sb;
        }
        const uint32_t a0 = to_tf32(x0), a1 = to_tf32(x1), a2 = to_tf32(x2), a3 = to_tf32(x3);
#pragma unroll
        for (int cc = 0; cc < TC; cc++) {
            const uint32_t b0 = to_tf32(bp[cc][ka * b_sk]), b1 = to_tf32(bp[cc][kb * b_sk]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
                "{%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[0][cc]), "+f"(acc[1][cc]), "+f"(acc[2][cc]), "+f"(acc[3][cc])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}

template <int TC>
__device__ __forceinline__ void tile_zero(float (&acc)[4][TC])
{
#pragma unroll
    for (int rr = 0; rr < 4; rr++)
#pragma unroll
        for (int cc = 0; cc < TC; cc++) acc[rr][cc] = 0.0f;
}

// The contraction engine of a kernel instance: the tensor cores (tf32 operands,
// fp32 accumulation) for bf16 activations, whose inputs tf32 holds exactly;
// fp32 SIMT for fp32 activations, whose 1e-5 tolerance tf32 rounding would miss.
// Both give a thread the same 4 x TC accumulator; row() and col() name the output
// element each entry holds.
template <typename T, int TC>
struct Prod {
    SimtMap m;
    __device__ explicit Prod(int tid) : m(tid) {}
    __device__ void mm(float (&acc)[4][TC], const float* A, int a_si, int a_sk, int R, const float* B,
                       int b_sk, int b_sj, int C, int K, const float* sk = nullptr) const
    {
        tile_mm<TC>(acc, A, a_si, a_sk, R, B, b_sk, b_sj, C, K, m.it, m.jt, sk);
    }
    __device__ int row(int rr, int cc) const { return m.row(rr, cc); }
    __device__ int col(int rr, int cc) const { return m.col(rr, cc); }
};
template <int TC>
struct Prod<bf16, TC> {
    MmaMap<TC> m;
    int tid;
    __device__ explicit Prod(int t) : m(t), tid(t) {}
    __device__ void mm(float (&acc)[4][TC], const float* A, int a_si, int a_sk, int R, const float* B,
                       int b_sk, int b_sj, int C, int K, const float* sk = nullptr) const
    {
        tile_mm_tc<TC>(acc, A, a_si, a_sk, R, B, b_sk, b_sj, C, K, tid, sk);
    }
    __device__ int row(int rr, int cc) const { return m.row(rr, cc); }
    __device__ int col(int rr, int cc) const { return m.col(rr, cc); }
};

// Row strides of the shared-memory operands: 4 floats of padding spread a warp's
// fragment loads over the banks.
constexpr int kPad = 4;
constexpr int kMS = kChunk + kPad;     // [64][64] token x token arrays

}  // namespace ssd
