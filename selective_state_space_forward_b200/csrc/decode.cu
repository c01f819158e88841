// decode.cu -- K6: one decode token per row, state updated in place.
//
// mojolearn Mamba3Block.step: "the same computation as forward at L = 1 with
// the state carried".  Per row b and head h:
//   conv window  [hist_0, hist_1, hist_2, x_new] -> u = SiLU(conv) (kernel 4),
//                history shifted by one token (model card, Architecture)
//   dt           softplus(dt_raw + dt_bias[h]);  a = A[h] or min(A[b,h], -1e-4)
//   state        h[p,n] <- exp(dt a) h[p,n] + dt u_x[p] B[n]      (fp32, in place)
//   output       out[p] = (sum_n C[n] h[p,n] + D[h] u_x[p]) * SiLU(z[p])
//
// One block per (row, B/C group): the group's B|C conv channels and its heads'
// x channels are convolved once, so each conv-history column has exactly one
// reader/writer.  The state is 95% of the bytes and is read and written once:
// in the main kernel 8 lanes share a state row (each lane a float4 per 32
// floats of the row, so a row is read in full 128-byte pieces), a warp walks 4
// rows at a time, the next rows' loads are issued before the current rows are
// computed, and the row's C.h sum is reduced over its 8 lanes.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kDecodeThreads = 128;

// Conv + SiLU of the new token, dt and decay per head, B/C norm: fills the
// block's shared arrays ux[hpg*P], ub[N], uc[N], dts[hpg], dec[hpg] and, with
// the norm, the per-head bh/ch[hpg][N].  Ends with a block barrier.
template <typename T>
__device__ void decode_prologue(const Shape& s, const FwdArgs& a, T* hist, float* ux, float* ub,
                                float* uc, float* dts, float* dec, float* bh, float* ch, int g, int b)
{
    const int H = s.nheads, P = s.headdim, N = s.dstate, G = s.ngroups;
    const int hpg = H / G, HP = H * P, GN = G * N, cd = s.conv_dim();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const T* x = (const T*)a.x;
    const T* Bm = (const T*)a.B;
    const T* Cm = (const T*)a.C;
    const T* w = (const T*)a.conv_w;
    const T* cb = (const T*)a.conv_b;
    const int nch = hpg * P + 2 * N;
    for (int i = tid; i < nch; i += blockDim.x) {
        int c;
        float raw;
        float* dst;
        if (i < hpg * P) {
            c = g * hpg * P + i;
            raw = to_f(x[(int64_t)b * HP + c]);
            dst = ux + i;
        } else if (i < hpg * P + N) {
            const int n = i - hpg * P;
            c = HP + g * N + n;
            raw = to_f(Bm[(int64_t)b * GN + g * N + n]);
            dst = ub + n;
        } else {
            const int n = i - hpg * P - N;
            c = HP + GN + g * N + n;
            raw = to_f(Cm[(int64_t)b * GN + g * N + n]);
            dst = uc + n;
        }
        if (s.dconv == kConvK) {
            T* hc = hist + (int64_t)b * 3 * cd + c;
            const float h0 = to_f(hc[0]), h1 = to_f(hc[cd]), h2 = to_f(hc[2 * cd]);
            const T* wc = w + (int64_t)c * 4;
            const float acc = to_f(cb[c]) + to_f(wc[0]) * h0 + to_f(wc[1]) * h1 +
                              to_f(wc[2]) * h2 + to_f(wc[3]) * raw;
            hc[0] = from_f<T>(h1);
            hc[cd] = from_f<T>(h2);
            hc[2 * cd] = from_f<T>(raw);
            *dst = silu_f(acc);
        } else {
            *dst = raw;
        }
    }
    for (int i = tid; i < hpg; i += blockDim.x) {
        const int h = g * hpg + i;
        const float dtv = softplus_f(a.dt_raw[(int64_t)b * H + h] + a.dt_bias[h]);
        const float av = s.a_per_token ? fminf(a.A[(int64_t)b * H + h], -kAFloor) : a.A[h];
        dts[i] = dtv;
        dec[i] = expf(dtv * av);
    }
    __syncthreads();
    if (s.bc_norm) {
        // warps 0 / 1 normalise B / C; every thread then adds the heads' biases
        if (warp < 2) {
            float* v = warp ? uc : ub;
            float ss = 0.0f;
            for (int n = lane; n < N; n += 32) ss += v[n] * v[n];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float rs = rsqrtf(ss / N + kNormEps);
            const float* wn = warp ? a.cn_w : a.bn_w;
            __syncwarp();
            for (int n = lane; n < N; n += 32) v[n] = v[n] * rs * (wn ? wn[n] : 1.0f);
        }
        __syncthreads();
        for (int i = tid; i < hpg * N; i += blockDim.x) {
            const int h = g * hpg + i / N, n = i % N;
            bh[i] = ub[n] + (a.bn_bias ? a.bn_bias[(int64_t)h * N + n] : 0.0f);
            ch[i] = uc[n] + (a.cn_bias ? a.cn_bias[(int64_t)h * N + n] : 0.0f);
        }
        __syncthreads();
    }
}

struct DecodeSmem {
    float *ux, *ub, *uc, *dts, *dec, *bh, *ch, *gz, *ys;
    __device__ DecodeSmem(float* sm, const Shape& s)
    {
        const int hpg = s.nheads / s.ngroups;
        const int hp4 = (hpg + 3) & ~3;      // keeps bh/ch 16-byte aligned
        ux = sm;
        ub = ux + hpg * s.headdim;
        uc = ub + s.dstate;
        dts = uc + s.dstate;
        dec = dts + hp4;
        bh = dec + hp4;
        ch = bh + (s.bc_norm ? hpg * s.dstate : 0);
        gz = ch + (s.bc_norm ? hpg * s.dstate : 0);   // SiLU(z) of the block's rows
        ys = gz + hpg * s.headdim;                     // C . h of the block's rows
    }
};
__host__ __device__ inline size_t decode_smem_floats(int hpg, int P, int N, bool bc_norm)
{
    const size_t hp4 = (size_t)((hpg + 3) & ~3);
    return (size_t)hpg * P + 2 * (size_t)N + 2 * hp4 + (bc_norm ? 2 * (size_t)hpg * N : 0) +
           2 * (size_t)hpg * P;
}

// Main kernel: N = 32 * NV.  Lane l8 of a row owns float4 q at floats
// (q * 8 + l8) * 4 .. +3, so the 8 lanes of a row cover 32 consecutive floats
// per q.
template <typename T, int NV>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_vec(Shape s, FwdArgs a, float* __restrict__ ssm, T* __restrict__ hist)
{
    extern __shared__ float sm[];
    const int H = s.nheads, P = s.headdim, N = s.dstate;
    const int hpg = H / s.ngroups, HP = H * P;
    const int g = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    DecodeSmem sv(sm, s);
    // SiLU(z) of the block's rows, so the row loop's output needs no global load
    for (int i = threadIdx.x; i < hpg * P; i += blockDim.x)
        sv.gz[i] = silu_f(to_f(((const T*)a.z)[(int64_t)b * HP + (int64_t)g * hpg * P + i]));
    decode_prologue<T>(s, a, hist, sv.ux, sv.ub, sv.uc, sv.dts, sv.dec, sv.bh, sv.ch, g, b);

    const int sub = lane >> 3, l8 = lane & 7;
    float4 Bq[NV], Cq[NV];
    if (!s.bc_norm) {
#pragma unroll
        for (int q = 0; q < NV; q++) {
            Bq[q] = *reinterpret_cast<const float4*>(sv.ub + (q * 8 + l8) * 4);
            Cq[q] = *reinterpret_cast<const float4*>(sv.uc + (q * 8 + l8) * 4);
        }
    }
    const int nrows = hpg * P;
    const int step = nw * 4;
    float* base = ssm + ((int64_t)b * H + (int64_t)g * hpg) * P * N;   // row r at base + r*N
    auto load_row = [&](int r, float4 (&v)[NV]) {
        if (r < nrows) {
#pragma unroll
            for (int q = 0; q < NV; q++)
                v[q] = *reinterpret_cast<const float4*>(base + (int64_t)r * N + (q * 8 + l8) * 4);
        }
    };
    int r = warp * 4 + sub;
    float4 cur[NV], nxt[NV];
    load_row(r, cur);
    for (; r - sub < nrows; r += step) {
        load_row(r + step, nxt);
        const bool valid = r < nrows;
        const int hl = valid ? r / P : 0;
        const float xdt = valid ? sv.dts[hl] * sv.ux[r] : 0.f;
        const float d = sv.dec[hl];
        float y = 0.f;
#pragma unroll
        for (int q = 0; q < NV; q++) {
            float4 bv = Bq[q], cv = Cq[q];
            if (s.bc_norm) {
                bv = *reinterpret_cast<const float4*>(sv.bh + hl * N + (q * 8 + l8) * 4);
                cv = *reinterpret_cast<const float4*>(sv.ch + hl * N + (q * 8 + l8) * 4);
            }
            float4 hv;
            hv.x = fmaf(d, cur[q].x, xdt * bv.x);
            hv.y = fmaf(d, cur[q].y, xdt * bv.y);
            hv.z = fmaf(d, cur[q].z, xdt * bv.z);
            hv.w = fmaf(d, cur[q].w, xdt * bv.w);
            y = fmaf(cv.x, hv.x, y);
            y = fmaf(cv.y, hv.y, y);
            y = fmaf(cv.z, hv.z, y);
            y = fmaf(cv.w, hv.w, y);
            if (valid)
                *reinterpret_cast<float4*>(base + (int64_t)r * N + (q * 8 + l8) * 4) = hv;
        }
        y += __shfl_xor_sync(0xffffffffu, y, 1);
        y += __shfl_xor_sync(0xffffffffu, y, 2);
        y += __shfl_xor_sync(0xffffffffu, y, 4);
        if (valid && l8 == 0) sv.ys[r] = y;
#pragma unroll
        for (int q = 0; q < NV; q++) cur[q] = nxt[q];
    }
    __syncthreads();
    // the block's outputs, one coalesced row of hpg * P values
    for (int i = threadIdx.x; i < nrows; i += blockDim.x) {
        const int hh = g * hpg + i / P;
        ((T*)a.out)[(int64_t)b * HP + (int64_t)g * hpg * P + i] =
            from_f<T>((sv.ys[i] + a.D[hh] * sv.ux[i]) * sv.gz[i]);
    }
}

// General kernel for any d_state (a multiple of 8): a warp per state row.
template <typename T>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_any(Shape s, FwdArgs a, float* __restrict__ ssm, T* __restrict__ hist)
{
    extern __shared__ float sm[];
    const int H = s.nheads, P = s.headdim, N = s.dstate;
    const int hpg = H / s.ngroups, HP = H * P;
    const int g = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    DecodeSmem sv(sm, s);
    decode_prologue<T>(s, a, hist, sv.ux, sv.ub, sv.uc, sv.dts, sv.dec, sv.bh, sv.ch, g, b);
    const int nrows = hpg * P;
    for (int r = warp; r < nrows; r += nw) {
        const int hl = r / P;
        const float* Bv = s.bc_norm ? sv.bh + hl * N : sv.ub;
        const float* Cv = s.bc_norm ? sv.ch + hl * N : sv.uc;
        const float xdt = sv.dts[hl] * sv.ux[r], d = sv.dec[hl];
        float* row = ssm + (((int64_t)b * H + g * hpg + hl) * P + r % P) * N;
        float y = 0.f;
        for (int n = lane; n < N; n += 32) {
            const float hv = fmaf(d, row[n], xdt * Bv[n]);
            row[n] = hv;
            y = fmaf(Cv[n], hv, y);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
        if (lane == 0) {
            const int hh = g * hpg + hl;
            const int64_t o = (int64_t)b * HP + hh * P + r % P;
            ((T*)a.out)[o] = from_f<T>((y + a.D[hh] * sv.ux[r]) * silu_f(to_f(((const T*)a.z)[o])));
        }
    }
}

template <typename T>
static cudaError_t launch_decode_t(const Shape& s, const FwdArgs& a, float* ssm, void* hist,
                                   cudaStream_t st)
{
    const int hpg = s.nheads / s.ngroups;
    const size_t smem = sizeof(float) * decode_smem_floats(hpg, s.headdim, s.dstate, s.bc_norm);
    const dim3 grid(s.ngroups, s.batch);
    void (*kern)(Shape, FwdArgs, float*, T*);
    switch (s.dstate) {
    case 32: kern = decode_step_vec<T, 1>; break;
    case 64: kern = decode_step_vec<T, 2>; break;
    case 128: kern = decode_step_vec<T, 4>; break;
    case 256: kern = decode_step_vec<T, 8>; break;
    default: kern = decode_step_any<T>; break;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kDecodeThreads, smem, st>>>(s, a, ssm, (T*)hist);
    return cudaGetLastError();
}

cudaError_t launch_decode_step(const Shape& s, const FwdArgs& a, float* ssm, void* conv_hist,
                               cudaStream_t st)
{
    return s.act_bf16 ? launch_decode_t<bf16>(s, a, ssm, conv_hist, st)
                      : launch_decode_t<float>(s, a, ssm, conv_hist, st);
}

}  // namespace ssd
