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
// reader/writer.  The state is the traffic (95% of the bytes): each warp owns
// state rows (head, p) of N floats, loads four rows' vectors before using any
// (memory-level parallelism), and writes each element back once.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kDecodeThreads = 128;
constexpr int kRowsInFlight = 4;

template <typename T, int V>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(Shape s, FwdArgs a, float* __restrict__ ssm, T* __restrict__ hist)
{
    extern __shared__ float sm[];
    const int H = s.nheads, P = s.headdim, N = s.dstate, G = s.ngroups;
    const int hpg = H / G, HP = H * P, GN = G * N, cd = s.conv_dim();
    const int g = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    float* ux = sm;                 // [hpg*P]
    float* ub = ux + hpg * P;       // [N]
    float* uc = ub + N;             // [N]
    float* dts = uc + N;            // [hpg]
    float* dec = dts + hpg;         // [hpg]
    float* bh = dec + hpg;          // [hpg][N] (B/C norm only)
    float* ch = bh + (s.bc_norm ? hpg * N : 0);

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
    if (tid < hpg) {
        const int h = g * hpg + tid;
        const float dtv = softplus_f(a.dt_raw[(int64_t)b * H + h] + a.dt_bias[h]);
        const float av = s.a_per_token ? fminf(a.A[(int64_t)b * H + h], -kAFloor) : a.A[h];
        dts[tid] = dtv;
        dec[tid] = expf(dtv * av);
    }
    __syncthreads();
    if (s.bc_norm) {
        // warps 0 / 1 normalise B / C; every warp then adds the heads' biases
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

    // state rows (hl, p), kRowsInFlight at a time per warp
    const int nrows = hpg * P;
    for (int r0 = warp * kRowsInFlight; r0 < nrows; r0 += nw * kRowsInFlight) {
        float st[kRowsInFlight][V];
        float* rowp[kRowsInFlight];
#pragma unroll
        for (int q = 0; q < kRowsInFlight; q++) {
            const int row = r0 + q;
            const int hl = row / P, p = row % P;
            rowp[q] = ssm + (((int64_t)b * H + g * hpg + hl) * P + p) * N;
        }
        float ysum[kRowsInFlight];
#pragma unroll
        for (int q = 0; q < kRowsInFlight; q++) ysum[q] = 0.0f;
        for (int n0 = lane * V; n0 < N; n0 += 32 * V) {
#pragma unroll
            for (int q = 0; q < kRowsInFlight; q++) {
                if (V == 4) {
                    const float4 t4 = *reinterpret_cast<const float4*>(rowp[q] + n0);
                    st[q][0] = t4.x; st[q][1] = t4.y; st[q][2] = t4.z; st[q][3] = t4.w;
                } else if (V == 2) {
                    const float2 t2 = *reinterpret_cast<const float2*>(rowp[q] + n0);
                    st[q][0] = t2.x; st[q][1] = t2.y;
                } else {
                    st[q][0] = rowp[q][n0];
                }
            }
#pragma unroll
            for (int q = 0; q < kRowsInFlight; q++) {
                const int row = r0 + q;
                const int hl = row / P;
                const float* Bv = s.bc_norm ? bh + hl * N : ub;
                const float* Cv = s.bc_norm ? ch + hl * N : uc;
                const float xdt = dts[hl] * ux[row];
                const float d = dec[hl];
#pragma unroll
                for (int k = 0; k < V; k++) {
                    const float hv = d * st[q][k] + xdt * Bv[n0 + k];
                    st[q][k] = hv;
                    ysum[q] += Cv[n0 + k] * hv;
                }
                if (V == 4) {
                    *reinterpret_cast<float4*>(rowp[q] + n0) =
                        make_float4(st[q][0], st[q][1], st[q][2], st[q][3]);
                } else if (V == 2) {
                    *reinterpret_cast<float2*>(rowp[q] + n0) = make_float2(st[q][0], st[q][1]);
                } else {
                    rowp[q][n0] = st[q][0];
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kRowsInFlight; q++) {
            float y = ysum[q];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
            if (lane == 0) {
                const int row = r0 + q;
                const int hl = row / P, p = row % P, h = g * hpg + hl;
                const int64_t o = (int64_t)b * HP + h * P + p;
                const float zv = to_f(((const T*)a.z)[o]);
                ((T*)a.out)[o] = from_f<T>((y + a.D[h] * ux[row]) * silu_f(zv));
            }
        }
    }
}

template <typename T>
static cudaError_t launch_decode_t(const Shape& s, const FwdArgs& a, float* ssm, void* hist,
                                   cudaStream_t st)
{
    const int hpg = s.nheads / s.ngroups;
    const size_t smem = sizeof(float) * ((size_t)hpg * s.headdim + 2 * s.dstate + 2 * hpg +
                                         (s.bc_norm ? 2 * (size_t)hpg * s.dstate : 0));
    const dim3 grid(s.ngroups, s.batch);
    auto kern = (s.dstate % 128 == 0) ? decode_step_kernel<T, 4>
              : (s.dstate % 64 == 0) ? decode_step_kernel<T, 2> : decode_step_kernel<T, 1>;
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
