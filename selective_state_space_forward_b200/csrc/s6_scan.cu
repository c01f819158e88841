// s6_scan.cu -- the Mamba-1 selective scan (S6) of the Falcon-Mamba port
// (falcon_mamba.ts header: a Mamba-1 / S6 model; A = -exp(clamp(A_log, -10, 5))
// as selective_scan.ts computes it; dt = softplus(dt + bias)).  Per batch row b
// and channel d, state size N:
//
//   h[n] <- exp(dt_t A[d,n]) h[n] + dt_t u_t B_t[n];   y_t = C_t . h + D[d] u_t
//   out_t = y_t SiLU(z_t)   (no z: y_t)
//
// A is diagonal, so channels never mix: one thread owns one channel and keeps
// its N states and N decay rates (pre-scaled by log2 e) in registers.  A block
// of 128 consecutive channels walks the sequence together; each 64-token chunk
// of B and C (shared by every channel of a token) is staged in shared memory
// once per block, and u, dt and z are read coalesced across the block's
// channels.  The bound is the N exponentials per (token, channel) on the MUFU
// pipe, then HBM.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kS6Threads = 128;
constexpr int kS6Chunk = 64;

template <typename T, int N>
__global__ void __launch_bounds__(kS6Threads)
s6_scan_kernel(int batch, int L, int DI, const T* __restrict__ u, const float* __restrict__ delta,
               const float* __restrict__ delta_bias, const float* __restrict__ A_log,
               const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ D,
               const T* __restrict__ z, const float* __restrict__ init, T* __restrict__ out,
               float* __restrict__ fin)
{
    __shared__ float sb[kS6Chunk][N], sc[kS6Chunk][N];
    const int d = blockIdx.x * kS6Threads + threadIdx.x;
    const int b = blockIdx.y;
    const bool live = d < DI;
    float a2[N], h[N];
#pragma unroll
    for (int n = 0; n < N; n++) {
        const float al = live ? fminf(fmaxf(A_log[(int64_t)d * N + n], -10.0f), 5.0f) : 0.0f;
        a2[n] = -expf(al) * 1.4426950408889634f;        // A[d,n] log2(e)
        h[n] = (live && init) ? init[((int64_t)b * DI + d) * N + n] : 0.0f;
    }
    const float bias = live ? delta_bias[d] : 0.0f;
    const float Dd = live ? D[d] : 0.0f;
    for (int t0 = 0; t0 < L; t0 += kS6Chunk) {
        const int Lc = min(kS6Chunk, L - t0);
        __syncthreads();                                 // the previous chunk's B, C are used
        for (int i = threadIdx.x; i < Lc * N; i += kS6Threads) {
            const int r = i / N, n = i % N;
            const int64_t o = ((int64_t)b * L + t0 + r) * N + n;
            sb[r][n] = to_f(Bm[o]);
            sc[r][n] = to_f(Cm[o]);
        }
        __syncthreads();
        if (!live) continue;
        for (int r = 0; r < Lc; r++) {
            const int64_t o = ((int64_t)b * L + t0 + r) * DI + d;
            const float dt = softplus_f(delta[o] + bias);
            const float uv = to_f(u[o]);
            const float du = dt * uv;
            float y = 0.0f;
#pragma unroll
            for (int n = 0; n < N; n++) {
                h[n] = fmaf(ex2(dt * a2[n]), h[n], du * sb[r][n]);
                y = fmaf(sc[r][n], h[n], y);
            }
            y = fmaf(Dd, uv, y);
            out[o] = from_f<T>(z ? y * silu_f(to_f(z[o])) : y);
        }
    }
    if (live && fin) {
#pragma unroll
        for (int n = 0; n < N; n++) fin[((int64_t)b * DI + d) * N + n] = h[n];
    }
}

template <typename T>
static cudaError_t launch_s6_t(const S6Args& s, cudaStream_t st)
{
    const dim3 grid((unsigned)((s.d_inner + kS6Threads - 1) / kS6Threads), (unsigned)s.batch);
#define SSD_S6(NN)                                                                                  \
    s6_scan_kernel<T, NN><<<grid, kS6Threads, 0, st>>>(                                             \
        s.batch, s.seqlen, s.d_inner, (const T*)s.u, s.delta, s.delta_bias, s.A_log, (const T*)s.B, \
        (const T*)s.C, s.D, (const T*)s.z, s.init, (T*)s.out, s.fin)
    switch (s.dstate) {
    case 8: SSD_S6(8); break;
    case 16: SSD_S6(16); break;
    case 32: SSD_S6(32); break;
    default: return cudaErrorInvalidValue;
    }
#undef SSD_S6
    return cudaGetLastError();
}

cudaError_t launch_s6_scan(const S6Args& s, cudaStream_t st)
{
    return s.bf16 ? launch_s6_t<bf16>(s, st) : launch_s6_t<float>(s, st);
}

}  // namespace ssd
