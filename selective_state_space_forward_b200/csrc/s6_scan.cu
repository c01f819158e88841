// s6_scan.cu -- the Mamba-1 selective scan (S6) of the Falcon-Mamba port
// (falcon_mamba.ts header: a Mamba-1 / S6 model; A = -exp(clamp(A_log, -10, 5))
// as selective_scan.ts computes it; dt = softplus(dt + bias)).  Per batch row b
// and channel d, state size N:
//
//   h[n] <- exp(dt_t A[d,n]) h[n] + dt_t u_t B_t[n];   y_t = C_t . h + D[d] u_t
//   out_t = y_t SiLU(z_t)   (no z: y_t)
//
// A is diagonal, so channels never mix.  A block of 128 threads takes 32
// channels of one row; the 4 lanes of a quartet share a channel and each keeps
// N/4 of its states and decay rates (pre-scaled by log2 e) in registers.  The
// row is walked in chunks of 64 tokens (32 at d_state 32):
//   stage   every thread turns its share of the chunk's (token, channel) inputs
//           into dt = softplus(delta + bias), dt u, D u and SiLU(z) in shared
//           memory, beside the chunk's B and C (shared by every channel);
//   scan    each quartet walks the chunk's tokens reading shared memory only:
//           its lanes update their states and sum C . h over two xor-shuffles;
//   write   the chunk's outputs leave as coalesced rows of the block's channels.
// The next chunk's raw inputs are loaded into registers before the scan starts,
// so their memory latency overlaps the scan.  The bound is the N exponentials
// per (token, channel) on the MUFU pipe.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kS6Threads = 128;
constexpr int kS6Ch = 32;                         // channels per block
constexpr int kS6Lanes = 4;                       // lanes per channel
// tokens per chunk: 64, or 32 at d_state 32 (static shared memory stays under 48 KB)
template <int N> constexpr int s6_chunk() { return N == 32 ? 32 : 64; }

template <typename T, int N>
__global__ void __launch_bounds__(kS6Threads)
s6_scan_kernel(int batch, int L, int DI, const T* __restrict__ u, const float* __restrict__ delta,
               const float* __restrict__ delta_bias, const float* __restrict__ A_log,
               const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ D,
               const T* __restrict__ z, const float* __restrict__ init, T* __restrict__ out,
               float* __restrict__ fin)
{
    constexpr int SPL = N / kS6Lanes;             // states per lane
    constexpr int kS6T = s6_chunk<N>();
    constexpr int kS6PerThread = kS6T * kS6Ch / kS6Threads;   // staged (token, channel) pairs
    __shared__ __align__(16) float sb[kS6T][N], sc[kS6T][N];
    __shared__ float s_dt[kS6T][kS6Ch], s_du[kS6T][kS6Ch], s_dx[kS6T][kS6Ch], s_g[kS6T][kS6Ch];
    __shared__ float s_y[kS6T][kS6Ch];
    const int tid = threadIdx.x;
    const int d0 = blockIdx.x * kS6Ch;
    const int b = blockIdx.y;
    // scan role: channel cq of the block, states q*SPL .. q*SPL+SPL-1
    const int cq = tid / kS6Lanes, q = tid % kS6Lanes;
    const int dq = d0 + cq;
    const bool live_q = dq < DI;
    // stage role: channel cs, tokens ts, ts + 4, ... (a warp covers one token row)
    const int cs = tid % kS6Ch, ts = tid / kS6Ch;
    const int dsr = d0 + cs;
    const bool live_s = dsr < DI;

    float a2[SPL], h[SPL];
#pragma unroll
    for (int j = 0; j < SPL; j++) {
        const int n = q * SPL + j;
        const float al = live_q ? fminf(fmaxf(A_log[(int64_t)dq * N + n], -10.0f), 5.0f) : 0.0f;
        a2[j] = -expf(al) * 1.4426950408889634f;        // A[d,n] log2(e)
        h[j] = (live_q && init) ? init[((int64_t)b * DI + dq) * N + n] : 0.0f;
    }
    const float bias = live_s ? delta_bias[dsr] : 0.0f;
    const float Dd = live_s ? D[dsr] : 0.0f;

    // raw inputs of one chunk for the stage role, held in registers
    float ru[kS6PerThread], rd[kS6PerThread], rz[kS6PerThread];
    auto fetch = [&](int t0) {
#pragma unroll
        for (int k = 0; k < kS6PerThread; k++) {
            const int t = t0 + ts + k * (kS6Threads / kS6Ch);
            const bool ok = live_s && t < L;
            const int64_t o = ((int64_t)b * L + t) * DI + dsr;
            ru[k] = ok ? to_f(u[o]) : 0.0f;
            rd[k] = ok ? delta[o] : 0.0f;
            rz[k] = (ok && z) ? to_f(z[o]) : 0.0f;
        }
    };
    fetch(0);
    for (int t0 = 0; t0 < L; t0 += kS6T) {
        const int Lc = min(kS6T, L - t0);
        __syncthreads();                     // the previous chunk's shared data is used
        for (int i = tid; i < Lc * N; i += kS6Threads) {
            const int r = i / N, n = i % N;
            const int64_t o = ((int64_t)b * L + t0 + r) * N + n;
            sb[r][n] = to_f(Bm[o]);
            sc[r][n] = to_f(Cm[o]);
        }
#pragma unroll
        for (int k = 0; k < kS6PerThread; k++) {
            const int r = ts + k * (kS6Threads / kS6Ch);
            const float dt = softplus_f(rd[k] + bias);
            s_dt[r][cs] = dt;
            s_du[r][cs] = dt * ru[k];
            s_dx[r][cs] = Dd * ru[k];
            s_g[r][cs] = z ? silu_f(rz[k]) : 1.0f;
        }
        __syncthreads();
        if (t0 + kS6T < L) fetch(t0 + kS6T);   // in flight during the scan
        for (int r = 0; r < Lc; r++) {
            const float dt = s_dt[r][cq], du = s_du[r][cq];
            float bv[SPL], cv[SPL];
            if constexpr (SPL % 4 == 0) {
#pragma unroll
                for (int j = 0; j < SPL; j += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(&sb[r][q * SPL + j]);
                    const float4 c4 = *reinterpret_cast<const float4*>(&sc[r][q * SPL + j]);
                    bv[j] = b4.x; bv[j + 1] = b4.y; bv[j + 2] = b4.z; bv[j + 3] = b4.w;
                    cv[j] = c4.x; cv[j + 1] = c4.y; cv[j + 2] = c4.z; cv[j + 3] = c4.w;
                }
            } else {
                static_assert(SPL == 2, "d_state 8, 16 or 32");
                const float2 b2 = *reinterpret_cast<const float2*>(&sb[r][q * SPL]);
                const float2 c2 = *reinterpret_cast<const float2*>(&sc[r][q * SPL]);
                bv[0] = b2.x; bv[1] = b2.y;
                cv[0] = c2.x; cv[1] = c2.y;
            }
            float y = 0.0f;
#pragma unroll
            for (int j = 0; j < SPL; j++) {
                h[j] = fmaf(ex2(dt * a2[j]), h[j], du * bv[j]);
                y = fmaf(cv[j], h[j], y);
            }
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            if (q == 0) s_y[r][cq] = y;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kS6PerThread; k++) {
            const int r = ts + k * (kS6Threads / kS6Ch);
            if (r < Lc && live_s) {
                const int64_t o = ((int64_t)b * L + t0 + r) * DI + dsr;
                out[o] = from_f<T>((s_y[r][cs] + s_dx[r][cs]) * s_g[r][cs]);
            }
        }
    }
    if (live_q && fin) {
#pragma unroll
        for (int j = 0; j < SPL; j++) fin[((int64_t)b * DI + dq) * N + q * SPL + j] = h[j];
    }
}

template <typename T>
static cudaError_t launch_s6_t(const S6Args& s, cudaStream_t st)
{
    const dim3 grid((unsigned)((s.d_inner + kS6Ch - 1) / kS6Ch), (unsigned)s.batch);
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
