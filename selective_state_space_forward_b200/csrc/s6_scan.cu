// s6_scan.cu -- the Mamba-1 selective scan (S6) of the Falcon-Mamba port
// (falcon_mamba.ts header: a Mamba-1 / S6 model; A = -exp(clamp(A_log, -10, 5))
// as selective_scan.ts computes it; dt = softplus(dt + bias)).  Per batch row b
// and channel d, state size N:
//
//   h[n] <- exp(dt_t A[d,n]) h[n] + dt_t u_t B_t[n];   y_t = C_t . h + D[d] u_t
//   out_t = y_t SiLU(z_t)   (no z: y_t)
//
// A is diagonal, so channels never mix.  A block of 64 threads takes 16
// channels of one row (up to 8 blocks per SM, so the blocks of a row spread
// evenly over the SMs); the 4 lanes of a quartet share a channel and each keeps
// N/4 of its states and decay rates (pre-scaled by log2 e) in registers.  The
// row is walked in chunks of 32 tokens:
//   stage   every thread turns its share of the chunk's (token, channel) inputs
//           into {dt, dt u} = {softplus(delta + bias), dt u}, D u and SiLU(z) in
//           shared memory, beside the chunk's B and C rows (shared by every
//           channel); tokens past the row's end get dt = 0, which leaves h as it is;
//   scan    each quartet walks the chunk four tokens at a time from shared
//           memory: the state updates of the four tokens are independent of the
//           C . h sums, and the four partial sums of the quartet's lanes are
//           reduced by a reduce-scatter (three shuffles, each lane finishing one);
//   write   the chunk's outputs leave as coalesced rows of the block's channels.
// The next chunk's raw inputs (u, delta, z, B, C rows) are copied into shared
// memory with cp.async before the scan starts (into registers when the rows are
// not 16-byte aligned), so their memory latency overlaps the scan; the copies
// are issued kind by kind, so each piece's row and column follow from
// compile-time piece counts.  The bound is
// the N exponentials per (token, channel) on the MUFU pipe.
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

constexpr int kS6Threads = 64;
constexpr int kS6Ch = 16;                         // channels per block
constexpr int kS6Lanes = 4;                       // lanes per channel
constexpr int kS6Group = 4;                       // tokens per unrolled scan group
// tokens per chunk: 32 (the next chunk's raw inputs wait in registers)
template <int N> constexpr int s6_chunk() { return 32; }

__device__ __forceinline__ uint64_t s6_p2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void s6_split(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t s6_fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t s6_mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// SiLU for the gate: the hardware tanh form for bf16 outputs, the IEEE form for fp32.
template <typename T> __device__ __forceinline__ float s6_gate(float v) { return silu_t(v); }
template <> __device__ __forceinline__ float s6_gate<float>(float v) { return silu_f(v); }

// softplus(v) = log(1 + e^v) for bf16 paths from the hardware exp2 and log2:
// v above 15 gives v (e^-15 is below fp32's resolution of v); below -5 the
// series e - e^2/2 + e^3/3 (e = e^v < 0.0068, the first dropped term e^4/4 is
// below 2.1e-9 of the result); in between log2(1 + e) ln 2, with 1 + e >= 1.0067
// so its rounding costs at most 2e-5 of the result.  fp32 paths keep softplus_f.
template <typename T> __device__ __forceinline__ float s6_softplus(float v)
{
    const float e = ex2(v * 1.4426950408889634f);
    if (v > 15.0f) return v;
    if (v < -5.0f) return e * (1.0f - e * (0.5f - e * 0.33333334f));
    float l;
    asm("lg2.approx.f32 %0, %1;" : "=f"(l) : "f"(1.0f + e));
    return l * 0.6931471805599453f;
}
template <> __device__ __forceinline__ float s6_softplus<float>(float v) { return softplus_f(v); }

// 16-byte asynchronous copy global -> shared (cp.async); bytes past src_bytes
// are zero-filled, and with src_bytes = 0 nothing is read.
__device__ __forceinline__ void s6_cp16(void* dst, const void* src, int src_bytes)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void s6_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void s6_cp_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename T, int N, bool ASYNC>
__global__ void __launch_bounds__(kS6Threads, 8)
s6_scan_kernel(int batch, int L, int DI, const T* __restrict__ u, const float* __restrict__ delta,
               const float* __restrict__ delta_bias, const float* __restrict__ A_log,
               const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ D,
               const T* __restrict__ z, const float* __restrict__ init, T* __restrict__ out,
               float* __restrict__ fin, int bc_vec)
{
    constexpr int SPL = N / kS6Lanes;             // states per lane
    static_assert(SPL % 2 == 0, "d_state 8, 16 or 32");
    constexpr int kS6T = s6_chunk<N>();
    constexpr int kS6PerThread = kS6T * kS6Ch / kS6Threads;   // staged (token, channel) pairs
    __shared__ __align__(16) float sb[kS6T][N], sc[kS6T][N];
    __shared__ __align__(8) float2 s_dd[kS6T][kS6Ch];          // {dt, dt u}
    __shared__ float s_dx[kS6T][kS6Ch], s_g[kS6T][kS6Ch];
    __shared__ float s_y[kS6T][kS6Ch];     // row r's channel c at column (c + kS6Ch/4 (r & 3)) mod kS6Ch
    // ASYNC: the next chunk's raw inputs, copied in while the current chunk is scanned
    constexpr int kRawT = ASYNC ? kS6T : 1;
    __shared__ __align__(16) T raw_u[kRawT][kS6Ch], raw_z[kRawT][kS6Ch], raw_b[kRawT][N], raw_c[kRawT][N];
    __shared__ __align__(16) float raw_d[kRawT][kS6Ch];
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

    uint64_t a2[SPL / 2], h[SPL / 2];             // state pairs (j, j+1)
#pragma unroll
    for (int j = 0; j < SPL; j += 2) {
        float av[2], hv[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int n = q * SPL + j + e;
            const float al = live_q ? fminf(fmaxf(A_log[(int64_t)dq * N + n], -10.0f), 5.0f) : 0.0f;
            av[e] = -expf(al) * 1.4426950408889634f;    // A[d,n] log2(e)
            hv[e] = (live_q && init) ? init[((int64_t)b * DI + dq) * N + n] : 0.0f;
        }
        a2[j / 2] = s6_p2(av[0], av[1]);
        h[j / 2] = s6_p2(hv[0], hv[1]);
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
    // ASYNC: copy chunk t0's u, delta, z rows (the block's channels) and B, C rows
    // into the raw buffers in 16-byte pieces; rows past L and channels past DI are
    // zero-filled (the host takes this path when every piece is 16-byte aligned
    // and whole: DI a multiple of 16 / sizeof(T))
    auto fetch_async = [&](int t0) {
        constexpr int kPu = kS6Ch * (int)sizeof(T) / 16;        // 16-byte pieces per token row of u, z
        constexpr int kPd = kS6Ch * 4 / 16;                     // of delta
        constexpr int kPb = N * (int)sizeof(T) / 16;            // of B, C
        constexpr int kEu = 16 / (int)sizeof(T);                // elements per piece of u, z, B, C
        for (int i = tid; i < kS6T * kPu; i += kS6Threads) {
            const int r = i / kPu, piece = i % kPu, t = t0 + r, c0 = d0 + piece * kEu;
            const bool ok = t < L && c0 < DI;
            const int64_t o = ok ? ((int64_t)b * L + t) * DI + c0 : 0;
            s6_cp16(&raw_u[r][piece * kEu], u + o, ok ? 16 : 0);
            s6_cp16(&raw_z[r][piece * kEu], (z ? z : u) + o, ok && z ? 16 : 0);
        }
        for (int i = tid; i < kS6T * kPd; i += kS6Threads) {
            const int r = i / kPd, piece = i % kPd, t = t0 + r, c0 = d0 + piece * 4;
            const bool ok = t < L && c0 < DI;
            const int64_t o = ok ? ((int64_t)b * L + t) * DI + c0 : 0;
            s6_cp16(&raw_d[r][piece * 4], delta + o, ok ? 16 : 0);
        }
        for (int i = tid; i < kS6T * kPb; i += kS6Threads) {
            const int r = i / kPb, piece = i % kPb, t = t0 + r;
            const bool ok = t < L;
            const int64_t o = ok ? ((int64_t)b * L + t) * N + piece * kEu : 0;
            s6_cp16(&raw_b[r][piece * kEu], Bm + o, ok ? 16 : 0);
            s6_cp16(&raw_c[r][piece * kEu], Cm + o, ok ? 16 : 0);
        }
        s6_cp_commit();
    };
    if (ASYNC) fetch_async(0);
    else fetch(0);
    for (int t0 = 0; t0 < L; t0 += kS6T) {
        const int Lc = min(kS6T, L - t0);
        if (ASYNC) s6_cp_wait();             // this chunk's raw inputs have landed
        __syncthreads();                     // ... for every thread; the previous chunk's shared data is used
        if (ASYNC) {
            for (int i = tid; i < kS6T * N; i += kS6Threads) {
                const int r = i / N, n = i % N;
                sb[r][n] = to_f(raw_b[r][n]);
                sc[r][n] = to_f(raw_c[r][n]);
            }
#pragma unroll
            for (int k = 0; k < kS6PerThread; k++) {
                const int r = ts + k * (kS6Threads / kS6Ch);
                ru[k] = to_f(raw_u[r][cs]);
                rd[k] = raw_d[r][cs];
                rz[k] = to_f(raw_z[r][cs]);
            }
        } else if (bc_vec) {
            // eight elements per load (rows start 16-byte aligned)
            for (int i = tid; i < kS6T * N / 8; i += kS6Threads) {
                const int r = (i * 8) / N, n0 = (i * 8) % N;
                float vb[8], vc[8];
                if (r < Lc) {
                    const int64_t o = ((int64_t)b * L + t0 + r) * N + n0;
                    load8(Bm + o, vb);
                    load8(Cm + o, vc);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; e++) vb[e] = vc[e] = 0.0f;
                }
                *reinterpret_cast<float4*>(&sb[r][n0]) = make_float4(vb[0], vb[1], vb[2], vb[3]);
                *reinterpret_cast<float4*>(&sb[r][n0 + 4]) = make_float4(vb[4], vb[5], vb[6], vb[7]);
                *reinterpret_cast<float4*>(&sc[r][n0]) = make_float4(vc[0], vc[1], vc[2], vc[3]);
                *reinterpret_cast<float4*>(&sc[r][n0 + 4]) = make_float4(vc[4], vc[5], vc[6], vc[7]);
            }
        } else {
            for (int i = tid; i < kS6T * N; i += kS6Threads) {
                const int r = i / N, n = i % N;
                const int64_t o = ((int64_t)b * L + t0 + r) * N + n;
                sb[r][n] = r < Lc ? to_f(Bm[o]) : 0.0f;
                sc[r][n] = r < Lc ? to_f(Cm[o]) : 0.0f;
            }
        }
#pragma unroll
        for (int k = 0; k < kS6PerThread; k++) {
            const int r = ts + k * (kS6Threads / kS6Ch);
            const bool ok = r < Lc;                 // past the row's end: dt = 0, h unchanged
            const float dt = ok ? s6_softplus<T>(rd[k] + bias) : 0.0f;
            s_dd[r][cs] = make_float2(dt, dt * ru[k]);
            s_dx[r][cs] = Dd * ru[k];
            s_g[r][cs] = z ? s6_gate<T>(rz[k]) : 1.0f;
        }
        __syncthreads();
        if (t0 + kS6T < L) {                   // in flight during the scan
            if (ASYNC) fetch_async(t0 + kS6T);
            else fetch(t0 + kS6T);
        }
        const int b0 = q & 1, b1 = (q >> 1) & 1;
        for (int r0 = 0; r0 < Lc; r0 += kS6Group) {
            float yv[kS6Group];
#pragma unroll
            for (int k = 0; k < kS6Group; k++) {
                const int r = r0 + k;
                const float2 dd = s_dd[r][cq];
                const uint64_t dtp = s6_p2(dd.x, dd.x), dup = s6_p2(dd.y, dd.y);
                uint64_t bv[SPL / 2], cv[SPL / 2];
                if constexpr (SPL % 4 == 0) {
#pragma unroll
                    for (int j = 0; j < SPL; j += 4) {
                        const float4 b4 = *reinterpret_cast<const float4*>(&sb[r][q * SPL + j]);
                        const float4 c4 = *reinterpret_cast<const float4*>(&sc[r][q * SPL + j]);
                        bv[j / 2] = s6_p2(b4.x, b4.y); bv[j / 2 + 1] = s6_p2(b4.z, b4.w);
                        cv[j / 2] = s6_p2(c4.x, c4.y); cv[j / 2 + 1] = s6_p2(c4.z, c4.w);
                    }
                } else {
                    const float2 b2 = *reinterpret_cast<const float2*>(&sb[r][q * SPL]);
                    const float2 c2 = *reinterpret_cast<const float2*>(&sc[r][q * SPL]);
                    bv[0] = s6_p2(b2.x, b2.y);
                    cv[0] = s6_p2(c2.x, c2.y);
                }
                uint64_t y2 = 0;                   // two fp32 zeros
#pragma unroll
                for (int j = 0; j < SPL / 2; j++) {
                    float x0, x1;
                    s6_split(s6_mul2(dtp, a2[j]), x0, x1);
                    h[j] = s6_fma2(s6_p2(ex2(x0), ex2(x1)), h[j], s6_mul2(dup, bv[j]));
                    y2 = s6_fma2(cv[j], h[j], y2);
                }
                float ylo, yhi;
                s6_split(y2, ylo, yhi);
                yv[k] = ylo + yhi;
            }
            // reduce-scatter over the quartet: lane (b0, b1) finishes token r0 + 2 b0 + b1
            float z1[2];
#pragma unroll
            for (int i = 0; i < 2; i++) {
                const float send = b0 ? yv[i] : yv[2 + i];
                const float keep = b0 ? yv[2 + i] : yv[i];
                z1[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            }
            const float send = b1 ? z1[0] : z1[1];
            const float keep = b1 ? z1[1] : z1[0];
            const float z2 = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            const int rb = r0 + 2 * b0 + b1;
            // the four lanes of a quartet store to four different banks
            s_y[rb][(cq + (kS6Ch / 4) * (rb & 3)) % kS6Ch] = z2;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kS6PerThread; k++) {
            const int r = ts + k * (kS6Threads / kS6Ch);
            if (r < Lc && live_s) {
                const int64_t o = ((int64_t)b * L + t0 + r) * DI + dsr;
                out[o] = from_f<T>((s_y[r][(cs + (kS6Ch / 4) * (r & 3)) % kS6Ch] + s_dx[r][cs]) * s_g[r][cs]);
            }
        }
    }
    if (live_q && fin) {
#pragma unroll
        for (int j = 0; j < SPL; j += 2) {
            float h0, h1;
            s6_split(h[j / 2], h0, h1);
            fin[((int64_t)b * DI + dq) * N + q * SPL + j] = h0;
            fin[((int64_t)b * DI + dq) * N + q * SPL + j + 1] = h1;
        }
    }
}

template <typename T>
static cudaError_t launch_s6_t(const S6Args& s, cudaStream_t st)
{
    const dim3 grid((unsigned)((s.d_inner + kS6Ch - 1) / kS6Ch), (unsigned)s.batch);
    // B and C rows are read eight elements at a time when both start 16-byte aligned
    const uintptr_t bc = reinterpret_cast<uintptr_t>(s.B) | reinterpret_cast<uintptr_t>(s.C);
    const int vec = (bc & 15u) == 0;
    // the asynchronous copies need every 16-byte piece of u, z, delta, B and C
    // aligned and whole: aligned bases and d_inner a multiple of 16 / sizeof(T)
    const uintptr_t all = bc | reinterpret_cast<uintptr_t>(s.u) | reinterpret_cast<uintptr_t>(s.z) |
                          reinterpret_cast<uintptr_t>(s.delta);
    const bool async = (all & 15u) == 0 && s.d_inner % (16 / (int)sizeof(T)) == 0 && s.d_inner % 4 == 0;
#define SSD_S6(NN)                                                                                    \
    (async ? s6_scan_kernel<T, NN, true><<<grid, kS6Threads, 0, st>>>(                                \
                 s.batch, s.seqlen, s.d_inner, (const T*)s.u, s.delta, s.delta_bias, s.A_log,         \
                 (const T*)s.B, (const T*)s.C, s.D, (const T*)s.z, s.init, (T*)s.out, s.fin, vec)     \
           : s6_scan_kernel<T, NN, false><<<grid, kS6Threads, 0, st>>>(                               \
                 s.batch, s.seqlen, s.d_inner, (const T*)s.u, s.delta, s.delta_bias, s.A_log,         \
                 (const T*)s.B, (const T*)s.C, s.D, (const T*)s.z, s.init, (T*)s.out, s.fin, vec))
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
