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
// the block's state is one contiguous run, moved through shared memory by 1-D
// bulk copies (the first pieces requested before the conv prologue), updated
// there in place with 8 lanes per row, and the row's C.h sum is reduced over
// its 8 lanes.  d_state other than 32/64/128/256 takes a warp-per-row kernel.
#include "ssd_device.cuh"
#include "ssd_kernels.h"
#include "tc05.cuh"

namespace ssd {

constexpr int kDecodeThreads = 128;
// The bulk kernel moves the block's state through a ring of kDecRing pieces of
// kDecPiece bytes in shared memory (16 KB: nine 128-thread blocks fit per SM,
// as many as the registers allow).
constexpr int kDecPiece = 8192;
constexpr int kDecRing = 2;

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

// 1-D bulk copies (no tensor map): global -> shared completing on an mbarrier,
// and shared -> global in a bulk group.  Addresses 16-byte aligned, sizes
// multiples of 16.
__device__ __forceinline__ void dec_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void dec_bulk_store(void* dst, const void* src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(tc::smem_u32(src)), "r"(bytes)
                 : "memory");
}

// Bulk kernel: N = 32 * NV.  The block's state (hpg * P rows of N fp32, one
// contiguous run) goes through shared memory in pieces of kDecPiece bytes:
// thread 0 requests the first kDecRing pieces before the conv prologue, so
// their DRAM latency overlaps it; every piece is updated in place by the
// block (8 lanes per row, lane l8 owning float4 q at (q * 8 + l8) * 4, so the
// 8 lanes cover 32 consecutive floats per q) and written back by one bulk
// store, and its slot is
// refilled once that store has read it.  Every wait is bounded (wait_ns): on
// timeout the block raises kStatusTimeout, stops updating, lets its copies land
// and exits.  withhold >= 0 (testing): that block never requests its first
// piece, so its first wait runs out.
template <typename T, int NV>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_bulk(Shape s, FwdArgs a, float* __restrict__ ssm, T* __restrict__ hist, int* status,
                 uint64_t wait_ns, int withhold)
{
    extern __shared__ __align__(128) float sm[];
    constexpr int N = 32 * NV;
    constexpr int kRows = kDecPiece / (N * 4);      // state rows per piece
    static_assert(kRows >= 1, "a piece holds at least one state row");
    const int H = s.nheads, P = s.headdim;
    const int hpg = H / s.ngroups;
    const int g = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    float* ring = sm;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kDecRing * kDecPiece / 4);
    volatile int* s_abort = reinterpret_cast<volatile int*>(full + kDecRing);
    DecodeSmem sv(sm + kDecRing * kDecPiece / 4 + 4 * kDecRing, s);   // past the barriers and the flag
    const int nrows = hpg * P;
    const int npieces = (nrows + kRows - 1) / kRows;
    float* base = ssm + ((int64_t)b * H + (int64_t)g * hpg) * P * N;
    auto piece_bytes = [&](int k) { return (uint32_t)(min(kRows, nrows - k * kRows) * N * 4); };
    auto issue_load = [&](int k) {
        uint64_t* bar = &full[k % kDecRing];
        tc::mbar_arrive_expect_tx(bar, piece_bytes(k));
        dec_bulk_load(ring + (k % kDecRing) * (kDecPiece / 4), base + (int64_t)k * kRows * N, piece_bytes(k), bar);
    };
    if (threadIdx.x == 0) {
        *s_abort = 0;
        for (int i = 0; i < kDecRing; i++) tc::mbar_init(&full[i], 1);
        tc::fence_mbar_init();
        // testing hook: block `withhold` never requests its first piece, so its wait runs out
        const bool held = withhold == (int)(blockIdx.y * gridDim.x + blockIdx.x);
        for (int k = held ? 1 : 0; k < min(kDecRing, npieces); k++) issue_load(k);
    }
    // SiLU(z) of the block's rows, so the outputs need no global load
    for (int i = threadIdx.x; i < nrows; i += blockDim.x)
        sv.gz[i] = silu_f(to_f(((const T*)a.z)[(int64_t)b * H * P + (int64_t)g * hpg * P + i]));
    decode_prologue<T>(s, a, hist, sv.ux, sv.ub, sv.uc, sv.dts, sv.dec, sv.bh, sv.ch, g, b);   // ends in a barrier

    const int sub = lane >> 3, l8 = lane & 7;
    float4 Bq[NV], Cq[NV];
    if (!s.bc_norm) {
#pragma unroll
        for (int q = 0; q < NV; q++) {
            Bq[q] = *reinterpret_cast<const float4*>(sv.ub + (q * 8 + l8) * 4);
            Cq[q] = *reinterpret_cast<const float4*>(sv.uc + (q * 8 + l8) * 4);
        }
    }
    int loaded = min(kDecRing, npieces);          // pieces requested so far (thread 0's count)
    int k = 0;
    for (; k < npieces; k++) {
        float* slot = ring + (k % kDecRing) * (kDecPiece / 4);
        // every thread waits on the piece; the block then leaves together if any gave up
        const bool ok = tc::mbar_wait(&full[k % kDecRing], (uint32_t)(k / kDecRing) & 1u, s_abort, status,
                                      kStatusTimeout, wait_ns);
        if (__syncthreads_or(!ok)) break;
        const int r0 = k * kRows, rows = min(kRows, nrows - r0);
        // a warp takes 4 rows per pass (the loop test is the same for its 32 lanes)
        for (int rr = warp * 4 + sub; rr - sub < rows; rr += nw * 4) {
            const bool valid = rr < rows;
            const int r = r0 + (valid ? rr : 0);
            const int hl = r / P;
            const float xdt = sv.dts[hl] * sv.ux[r];
            const float d = sv.dec[hl];
            float* row = slot + (valid ? rr : 0) * N;
            float y = 0.f;
#pragma unroll
            for (int q = 0; q < NV; q++) {
                float4 bv = Bq[q], cv = Cq[q];
                if (s.bc_norm) {
                    bv = *reinterpret_cast<const float4*>(sv.bh + hl * N + (q * 8 + l8) * 4);
                    cv = *reinterpret_cast<const float4*>(sv.ch + hl * N + (q * 8 + l8) * 4);
                }
                float4* hp = reinterpret_cast<float4*>(row + (q * 8 + l8) * 4);
                const float4 hc = *hp;
                float4 hv;
                hv.x = fmaf(d, hc.x, xdt * bv.x);
                hv.y = fmaf(d, hc.y, xdt * bv.y);
                hv.z = fmaf(d, hc.z, xdt * bv.z);
                hv.w = fmaf(d, hc.w, xdt * bv.w);
                y = fmaf(cv.x, hv.x, y);
                y = fmaf(cv.y, hv.y, y);
                y = fmaf(cv.z, hv.z, y);
                y = fmaf(cv.w, hv.w, y);
                if (valid) *hp = hv;
            }
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            y += __shfl_xor_sync(0xffffffffu, y, 4);
            if (valid && l8 == 0) sv.ys[r] = y;
        }
        tc::fence_async_smem();                   // the updated rows, to the bulk store
        __syncthreads();
        if (threadIdx.x == 0) {
            dec_bulk_store(base + (int64_t)r0 * N, slot, piece_bytes(k));
            tc::bulk_commit();
            if (loaded < npieces) {
                tc::bulk_wait_read0();            // the store has read the slot
                issue_load(loaded);
                loaded++;
            }
        }
    }
    if (threadIdx.x == 0) {
        // an aborted block lets every requested piece land before it exits
        for (int j = k; j < loaded; j++)
            tc::mbar_drain(&full[j % kDecRing], (uint32_t)(j / kDecRing) & 1u, status, kStatusTimeout, wait_ns);
        tc::bulk_wait0();
    }
    __syncthreads();
    if (*s_abort) return;
    // the block's outputs, one coalesced row of hpg * P values
    for (int i = threadIdx.x; i < nrows; i += blockDim.x) {
        const int hh = g * hpg + i / P;
        ((T*)a.out)[(int64_t)b * H * P + (int64_t)g * hpg * P + i] =
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
                                   int* status, uint64_t wait_ns, int withhold, cudaStream_t st)
{
    const int hpg = s.nheads / s.ngroups;
    const size_t smem = sizeof(float) * decode_smem_floats(hpg, s.headdim, s.dstate, s.bc_norm);
    const dim3 grid(s.ngroups, s.batch);
    if (s.dstate == 32 || s.dstate == 64 || s.dstate == 128 || s.dstate == 256) {
        // the bulk kernel: the ring, its barriers and the abort flag ahead of the arrays
        void (*kern)(Shape, FwdArgs, float*, T*, int*, uint64_t, int);
        switch (s.dstate) {
        case 32: kern = decode_step_bulk<T, 1>; break;
        case 64: kern = decode_step_bulk<T, 2>; break;
        case 128: kern = decode_step_bulk<T, 4>; break;
        default: kern = decode_step_bulk<T, 8>; break;
        }
        const size_t bsmem = smem + (size_t)kDecRing * kDecPiece + 16 * (size_t)kDecRing;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsmem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kDecodeThreads, bsmem, st>>>(s, a, ssm, (T*)hist, status,
                                                  wait_ns ? wait_ns : tc::kWaitLimitNs, withhold);
        return cudaGetLastError();
    }
    cudaError_t e = cudaFuncSetAttribute(decode_step_any<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_step_any<T><<<grid, kDecodeThreads, smem, st>>>(s, a, ssm, (T*)hist);
    return cudaGetLastError();
}

cudaError_t launch_decode_step(const Shape& s, const FwdArgs& a, float* ssm, void* conv_hist,
                               int* status, uint64_t wait_ns, int withhold, cudaStream_t st)
{
    return s.act_bf16 ? launch_decode_t<bf16>(s, a, ssm, conv_hist, status, wait_ns, withhold, st)
                      : launch_decode_t<float>(s, a, ssm, conv_hist, status, wait_ns, withhold, st);
}

}  // namespace ssd
