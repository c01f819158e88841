// chunk_fused.cu -- KF: the fused chunk sweep of the SSD scan on sm_100a.
//
// One CTA owns one (batch row, head) and walks its 64-token chunks in order
// (chunk 64: mojolearn Mamba3Block), so the running state never leaves the
// SM.  Per chunk c (tokens t0 .. t0+63), with acs the segmented cumsum of
// dt*a written by K2 and seg_t the number of document boundaries at t0 .. t:
//
//   conv      u_t = SiLU(conv(x)) for the head's 64 channels (K1's arithmetic;
//             B and C of the group come pre-convolved from K1, or raw)
//   operands  Xd[s] = dt_s u_s              (intra-chunk right operand)
//             Xs[s] = exp(acs_last - acs_s) dt_s u_s  [seg_s = seg_last]
//   CB        S = C B^T                      tcgen05, 64 x 64 x N
//   mask      M[t,s] = S[t,s] exp(acs_t - acs_s)  [s <= t, seg_s = seg_t]
//   Ydiag     M Xd                           tcgen05, 64 x 64 x 64
//   Yoff      C h_c^T                        tcgen05, 64 x 64 x N (bf16 copy of h_c)
//   state     h_{c+1} = k_c h_c + B^T Xs     tcgen05, accumulates in TMEM
//             (k_c = exp(acs_last), or 0 when the chunk holds a boundary)
//   epilogue  out_t = (Ydiag_t + [seg_t = 0] exp(acs_t) Yoff_t + D u_t) SiLU(z_t)
//
// The chunk-state contraction accumulates onto k_c h_c inside the tensor
// memory, so the fp32 state is carried on chip from the initial state to the
// final one; only a bf16 copy of it is staged in shared memory as the Yoff
// operand.  The gate, the D skip and the output cast are fused in the
// epilogue (spec kernel list items 3-5).
//
// Roles (192 threads): warps 0-3 compute (conv, state hand-off, masks,
// epilogue; each warp reaches TMEM lanes 32w .. 32w+31), warp 4 produces (TMA
// tile loads into a 2-stage ring, dt/acs/boundary flags), warp 5 issues the
// MMAs from one thread.  Every wait is bounded: after 1 s a waiter raises the
// CTA's abort flag and the device status word, and all roles drain and exit.
//
// Tile layouts (see tc05.cuh): x, z, B, C, out tiles are [64 tokens][64
// channels] bf16 with the 128-byte swizzle, as TMA writes them; N = 128
// operands are two such tiles side by side.  M=64 accumulators put row r in
// TMEM lane 32*(r/16) + r%16; M=128 ones put row r in lane r.
#include <cudaTypedefs.h>

#include "ssd_device.cuh"
#include "ssd_kernels.h"
#include "tc05.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 192;
constexpr int kComputeThreads = 128;
constexpr int kTile = 64 * 128;        // one [64][64] bf16 tile
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColCB = 0, kColY = 64, kColYO = 128, kColST = 192;

struct FusedParams {
    int batch, seqlen, nheads, ngroups, conv;
    const float* dt;          // (B, H, L) from K2
    const float* acs;         // (B, H, L) segmented cumsum from K2
    const int32_t* seq;       // (B, L) or null
    const float* D;
    const bf16* conv_w;       // (conv_dim, 4) or null
    const bf16* conv_b;
    const bf16* init_conv;    // (B, 3, conv_dim) or null
    const float* init_ssm;    // (B, H, 64, N) or null
    float* final_ssm;         // or null
    int* status;
};

template <int NS>
struct Layout {
    static constexpr int kBC = (NS / 64) * kTile;
    static constexpr int kStage = 2 * kTile + 2 * kBC;        // x, z, B, C
    static constexpr int kRing = 2 * kStage;
    static constexpr int kMop = kRing;                        // mask operand / out tile
    static constexpr int kXd = kMop + kTile;
    static constexpr int kXs = kXd + kTile;
    static constexpr int kXb = kXs + kTile;
    static constexpr int kHt = kXb + kTile;                   // h^T, NS rows x 128 B
    static constexpr int kSmall = kHt + NS * 128;
    // small region
    static constexpr int kDt = kSmall;                        // [2][64] f32
    static constexpr int kAcs = kDt + 2 * 64 * 4;             // [2][64] f32
    static constexpr int kBd = kAcs + 2 * 64 * 4;             // [2][4] u32: mask lo, mask hi, pre, pad
    static constexpr int kHalo = kBd + 2 * 16;                // [2][3][64] bf16
    static constexpr int kBar = kHalo + 2 * 3 * 64 * 2;       // 7 mbarriers
    static constexpr int kMisc = kBar + 8 * 8;                // tmem base, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;              // slack for 1024-byte alignment
};

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Compute-warp barrier that also returns the OR of v over the 128 threads, so
// every thread takes the same branch afterwards.
__device__ __forceinline__ int bar_compute_or(int v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v)
        : "memory");
    return (int)r;
}

__device__ __forceinline__ uint32_t mask_le(int i) { return i >= 31 ? 0xffffffffu : ((2u << i) - 1u); }

// Number of document boundaries at chunk positions 0 .. t.
__device__ __forceinline__ int seg_of(uint32_t m0, uint32_t m1, int t)
{
    return t < 32 ? __popc(m0 & mask_le(t)) : __popc(m0) + __popc(m1 & mask_le(t - 32));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float fast_silu(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

template <int NS, bool CONV>
__global__ void __launch_bounds__(kThreads, 1)
ssd_chunk_fused(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                const __grid_constant__ CUtensorMap tm_out, FusedParams p)
{
    using LY = Layout<NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* s_dt = (float*)(sm + LY::kDt);
    float* s_acs = (float*)(sm + LY::kAcs);
    uint32_t* s_bd = (uint32_t*)(sm + LY::kBd);
    bf16* s_halo = (bf16*)(sm + LY::kHalo);
    uint64_t* bar = (uint64_t*)(sm + LY::kBar);
    uint64_t* full = bar;           // [2]
    uint64_t* empty = bar + 2;      // [2]
    uint64_t* cb_done = bar + 4;
    uint64_t* ops_ready = bar + 5;
    uint64_t* mma_done = bar + 6;
    uint32_t* s_tmem = (uint32_t*)(sm + LY::kMisc);
    volatile int* s_abort = (volatile int*)(sm + LY::kMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.nheads, L = p.seqlen;
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const int g = h / (H / p.ngroups);
    const int nc = (L + 63) / 64;
    const int64_t bh = (int64_t)b * H + h;

    if (tid == 0) {
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&full[i], 33);     // producer: expect_tx arrive + 32 lane arrivals
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(cb_done, 1);
        tc::mbar_init(ops_ready, kComputeThreads);
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(&bar[7], 1);           // teardown drain of the MMA pipe
        *s_abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(s_tmem, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        tc::tma_prefetch_desc(&tm_x);
        tc::tma_prefetch_desc(&tm_z);
        tc::tma_prefetch_desc(&tm_b);
        tc::tma_prefetch_desc(&tm_c);
        tc::tma_prefetch_desc(&tm_out);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        const int32_t* seq_row = p.seq ? p.seq + (int64_t)b * L : nullptr;
        const float* dt_row = p.dt + bh * L;
        const float* acs_row = p.acs + bh * L;
        const uint32_t tx = (uint32_t)(2 * kTile + 2 * LY::kBC);
        int issued = 0;
        for (int c = 0; c < nc; c++) {
            const int s = c & 1;
            if (c >= 2 && !tc::mbar_wait(&empty[s], ((c >> 1) & 1) ^ 1, s_abort, p.status, kStatusTimeout))
                break;
            const int t0 = c * 64;
            uint8_t* st = sm + s * LY::kStage;
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&full[s], tx);
                tc::tma_load_3d(st, &tm_x, &full[s], h * 64, t0, b);
                tc::tma_load_3d(st + kTile, &tm_z, &full[s], h * 64, t0, b);
#pragma unroll
                for (int j = 0; j < NS / 64; j++) {
                    const int bx = CONV ? g * NS + 64 * j : g * NS + 64 * j;
                    const int cx = CONV ? p.ngroups * NS + g * NS + 64 * j : g * NS + 64 * j;
                    tc::tma_load_3d(st + 2 * kTile + j * kTile, &tm_b, &full[s], bx, t0, b);
                    tc::tma_load_3d(st + 2 * kTile + LY::kBC + j * kTile, &tm_c, &full[s], cx, t0, b);
                }
            }
            float* dts = s_dt + s * 64;
            float* acv = s_acs + s * 64;
            int bdv[2];
#pragma unroll
            for (int half = 0; half < 2; half++) {
                const int t = t0 + half * 32 + lane;
                const bool ok = t < L;
                dts[half * 32 + lane] = ok ? dt_row[t] : 0.0f;
                acv[half * 32 + lane] = ok ? acs_row[t] : 0.0f;
                bdv[half] = ok ? is_boundary(seq_row, t) : 0;
            }
            const uint32_t m0 = __ballot_sync(0xffffffffu, bdv[0]);
            const uint32_t m1 = __ballot_sync(0xffffffffu, bdv[1]);
            if (lane == 0) {
                uint32_t pre = 0;
                if (t0 - 2 >= 1 && is_boundary(seq_row, t0 - 2)) pre |= 1u;
                if (t0 - 1 >= 1 && is_boundary(seq_row, t0 - 1)) pre |= 2u;
                s_bd[s * 4 + 0] = m0;
                s_bd[s * 4 + 1] = m1;
                s_bd[s * 4 + 2] = pre;
            }
            __syncwarp();
            tc::mbar_arrive(&full[s]);
            issued = c + 1;
        }
        // an aborting CTA lets its last loads land before the shared memory is released
        for (int k = max(0, issued - 2); k < issued; k++)
            tc::mbar_drain(&full[k & 1], (k >> 1) & 1, p.status, kStatusTimeout);
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t id_cb = tc::idesc_bf16(64, 64, false, false);
            const uint32_t id_yo = tc::idesc_bf16(64, 64, false, true);
            const uint32_t id_st = tc::idesc_bf16(NS, 64, true, false);
            const uint32_t a_mop = tc::smem_u32(sm + LY::kMop);
            const uint32_t a_xd = tc::smem_u32(sm + LY::kXd);
            const uint32_t a_xs = tc::smem_u32(sm + LY::kXs);
            const uint32_t a_ht = tc::smem_u32(sm + LY::kHt);
            for (int c = 0; c < nc; c++) {
                const int s = c & 1;
                if (!tc::mbar_wait(&full[s], (c >> 1) & 1, s_abort, p.status, kStatusTimeout)) break;
                tc::tc_fence_after();
                const uint32_t a_b = tc::smem_u32(sm + s * LY::kStage + 2 * kTile);
                const uint32_t a_c = a_b + LY::kBC;
                // CB = C B^T: both K-major over n
#pragma unroll
                for (int kk = 0; kk < NS / 16; kk++) {
                    const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                    tc::mma_bf16(tmem + kColCB, tc::sdesc_sw128(a_c + off, 16, 1024),
                                 tc::sdesc_sw128(a_b + off, 16, 1024), id_cb, kk > 0);
                }
                tc::mma_commit(cb_done);
                if (!tc::mbar_wait(ops_ready, c & 1, s_abort, p.status, kStatusTimeout)) break;
                tc::tc_fence_after();
                // Ydiag = M Xd (K = s)
#pragma unroll
                for (int kk = 0; kk < 4; kk++)
                    tc::mma_bf16(tmem + kColY, tc::sdesc_sw128(a_mop + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(a_xd + kk * 32, 16, 1024), id_cb, kk > 0);
                // Yoff = C h^T (K = n; h^T is MN-major: rows n, 64 p per row)
#pragma unroll
                for (int kk = 0; kk < NS / 16; kk++) {
                    const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                    tc::mma_bf16(tmem + kColYO, tc::sdesc_sw128(a_c + off, 16, 1024),
                                 tc::sdesc_sw128(a_ht + kk * 2048, 8192, 1024), id_yo, kk > 0);
                }
                // state^T[n][p] += B^T Xs (A = B tile as MN-major over n, K = s)
#pragma unroll
                for (int kk = 0; kk < 4; kk++)
                    tc::mma_bf16(tmem + kColST, tc::sdesc_sw128(a_b + kk * 2048, kTile, 1024),
                                 tc::sdesc_sw128(a_xs + kk * 32, 16, 1024), id_st, 1);
                tc::mma_commit(mma_done);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ compute warps 0-3
        const int HP = H * 64;
        const int cdim = HP + 2 * p.ngroups * NS;
        const int pch = tid & 63;            // conv channel
        const int tgb = tid >> 6;            // token-group parity for the conv
        float wk[4] = {0.f, 0.f, 0.f, 1.f}, cbias = 0.f;
        if (CONV) {
            const int ch = h * 64 + pch;
#pragma unroll
            for (int k = 0; k < 4; k++) wk[k] = __bfloat162float(p.conv_w[(int64_t)ch * 4 + k]);
            cbias = __bfloat162float(p.conv_b[ch]);
            // halo for chunk 0: the caller's conv history of this channel (zeros when none)
            if (tid < 64) {
#pragma unroll
                for (int j = 0; j < 3; j++)
                    s_halo[j * 64 + pch] = p.init_conv
                        ? p.init_conv[((int64_t)b * 3 + j) * cdim + h * 64 + pch]
                        : __float2bfloat16(0.0f);
            }
        }
        const float Dh = p.D[h];
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        // M=64 accumulator mapping: row r16 = 16*warp + (lane & 15); this thread's
        // 32 columns start at c16 (0 or 32)
        const int r16 = 16 * warp + (lane & 15);
        const int c16 = lane < 16 ? 0 : 32;

        // ---- initial state into TMEM (state^T: rows n, columns p)
        {
            const float* s0 = p.init_ssm ? p.init_ssm + bh * 64 * NS : nullptr;
            if (NS == 128) {
                const int n = 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint32_t r[16];
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        r[j] = __float_as_uint(s0 ? s0[(int64_t)(q * 16 + j) * NS + n] : 0.0f);
                    tc::tmem_st16(tmem + lane_base + kColST + q * 16, r);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    uint32_t r[16];
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        r[j] = __float_as_uint(s0 ? s0[(int64_t)(c16 + q * 16 + j) * NS + r16] : 0.0f);
                    tc::tmem_st16_x2_32(tmem + lane_base + kColST + q * 16, r);
                }
            }
            tc::tmem_wait_st();
        }
        bar_compute();

        for (int c = 0; c < nc; c++) {
            const int s = c & 1;
            const int t0 = c * 64;
            const int Lc = min(64, L - t0);
            // On abort the waits return at once; every thread still runs the same
            // sequence of compute barriers and leaves at the end of the iteration.
            tc::mbar_wait(&full[s], (c >> 1) & 1, s_abort, p.status, kStatusTimeout);
            const uint8_t* st = sm + s * LY::kStage;
            const float* dts = s_dt + s * 64;
            const float* acv = s_acs + s * 64;
            const uint32_t m0 = s_bd[s * 4 + 0], m1 = s_bd[s * 4 + 1], pre = s_bd[s * 4 + 2];
            const int seg_last = seg_of(m0, m1, Lc - 1);
            const float acs_last = acv[Lc - 1];
            const bool reset = (m0 | m1) != 0;

            // ---- (A) conv and the operand tiles: channel pch, tokens 8*tg .. 8*tg+7
            const bf16* halo_in = s_halo + (c & 1) * 192;
            bf16* halo_out = s_halo + ((c + 1) & 1) * 192;
#pragma unroll 1
            for (int i = 0; i < 4; i++) {
                const int tg = tgb + 2 * i;
                const int r0 = tg * 8;
                float raw[11];
#pragma unroll
                for (int q = 0; q < 11; q++) {
                    const int row = r0 - 3 + q;
                    if (row >= 0)
                        raw[q] = __bfloat162float(*(const bf16*)(st + tc::sw128_offset(row, pch)));
                    else
                        raw[q] = CONV ? __bfloat162float(halo_in[(row + 3) * 64 + pch]) : 0.f;
                }
                if (CONV && tg == 7) {
#pragma unroll
                    for (int j = 0; j < 3; j++)
                        halo_out[j * 64 + pch] = *(const bf16*)(st + tc::sw128_offset(61 + j, pch));
                }
                float ud[8], us[8];
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    const int t = r0 + q;
                    float u;
                    if (CONV) {
                        // a boundary at chunk position r (r >= 0 from the masks,
                        // -2/-1 from the two positions before the chunk)
                        auto bd = [&](int r) -> bool {
                            if (r >= 32) return (m1 >> (r - 32)) & 1u;
                            if (r >= 0) return (m0 >> r) & 1u;
                            return (pre >> (r + 2)) & 1u;
                        };
                        const bool ok2 = !bd(t);
                        const bool ok1 = ok2 && !bd(t - 1);
                        const bool ok0 = ok1 && !bd(t - 2);
                        float acc = cbias + wk[3] * raw[q + 3];
                        acc += ok2 ? wk[2] * raw[q + 2] : 0.f;
                        acc += ok1 ? wk[1] * raw[q + 1] : 0.f;
                        acc += ok0 ? wk[0] * raw[q] : 0.f;
                        u = fast_silu(acc);
                    } else {
                        u = raw[q + 3];
                    }
                    *(bf16*)(sm + LY::kXb + tc::sw128_offset(t, pch)) = __float2bfloat16(u);
                    const bool valid = t < Lc;
                    ud[q] = valid ? dts[t] * u : 0.f;
                    us[q] = (valid && seg_of(m0, m1, t) == seg_last)
                                ? __expf(acs_last - acv[t]) * ud[q] : 0.f;
                }
                const uint4 vd = make_uint4(pack_bf16(ud[0], ud[1]), pack_bf16(ud[2], ud[3]),
                                            pack_bf16(ud[4], ud[5]), pack_bf16(ud[6], ud[7]));
                const uint4 vs = make_uint4(pack_bf16(us[0], us[1]), pack_bf16(us[2], us[3]),
                                            pack_bf16(us[4], us[5]), pack_bf16(us[6], us[7]));
                *(uint4*)(sm + LY::kXd + tc::sw128_offset(pch, r0)) = vd;
                *(uint4*)(sm + LY::kXs + tc::sw128_offset(pch, r0)) = vs;
            }

            // ---- (B) state hand-off: h_c -> bf16 h^T operand; TMEM state <- k_c h_c
            const float carry = reset ? 0.f : __expf(acs_last);
            if (NS == 128) {
                const int n = 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint32_t r[16];
                    tc::tmem_ld16(tmem + lane_base + kColST + q * 16, r);
                    tc::tmem_wait_ld();
                    uint4 lo, hi;
                    lo.x = pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
                    lo.y = pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
                    lo.z = pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
                    lo.w = pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
                    hi.x = pack_bf16(__uint_as_float(r[8]), __uint_as_float(r[9]));
                    hi.y = pack_bf16(__uint_as_float(r[10]), __uint_as_float(r[11]));
                    hi.z = pack_bf16(__uint_as_float(r[12]), __uint_as_float(r[13]));
                    hi.w = pack_bf16(__uint_as_float(r[14]), __uint_as_float(r[15]));
                    *(uint4*)(sm + LY::kHt + tc::sw128_offset(n, q * 16)) = lo;
                    *(uint4*)(sm + LY::kHt + tc::sw128_offset(n, q * 16 + 8)) = hi;
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        r[j] = __float_as_uint(reset ? 0.f : carry * __uint_as_float(r[j]));
                    tc::tmem_st16(tmem + lane_base + kColST + q * 16, r);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    uint32_t r[16];
                    tc::tmem_ld16_x2_32(tmem + lane_base + kColST + q * 16, r);
                    tc::tmem_wait_ld();
                    uint4 lo, hi;
                    lo.x = pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
                    lo.y = pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
                    lo.z = pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
                    lo.w = pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
                    hi.x = pack_bf16(__uint_as_float(r[8]), __uint_as_float(r[9]));
                    hi.y = pack_bf16(__uint_as_float(r[10]), __uint_as_float(r[11]));
                    hi.z = pack_bf16(__uint_as_float(r[12]), __uint_as_float(r[13]));
                    hi.w = pack_bf16(__uint_as_float(r[14]), __uint_as_float(r[15]));
                    *(uint4*)(sm + LY::kHt + tc::sw128_offset(r16, c16 + q * 16)) = lo;
                    *(uint4*)(sm + LY::kHt + tc::sw128_offset(r16, c16 + q * 16 + 8)) = hi;
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        r[j] = __float_as_uint(reset ? 0.f : carry * __uint_as_float(r[j]));
                    tc::tmem_st16_x2_32(tmem + lane_base + kColST + q * 16, r);
                }
            }
            tc::tmem_wait_st();

            // ---- (C) mask: M[t][s] from the C B^T accumulator
            if (tid == 0) tc::bulk_wait_read0();     // the previous out tile has left shared memory
            bar_compute();
            tc::mbar_wait(cb_done, c & 1, s_abort, p.status, kStatusTimeout);
            tc::tc_fence_after();
            {
                const int t = r16;
                const float at = acv[t];
                const int segt = seg_of(m0, m1, t);
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    uint32_t r[16];
                    tc::tmem_ld16_x2_32(tmem + lane_base + kColCB + q * 16, r);
                    tc::tmem_wait_ld();
                    float mv[16];
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const int sidx = c16 + q * 16 + j;
                        const bool keep = sidx <= t && seg_of(m0, m1, sidx) == segt;
                        mv[j] = keep ? __uint_as_float(r[j]) * __expf(at - acv[sidx]) : 0.f;
                    }
                    const uint4 lo = make_uint4(pack_bf16(mv[0], mv[1]), pack_bf16(mv[2], mv[3]),
                                                pack_bf16(mv[4], mv[5]), pack_bf16(mv[6], mv[7]));
                    const uint4 hi = make_uint4(pack_bf16(mv[8], mv[9]), pack_bf16(mv[10], mv[11]),
                                                pack_bf16(mv[12], mv[13]), pack_bf16(mv[14], mv[15]));
                    *(uint4*)(sm + LY::kMop + tc::sw128_offset(t, c16 + q * 16)) = lo;
                    *(uint4*)(sm + LY::kMop + tc::sw128_offset(t, c16 + q * 16 + 8)) = hi;
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::mbar_arrive(ops_ready);

            // ---- (D) epilogue: out = (Ydiag + f Yoff + D u) SiLU(z)
            tc::mbar_wait(mma_done, c & 1, s_abort, p.status, kStatusTimeout);
            tc::tc_fence_after();
            {
                const int t = r16;
                const float f = (seg_of(m0, m1, t) == 0) ? __expf(acv[t]) : 0.f;
                const uint8_t* zt = st + kTile;
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    uint32_t ry[16], ro[16];
                    tc::tmem_ld16_x2_32(tmem + lane_base + kColY + q * 16, ry);
                    tc::tmem_ld16_x2_32(tmem + lane_base + kColYO + q * 16, ro);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int hh = 0; hh < 2; hh++) {
                        const int col = c16 + q * 16 + hh * 8;
                        const uint4 xv = *(const uint4*)(sm + LY::kXb + tc::sw128_offset(t, col));
                        const uint4 zv = *(const uint4*)(zt + tc::sw128_offset(t, col));
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                        const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
                        uint32_t ow[4];
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            float o2[2];
#pragma unroll
                            for (int k = 0; k < 2; k++) {
                                const int j = hh * 8 + e * 2 + k;
                                const float xu = __uint_as_float(k ? (xw[e] & 0xFFFF0000u) : (xw[e] << 16));
                                const float zz = __uint_as_float(k ? (zw[e] & 0xFFFF0000u) : (zw[e] << 16));
                                const float y = __uint_as_float(ry[j]) + f * __uint_as_float(ro[j]) + Dh * xu;
                                o2[k] = y * fast_silu(zz);
                            }
                            ow[e] = pack_bf16(o2[0], o2[1]);
                        }
                        *(uint4*)(sm + LY::kMop + tc::sw128_offset(t, col)) =
                            make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
            tc::fence_async_smem();
            const int aborted = bar_compute_or(*s_abort);
            if (tid == 0) {
                tc::tma_store_3d(&tm_out, sm + LY::kMop, h * 64, t0, b);
                tc::bulk_commit();
                tc::mbar_arrive(&empty[s]);
            }
            if (aborted) break;
        }

        // ---- final state (state^T in TMEM: rows n, columns p) -> (b, h, p, n)
        if (p.final_ssm != nullptr && !*s_abort) {
            tc::tc_fence_after();
            float* fs = p.final_ssm + bh * 64 * NS;
            if (NS == 128) {
                const int n = 32 * warp + lane;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint32_t r[16];
                    tc::tmem_ld16(tmem + lane_base + kColST + q * 16, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; j++) fs[(int64_t)(q * 16 + j) * NS + n] = __uint_as_float(r[j]);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    uint32_t r[16];
                    tc::tmem_ld16_x2_32(tmem + lane_base + kColST + q * 16, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        fs[(int64_t)(c16 + q * 16 + j) * NS + r16] = __uint_as_float(r[j]);
                }
            }
        }
        if (tid == 0) tc::bulk_wait0();
    }

    // ---- teardown: no MMA may still be running when the tensor memory is freed
    if (warp == 5 && lane == 0) {
        tc::mma_commit(&bar[7]);
        tc::mbar_drain(&bar[7], 0, p.status, kStatusTimeout);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// ------------------------------------------------------------------------------------------
// host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
    }
    return fn;
}

// [64 channels x 64 tokens] bf16 boxes with the 128-byte swizzle over a
// (batch, seqlen, width) row-major tensor.
static bool encode_tile_map(CUtensorMap* m, const void* base, int width, int seqlen, int batch)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)seqlen, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)width * 2 * seqlen};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool fused_path_available() { return tensor_map_encoder() != nullptr; }

template <int NS, bool CONV>
static cudaError_t launch_t(const Shape& s, const FusedParams& fp, const CUtensorMap* maps,
                            cudaStream_t st)
{
    auto kern = ssd_chunk_fused<NS, CONV>;
    const int smem = Layout<NS>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<s.batch * s.nheads, kThreads, smem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], fp);
    return cudaGetLastError();
}

cudaError_t launch_chunk_fused(const Shape& s, const FwdArgs& a, const void* ubc, const float* dt,
                               const float* acs, int* status, cudaStream_t st)
{
    if (!s.act_bf16 || s.headdim != 64 || (s.dstate != 64 && s.dstate != 128) || s.bc_norm)
        return cudaErrorNotSupported;
    const int HP = s.nheads * 64, GN = s.ngroups * s.dstate;
    CUtensorMap maps[5];
    bool ok = encode_tile_map(&maps[0], a.x, HP, s.seqlen, s.batch) &&
              encode_tile_map(&maps[1], a.z, HP, s.seqlen, s.batch) &&
              encode_tile_map(&maps[4], a.out, HP, s.seqlen, s.batch);
    if (s.dconv == 4) {
        ok = ok && encode_tile_map(&maps[2], ubc, 2 * GN, s.seqlen, s.batch);
        maps[3] = maps[2];
    } else {
        ok = ok && encode_tile_map(&maps[2], a.B, GN, s.seqlen, s.batch) &&
             encode_tile_map(&maps[3], a.C, GN, s.seqlen, s.batch);
    }
    if (!ok) return cudaErrorInvalidValue;
    FusedParams fp;
    fp.batch = s.batch;
    fp.seqlen = s.seqlen;
    fp.nheads = s.nheads;
    fp.ngroups = s.ngroups;
    fp.conv = s.dconv == 4;
    fp.dt = dt;
    fp.acs = acs;
    fp.seq = a.seq_idx;
    fp.D = a.D;
    fp.conv_w = (const bf16*)a.conv_w;
    fp.conv_b = (const bf16*)a.conv_b;
    fp.init_conv = (const bf16*)a.init_conv;
    fp.init_ssm = a.init_ssm;
    fp.final_ssm = a.final_ssm;
    fp.status = status;
    if (s.dstate == 64)
        return s.dconv == 4 ? launch_t<64, true>(s, fp, maps, st) : launch_t<64, false>(s, fp, maps, st);
    return s.dconv == 4 ? launch_t<128, true>(s, fp, maps, st) : launch_t<128, false>(s, fp, maps, st);
}

}  // namespace ssd

