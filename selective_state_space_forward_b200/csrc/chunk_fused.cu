// chunk_fused.cu -- KF: the fused chunk sweep of the SSD scan on sm_100a.
//
// Work: every (batch row, head) stream of 64-token chunks (chunk 64: mojolearn
// Mamba3Block) is cut into segments of consecutive chunks.  Per chunk c, with
// acs the segmented cumsum of dt*a written by K2 and seg_t the number of
// document boundaries at t0 .. t:
//
//   conv      u_t = SiLU(conv(x)) for the head's 64 channels (K1's arithmetic;
//             B and C of the group come pre-convolved from K1, or raw)
//             Xs[s] = exp(acs_last - acs_s) dt_s u_s  [seg_s = seg_last]
//   CB        S = C B^T                      tcgen05, 64 x 64 x N
//   mask      M[t,s] = S[t,s] exp(acs_t - acs_s) dt_s  [s <= t, seg_s = seg_t]
//   Ydiag     M u                            tcgen05, 64 x 64 x 64
//   Yoff      C h_c^T                        tcgen05, 64 x 64 x N (bf16 copy of h_c)
//   chunk     S_c = B^T Xs                   tcgen05, N x 64 x 64
//   state     h_{c+1} = k_c h_c + S_c        fp32, in registers
//             (k_c = exp(acs_last), dropped when the chunk holds a boundary)
//   epilogue  out_t = (Ydiag_t + [seg_t = 0] exp(acs_t) Yoff_t + D u_t) SiLU(z_t)
//
// Schedule: a persistent grid (every CTA resident) takes work items -- segment
// k of stream s -- in the order j = k * streams + s, CTA i taking i, i + G, ...
// A segment's entering state is the previous segment's leaving state, handed
// over through global memory with an epoch-tagged flag; because items are
// segment-major and every CTA is resident, each dependency points to an item
// started earlier and the wait ends.  This keeps every SM busy to within one
// item whatever the number of streams, and lets two CTAs share each SM.
//
// Roles (544 threads).  The work of a chunk splits in two: what does not
// depend on the carried state (conv, operand tiles, C B^T, mask, Ydiag, the
// chunk state S) and what does (the state update, Yoff, the epilogue).
// Group A (warps 0-7) does the first part and its thread 0 issues those MMAs;
// group B (warps 8-15) does the second, its thread 0 issuing Yoff and the TMA
// store.  Operand tiles, Ydiag and S are double-buffered, so group A works on
// chunk c+1 while group B finishes chunk c; warp 16 feeds both from a TMA
// ring (tiles plus the chunk's per-token scalars).  A warp reaches TMEM lanes
// 32*(w%4) .. +31.  Every wait is bounded: after 1 s a waiter raises the
// CTA's abort flag and the device status word, and all roles drain and exit.
//
// Tile layouts (see tc05.cuh): x, z, B, C, out tiles are [64 tokens][64
// channels] bf16 with the 128-byte swizzle, as TMA writes them; N = 128
// operands are two such tiles side by side.  M=64 accumulators put row r in
// TMEM lane 32*(r/16) + r%16; M=128 ones put row r in lane r.
#include <cudaTypedefs.h>

#include <type_traits>

#include "ssd_device.cuh"
#include "ssd_kernels.h"
#include "tc05.cuh"

namespace ssd {
namespace {

constexpr int kGroupWarps = 8;                       // warps per compute group
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kProducerWarp = 2 * kGroupWarps;       // after groups A (0-7) and B (8-15)
constexpr int kThreads = 32 * (2 * kGroupWarps + 1);
constexpr int kBarA = 1, kBarB = 2;                  // named barriers of the groups
constexpr int kTile = 64 * 128;        // one [64][64] bf16 tile
constexpr uint32_t kTmemCols = 512;
// TMEM columns: C B^T; Ydiag [2]; Yoff; chunk state S [2]
constexpr uint32_t kColCB = 0, kColY = 64, kColYO = 192, kColS = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kItemsPerSm = 16;        // bound on work items per SM (sizes the hand-off buffers)

struct FusedParams {
    int batch, seqlen, nheads, ngroups;
    int nseg, cps, nitems;    // segments per stream, chunks per segment, items
    unsigned epoch;           // tag of this call's hand-off flags
    const float* dt;          // (B, H, L) from K2
    const float* acs;         // (B, H, L) segmented cumsum from K2
    const int32_t* seq;       // (B, L) or null
    const int32_t* lengths;   // (B) real tokens per row of a ragged batch, or null
    const float* D;
    const bf16* x;            // raw x, for the conv history at segment starts
    int64_t ld_x;             // its row stride (elements)
    const bf16* conv_w;       // (conv_dim, 4) or null
    const bf16* conv_b;
    const bf16* init_conv;    // (B, 3, conv_dim) or null
    const float* init_ssm;    // (B, H, 64, N) or null
    float* final_ssm;         // or null
    float* hseg;              // (streams, nseg, 64, N) segment leaving states
    unsigned* flags;          // (streams, nseg)
    int* status;
    uint64_t wait_ns;         // limit of every bounded wait
    int withhold;             // testing: this stream's first hand-off is never published (-1: none)
    // B/C RMSNorm + per-head bias (NORM kernels only)
    const float* rinv;        // (B, L, 2G): 1/rms of B (g) and C (G + g) per token
    const float *bn_w, *cn_w; // (N) or null (ones)
    const float *bn_bias, *cn_bias;   // (H, N) or null (zeros)
};

// Per-token values of one chunk, written by the producer warp.
struct ChunkScalars {
    float dt[64];      // dt_t (0 past the end of the sequence)
    float wd[64];      // [seg_t = seg_last] exp(acs_last - acs_t) dt_t
    float f[64];       // [seg_t = 0] exp(acs_t): weight of the carried-state term
    float a2[64];      // acs_t * log2(e)
    float g[64];       // dt_s 2^(a2ref(block of s) - a2_s): column factor of the mask
    float rb[64], rc[64];   // NORM: 1/rms of the token's B and C rows
    uint8_t seg[64];   // document boundaries at chunk positions 0 .. t
    float a2ref[4];    // a2 at the last token of each 16-token block (within the chunk)
    float carry;       // exp(acs_last), or kChunkReset when the chunk holds a boundary
    uint32_t m0, m1;   // boundary at chunk position r (bit r of m0 | m1 << 32)
    uint32_t pre;      // bit 0: boundary at t0-2, bit 1: at t0-1
    uint32_t fast;     // bit b: the mask of column block b may use the factored decay
    uint32_t nvalid;   // real tokens of the chunk (rows from here on are ragged-batch padding)
    uint32_t pad[2];
};
static_assert(sizeof(ChunkScalars) % 16 == 0, "ChunkScalars keeps 16-byte alignment");

// Largest decay (in log2 units) across a 16-token block for which the mask
// factors exp2(a2_t - a2_s) into 2^(a2_t - a2ref) 2^(a2ref - a2_s): both factors
// then stay within 2^-64 .. 2^64, far from fp32 under- and overflow.
constexpr float kMaskBlockRange = 64.0f;

template <int NS>
struct Layout {
    static constexpr int kStages = NS == 64 ? 3 : 2;          // TMA ring depth
    static constexpr int kBC = (NS / 64) * kTile;
    static constexpr int kStage = 2 * kTile + 2 * kBC;        // x, z, B, C
    static constexpr int kRing = kStages * kStage;
    static constexpr int kXb = kRing;                         // [2] u in bf16, [t][p]
    static constexpr int kXs = kXb + 2 * kTile;               // [2] decayed dt u, [p][t]
    static constexpr int kMop = kXs + 2 * kTile;              // [2] mask operand, [t][s]
    static constexpr int kOut = kMop + 2 * kTile;             // [2] out tiles
    static constexpr int kHt = kOut + 2 * kTile;              // h^T, NS rows x 128 B
    static constexpr int kScal = kHt + NS * 128;              // ChunkScalars[kStages]
    static constexpr int kHalo = kScal + kStages * (int)sizeof(ChunkScalars);   // u32 [2][3][32]
    static constexpr int kBar = kHalo + 2 * 3 * 32 * 4;
    static constexpr int kNumBars = 3 * kStages + 12;
    static constexpr int kMisc = kBar + kNumBars * 8;         // tmem base, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;              // slack for 1024-byte alignment
};

// Named barriers of the two compute groups (barrier 0 is __syncthreads).
__device__ __forceinline__ void bar_group(int id)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGroupThreads) : "memory");
}

// Group barrier that also returns the OR of v over the group, so every thread
// of the group takes the same branch afterwards.
__device__ __forceinline__ int bar_group_or(int id, int v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v), "r"(id), "n"(kGroupThreads)
        : "memory");
    return (int)r;
}

__device__ __forceinline__ uint32_t mask_le(int i) { return i >= 31 ? 0xffffffffu : ((2u << i) - 1u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed fp32 pairs (the f32x2 arithmetic of sm_100): one instruction computes
// both lanes, each rounded exactly as the scalar fma.rn / mul.rn would.
__device__ __forceinline__ uint64_t p2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void p2split(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// both halves of a packed bf16 pair as an fp32 pair
__device__ __forceinline__ uint64_t bf2(uint32_t w) { return p2(bf_lo(w), bf_hi(w)); }
// SiLU of a pair, as silu_t: h + h tanh(h) with h = v/2
__device__ __forceinline__ uint64_t silu2(uint64_t v)
{
    const uint64_t h = mul2(v, p2(0.5f, 0.5f));
    float h0, h1, t0, t1;
    p2split(h, h0, h1);
    asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(h0));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(h1));
    return fma2(h, p2(t0, t1), h);
}
__device__ __forceinline__ uint32_t pack_bf16_2(uint64_t v)
{
    float lo, hi;
    p2split(v, lo, hi);
    return pack_bf16(lo, hi);
}

// The flattened step sequence a CTA walks: its work items in order, each item's
// chunks in order.  Every role iterates it identically.
struct StepIter {
    int j, c, cend, b, h, k;
    int H, nstr, cps, nc, nitems, G;
    __device__ StepIter(const FusedParams& p, int nc_)
    {
        H = p.nheads; nstr = p.batch * p.nheads; cps = p.cps; nc = nc_;
        nitems = p.nitems; G = gridDim.x;
        j = blockIdx.x;
        load_item();
    }
    __device__ void load_item()
    {
        if (j >= nitems) return;
        k = j / nstr;
        const int s = j % nstr;
        b = s / H;
        h = s % H;
        c = k * cps;
        cend = min(c + cps, nc);
    }
    __device__ bool valid() const { return j < nitems; }
    __device__ bool first() const { return c == k * cps; }
    __device__ bool last() const { return c == cend - 1; }
    __device__ void next()
    {
        if (++c >= cend) {
            j += G;
            load_item();
        }
    }
};

// Phase parity of the n-th completion (0-based) of a barrier.
__device__ __forceinline__ uint32_t par(int n) { return (uint32_t)n & 1u; }

template <int NS, bool CONV, bool NORM, bool RAG>
__global__ void __launch_bounds__(kThreads, 1)
ssd_chunk_fused(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                const __grid_constant__ CUtensorMap tm_out, FusedParams p)
{
    using LY = Layout<NS>;
    constexpr int NST = LY::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the shared array by pointer
    // arithmetic so that every access through it compiles to ld/st.shared
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    ChunkScalars* scal = (ChunkScalars*)(sm + LY::kScal);
    uint32_t* s_halo = (uint32_t*)(sm + LY::kHalo);
    uint64_t* bar = (uint64_t*)(sm + LY::kBar);
    uint64_t* full = bar;                  // [NST] tiles + scalars of a step landed
    uint64_t* empty = bar + NST;           // [NST] group B released the stage
    uint64_t* cb_done = bar + 2 * NST;     // C B^T of the next step in TMEM
    uint64_t* s_done = cb_done + 1;        // [2] chunk state S(q) in TMEM
    uint64_t* s_free = s_done + 2;         // [2] group B has read S(q)
    uint64_t* y_done = s_free + 2;         // [2] Ydiag(q) done (with every earlier MMA of group A)
                                           //     and the step's Xb written
    uint64_t* yo_done = y_done + 2;        // Yoff(q)
    uint64_t* epi_done = yo_done + 1;      // [2] group B is done with the step's operands
    uint64_t* drain_a = epi_done + 2;
    uint64_t* drain_b = drain_a + 1;
    uint64_t* norm_done = drain_b + 1;     // [NST] NORM: the stage's B and C tiles are normalised
    uint32_t* s_tmem = (uint32_t*)(sm + LY::kMisc);
    volatile int* s_abort = (volatile int*)(sm + LY::kMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.nheads, L = p.seqlen;
    const int nc = (L + 63) / 64;

    if (tid == 0) {
        for (int i = 0; i < NST; i++) {
            tc::mbar_init(&full[i], 33);     // producer: expect_tx arrive + 32 lane arrivals
            tc::mbar_init(&empty[i], 1);
            tc::mbar_init(&norm_done[i], 1);
        }
        tc::mbar_init(cb_done, 1);
        tc::mbar_init(yo_done, 1);
        tc::mbar_init(drain_a, 1);
        tc::mbar_init(drain_b, 1);
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&s_done[i], 1);
            tc::mbar_init(&s_free[i], 1);
            tc::mbar_init(&y_done[i], 2);    // A's release arrive (Xb written) + the MMA commit
            tc::mbar_init(&epi_done[i], 1);
        }
        *s_abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(s_tmem, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
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
    const int sub = warp & 3;                           // TMEM lane quarter of this warp
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        // Software-pipelined by one step: the global loads of step q+1's per-token
        // values are issued, then step q's scalars are computed from the values
        // loaded one iteration earlier, and only then does the warp wait for step
        // q's ring slot.  A freed slot is refilled by the TMA issue and a few
        // shared-memory stores.
        const uint32_t tx = (uint32_t)(2 * kTile + 2 * LY::kBC);
        struct Raw {
            float dt[2], ac[2], rb[2], rc[2];
            int32_t sq[2], sqm[2];    // seq_idx at t and t-1
            int32_t ps, psm;          // lanes 0, 1: seq_idx at t0-2+lane and one before
            int32_t len;              // lengths[b] (ragged batch)
        };
        auto load_raw = [&](const StepIter& s, Raw& r) {
            const int b = s.b, h = s.h, g = h / (H / p.ngroups);
            const int t0 = s.c * 64;
            const int64_t bh = (int64_t)b * H + h;
            const int32_t* seq_row = p.seq ? p.seq + (int64_t)b * L : nullptr;
            const float* dt_row = p.dt + bh * L;
            const float* acs_row = p.acs + bh * L;
            r.len = RAG ? p.lengths[b] : L;
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int t = t0 + hf * 32 + lane;
                const bool ok = t < L;
                r.dt[hf] = ok ? dt_row[t] : 0.0f;
                r.ac[hf] = ok ? acs_row[t] : 0.0f;
                r.sq[hf] = (seq_row && ok) ? seq_row[t] : 0;
                r.sqm[hf] = (seq_row && ok && t > 0) ? seq_row[t - 1] : 0;
                if (NORM) {
                    const int64_t tok = ((int64_t)b * L + t) * (2 * p.ngroups);
                    r.rb[hf] = ok ? p.rinv[tok + g] : 0.0f;
                    r.rc[hf] = ok ? p.rinv[tok + p.ngroups + g] : 0.0f;
                }
            }
            const int tt = t0 - 2 + lane;
            const bool okp = seq_row && lane < 2 && tt >= 1 && tt < L;
            r.ps = okp ? seq_row[tt] : 0;
            r.psm = okp ? seq_row[tt - 1] : 0;
        };
        // the scalars of one step, as each lane stores them
        struct Vals {
            float dt[2], wd[2], f[2], a2[2], g[2], rb[2], rc[2], a2ref[2], carry;
            int seg[2];
            uint32_t m0, m1, pre, fast, nvalid;
        };
        auto compute = [&](const StepIter& s, const Raw& r, Vals& v) {
            const int t0 = s.c * 64;
            const int Lb = RAG ? min(max((int)r.len, 0), L) : L;
            const int Lc = min(64, L - t0);
            int bdv[2];
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int t = t0 + hf * 32 + lane;
                bdv[hf] = (p.seq && t > 0 && t < Lb) ? (r.sq[hf] != r.sqm[hf]) : 0;
            }
            const uint32_t m0 = __ballot_sync(0xffffffffu, bdv[0]);
            const uint32_t m1 = __ballot_sync(0xffffffffu, bdv[1]);
            const int seg0 = __popc(m0 & mask_le(lane));
            const int seg1 = __popc(m0) + __popc(m1 & mask_le(lane));
            const int last = Lc - 1;
            const int seg_last = __shfl_sync(0xffffffffu, last < 32 ? seg0 : seg1, last & 31);
            const float acs_last = __shfl_sync(0xffffffffu, last < 32 ? r.ac[0] : r.ac[1], last & 31);
            const int segv[2] = {seg0, seg1};
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int rref = min((hf * 32 + lane) | 15, last);
                const float v0 = __shfl_sync(0xffffffffu, r.ac[0], rref & 31);
                const float v1 = __shfl_sync(0xffffffffu, r.ac[1], rref & 31);
                v.a2ref[hf] = (rref < 32 ? v0 : v1) * kLog2e;
            }
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int rr = hf * 32 + lane;
                const bool ok = rr < Lc;
                const float a2 = r.ac[hf] * kLog2e;
                v.dt[hf] = r.dt[hf];
                v.wd[hf] = (ok && segv[hf] == seg_last) ? __expf(acs_last - r.ac[hf]) * r.dt[hf] : 0.0f;
                v.f[hf] = (ok && segv[hf] == 0) ? __expf(r.ac[hf]) : 0.0f;
                v.a2[hf] = a2;
                v.g[hf] = ok ? r.dt[hf] * ex2(fminf(v.a2ref[hf] - a2, 0.0f)) : 0.0f;
                v.seg[hf] = segv[hf];
                v.rb[hf] = ok ? r.rb[hf] : 0.0f;
                v.rc[hf] = ok ? r.rc[hf] : 0.0f;
            }
            // block b may use the factored mask when the chunk holds no boundary and the
            // decay across the block stays within kMaskBlockRange
            const float a2first0 = __shfl_sync(0xffffffffu, r.ac[0], lane & 16) * kLog2e;
            const float a2first1 = __shfl_sync(0xffffffffu, r.ac[1], lane & 16) * kLog2e;
            const uint32_t okb0 = __ballot_sync(0xffffffffu, a2first0 - v.a2ref[0] <= kMaskBlockRange);
            const uint32_t okb1 = __ballot_sync(0xffffffffu, a2first1 - v.a2ref[1] <= kMaskBlockRange);
            const int tt = t0 - 2 + lane;
            const int pb = (lane < 2 && p.seq && tt >= 1 && tt < Lb) ? (r.ps != r.psm) : 0;
            v.pre = __ballot_sync(0xffffffffu, pb) & 3u;        // bit 0: t0-2, bit 1: t0-1
            v.nvalid = (uint32_t)min(max(Lb - t0, 0), 64);
            v.carry = (m0 | m1) ? kChunkReset : __expf(acs_last);
            v.m0 = m0;
            v.m1 = m1;
            // lanes 0 and 16 hold blocks 0, 1 (first half) and 2, 3 (second half)
            const uint32_t fb = ((okb0 & 1u) ? 1u : 0u) | ((okb0 >> 16) & 1u) << 1 |
                                ((okb1 & 1u) ? 1u : 0u) << 2 | ((okb1 >> 16) & 1u) << 3;
            v.fast = (m0 | m1) ? 0u : fb;
        };
        auto store = [&](ChunkScalars* cs, const Vals& v) {
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                const int rr = hf * 32 + lane;
                cs->dt[rr] = v.dt[hf];
                cs->wd[rr] = v.wd[hf];
                cs->f[rr] = v.f[hf];
                cs->a2[rr] = v.a2[hf];
                cs->g[rr] = v.g[hf];
                cs->seg[rr] = (uint8_t)v.seg[hf];
                if (NORM) {
                    cs->rb[rr] = v.rb[hf];
                    cs->rc[rr] = v.rc[hf];
                }
            }
            if (lane == 0) {
                if (RAG) cs->nvalid = v.nvalid;
                cs->carry = v.carry;
                cs->m0 = v.m0;
                cs->m1 = v.m1;
                cs->pre = v.pre;
                cs->fast = v.fast;
            }
            if (lane == 0 || lane == 16) {
                cs->a2ref[lane >> 4] = v.a2ref[0];
                cs->a2ref[2 + (lane >> 4)] = v.a2ref[1];
            }
        };
        int q = 0;
        StepIter it(p, nc);
        Raw cur, nxt;
        if (it.valid()) load_raw(it, cur);
        for (; it.valid(); q++) {
            const int st = q % NST;
            StepIter nx = it;
            nx.next();
            if (nx.valid()) load_raw(nx, nxt);          // in flight while this step is finished
            Vals v;
            compute(it, cur, v);
            if (q >= NST && !tc::mbar_wait_sleep(&empty[st], par(q / NST - 1), s_abort, p.status, kStatusTimeout, p.wait_ns))
                break;
            const int g = it.h / (H / p.ngroups);
            const int t0 = it.c * 64;
            uint8_t* stg = sm + st * LY::kStage;
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&full[st], tx);
                tc::tma_load_3d(stg, &tm_x, &full[st], it.h * 64, t0, it.b);
                tc::tma_load_3d(stg + kTile, &tm_z, &full[st], it.h * 64, t0, it.b);
#pragma unroll
                for (int jj = 0; jj < NS / 64; jj++) {
                    const int bx = g * NS + 64 * jj;
                    const int cx = (CONV ? p.ngroups * NS : 0) + g * NS + 64 * jj;
                    tc::tma_load_3d(stg + 2 * kTile + jj * kTile, &tm_b, &full[st], bx, t0, it.b);
                    tc::tma_load_3d(stg + 2 * kTile + LY::kBC + jj * kTile, &tm_c, &full[st], cx, t0, it.b);
                }
            }
            store(&scal[st], v);
            __syncwarp();
            tc::mbar_arrive(&full[st]);
            it = nx;
            cur = nxt;
        }
        // an aborting CTA lets its last loads land before the shared memory is released
        for (int k2 = max(0, q - NST); k2 < q; k2++)
            tc::mbar_drain(&full[k2 % NST], par(k2 / NST), p.status, kStatusTimeout, p.wait_ns);
    } else if (warp < kGroupWarps) {
        // ------------------------------------------------------------ group A: conv, mask
        // Warps 0-7.  Per step: conv -> Xb, Xs; [thread 0: S = B^T Xs]; mask from
        // C B^T -> Mop; [thread 0: Ydiag = M u, then C B^T of the next step].
        const int half = warp >> 2;                // column half
        const int r16 = 16 * sub + (lane & 15);    // M=64 accumulator row of this thread
        const int c16 = half * 16 + (lane < 16 ? 0 : 32);
        const int pp = lane;                       // conv: channel pair 2pp, 2pp+1
        const int r0 = 8 * warp;                   // conv: tokens r0 .. r0+7
        const int cdim = H * 64 + 2 * p.ngroups * NS;
        const bool issuer = tid == 0;
        const uint32_t id_64 = tc::idesc_bf16(64, 64, false, false);
        const uint32_t id_st = tc::idesc_bf16(NS, 64, true, false);
        const uint32_t id_mn = tc::idesc_bf16(64, 64, false, true);
        float wk[2][4] = {{0.f, 0.f, 0.f, 1.f}, {0.f, 0.f, 0.f, 1.f}}, cbias[2] = {0.f, 0.f};
        uint64_t wkp[4] = {0, 0, 0, 0}, cbp = 0;   // the same, channel pairs packed
        int cur_h = -1;

        // C B^T of one step into the CB columns (both operands K-major over n)
        auto issue_cb = [&](int st) {
            const uint32_t a_b = tc::smem_u32(sm + st * LY::kStage + 2 * kTile);
            const uint32_t a_c = a_b + LY::kBC;
#pragma unroll
            for (int kk = 0; kk < NS / 16; kk++) {
                const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                tc::mma_bf16(tmem + kColCB, tc::sdesc_sw128(a_c + off, 16, 1024),
                             tc::sdesc_sw128(a_b + off, 16, 1024), id_64, kk > 0);
            }
            tc::mma_commit(cb_done);
        };
        // NORM: rewrite the B and C tiles of stage st (step with head hh) in place as
        // B w / rms(B) + bias_h; thread tid takes 8 columns of rows tid / (NS/8) + k*(256/(NS/8))
        auto normalise = [&](int st, int hh) {
            uint8_t* stg = sm + st * LY::kStage;
            const ChunkScalars* cs = &scal[st];
            constexpr int kCh = NS / 8;                  // 8-column chunks per row
            constexpr int kRowStep = kGroupThreads / kCh;
            const int n8 = tid % kCh, n0 = n8 * 8;
            const int tile = n0 >> 6, col = n0 & 63;
#pragma unroll
            for (int which = 0; which < 2; which++) {
                const float* wv = which ? p.cn_w : p.bn_w;
                const float* bv = which ? p.cn_bias : p.bn_bias;
                float w8[8], b8[8];
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    w8[j] = wv ? __ldg(wv + n0 + j) : 1.0f;
                    b8[j] = bv ? __ldg(bv + (int64_t)hh * NS + n0 + j) : 0.0f;
                }
                uint8_t* tb = stg + 2 * kTile + which * LY::kBC + tile * kTile;
#pragma unroll
                for (int t = tid / kCh; t < 64; t += kRowStep) {
                    const float ri = which ? cs->rc[t] : cs->rb[t];
                    uint4* ptr = (uint4*)(tb + tc::sw128_offset(t, col));
                    const uint4 v = *ptr;
                    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const uint64_t sc = mul2(p2(w8[2 * j], w8[2 * j + 1]), p2(ri, ri));
                        o[j] = pack_bf16_2(fma2(bf2(vw[j]), sc, p2(b8[2 * j], b8[2 * j + 1])));
                    }
                    *ptr = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        };
        if (NORM) {
            StepIter it0(p, nc);
            tc::mbar_wait(&full[0], 0, s_abort, p.status, kStatusTimeout, p.wait_ns);
            normalise(0, it0.h);
            tc::fence_async_smem();
            bar_group(kBarA);
            if (issuer) tc::mbar_arrive(&norm_done[0]);
        }
        if (issuer && tc::mbar_wait(&full[0], 0, s_abort, p.status, kStatusTimeout, p.wait_ns)) {
            tc::tc_fence_after();
            issue_cb(0);
        }

        int q = 0;
        for (StepIter it(p, nc); it.valid(); q++) {
            const int st = q % NST, i = q & 1;
            const int b = it.b, h = it.h, t0 = it.c * 64;
            const bool first = it.first();
            if (CONV && h != cur_h) {
                cur_h = h;
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int ch = h * 64 + 2 * pp + e;
#pragma unroll
                    for (int kq = 0; kq < 4; kq++) wk[e][kq] = __bfloat162float(p.conv_w[(int64_t)ch * 4 + kq]);
                    cbias[e] = __bfloat162float(p.conv_b[ch]);
                }
#pragma unroll
                for (int kq = 0; kq < 4; kq++) wkp[kq] = p2(wk[0][kq], wk[1][kq]);
                cbp = p2(cbias[0], cbias[1]);
            }
            // On abort the waits return at once; every thread still runs the same
            // sequence of group barriers and leaves at the end of the iteration.
            tc::mbar_wait(&full[st], par(q / NST), s_abort, p.status, kStatusTimeout, p.wait_ns);
            // the operand buffers [i] and Ydiag columns [i] are free once group B
            // has finished step q-2
            if (q >= 2) tc::mbar_wait(&epi_done[i], par((q >> 1) - 1), s_abort, p.status, kStatusTimeout, p.wait_ns);
            const uint8_t* stg = sm + st * LY::kStage;
            const ChunkScalars* cs = &scal[st];
            const uint32_t m0 = cs->m0, m1 = cs->m1, pre = cs->pre;
            const bool quiet = (m0 | m1 | pre) == 0;      // no boundary near this chunk
            uint8_t* xb = sm + LY::kXb + i * kTile;
            uint8_t* xs = sm + LY::kXs + i * kTile;
            uint8_t* mop = sm + LY::kMop + i * kTile;

            // ---- conv and the operand tiles: channels 2pp, 2pp+1; tokens r0 .. r0+7
            {
                const uint32_t* halo_in = s_halo + (q & 1) * 96;
                uint32_t* halo_out = s_halo + ((q + 1) & 1) * 96;
                uint32_t raw[11];
#pragma unroll
                for (int qq = 0; qq < 11; qq++) {
                    const int row = r0 - 3 + qq;
                    if (row >= 0) {
                        raw[qq] = *(const uint32_t*)(stg + tc::sw128_offset(row, 2 * pp));
                    } else if (!CONV) {
                        raw[qq] = 0u;
                    } else if (!first) {
                        raw[qq] = halo_in[(row + 3) * 32 + pp];
                    } else {
                        // segment start: the three tokens before the chunk from the raw x,
                        // or the caller's conv history before token 0
                        const int tok = t0 + row;
                        raw[qq] = tok >= 0
                            ? *(const uint32_t*)(p.x + ((int64_t)b * L + tok) * p.ld_x + h * 64 + 2 * pp)
                            : (p.init_conv ? *(const uint32_t*)(p.init_conv + ((int64_t)b * 3 + (tok + 3)) * cdim +
                                                               h * 64 + 2 * pp)
                                           : 0u);
                    }
                }
                if (CONV && warp == 7) {
#pragma unroll
                    for (int jj = 0; jj < 3; jj++) halo_out[jj * 32 + pp] = raw[8 + jj];
                }
                // `quiet` is uniform over the block: a tap-mask-free body for it
                auto conv_tokens = [&](auto quiet_c) {
                    constexpr bool QUIET = decltype(quiet_c)::value;
                    float us[2][8];
#pragma unroll
                    for (int qq = 0; qq < 8; qq++) {
                        const int t = r0 + qq;
                        float u[2];
                        if (CONV && QUIET) {
                            // both channels at once: four taps and the SiLU on fp32 pairs
                            uint64_t acc = fma2(wkp[3], bf2(raw[qq + 3]), cbp);
                            acc = fma2(wkp[2], bf2(raw[qq + 2]), acc);
                            acc = fma2(wkp[1], bf2(raw[qq + 1]), acc);
                            acc = fma2(wkp[0], bf2(raw[qq]), acc);
                            p2split(silu2(acc), u[0], u[1]);
                        } else if (CONV) {
                            bool ok2 = true, ok1 = true, ok0 = true;
                            if (!QUIET) {
                                auto bd = [&](int r) -> bool {
                                    if (r >= 32) return (m1 >> (r - 32)) & 1u;
                                    if (r >= 0) return (m0 >> r) & 1u;
                                    return (pre >> (r + 2)) & 1u;
                                };
                                ok2 = !bd(t);
                                ok1 = ok2 && !bd(t - 1);
                                ok0 = ok1 && !bd(t - 2);
                            }
#pragma unroll
                            for (int e = 0; e < 2; e++) {
                                auto xv = [&](int k3) { return e ? bf_hi(raw[k3]) : bf_lo(raw[k3]); };
                                float acc = fmaf(wk[e][3], xv(qq + 3), cbias[e]);
                                if (QUIET) {
                                    acc = fmaf(wk[e][2], xv(qq + 2), acc);
                                    acc = fmaf(wk[e][1], xv(qq + 1), acc);
                                    acc = fmaf(wk[e][0], xv(qq), acc);
                                } else {
                                    acc += ok2 ? wk[e][2] * xv(qq + 2) : 0.f;
                                    acc += ok1 ? wk[e][1] * xv(qq + 1) : 0.f;
                                    acc += ok0 ? wk[e][0] * xv(qq) : 0.f;
                                }
                                u[e] = silu_t(acc);
                            }
                        } else {
                            u[0] = bf_lo(raw[qq + 3]);
                            u[1] = bf_hi(raw[qq + 3]);
                        }
                        *(uint32_t*)(xb + tc::sw128_offset(t, 2 * pp)) = pack_bf16(u[0], u[1]);
                        const float wdt = cs->wd[t];
                        p2split(mul2(p2(u[0], u[1]), p2(wdt, wdt)), us[0][qq], us[1][qq]);
                    }
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const uint4 vs = make_uint4(pack_bf16(us[e][0], us[e][1]), pack_bf16(us[e][2], us[e][3]),
                                                    pack_bf16(us[e][4], us[e][5]), pack_bf16(us[e][6], us[e][7]));
                        *(uint4*)(xs + tc::sw128_offset(2 * pp + e, r0)) = vs;
                    }
                };
                if (quiet) conv_tokens(std::true_type{});
                else conv_tokens(std::false_type{});
            }
            tc::fence_async_smem();
            bar_group(kBarA);
            // S_c^T[n][p] = B^T Xs into S[i] (A = the B tile as MN-major over n, K = s);
            // S[i] last held S(q-2), which group B has read once it arrived on s_free[i]
            if (issuer && (q < 2 || tc::mbar_wait(&s_free[i], par((q >> 1) - 1), s_abort, p.status,
                                                   kStatusTimeout, p.wait_ns))) {
                tc::tc_fence_after();
                const uint32_t a_b = tc::smem_u32(stg + 2 * kTile);
                const uint32_t a_xs = tc::smem_u32(xs);
#pragma unroll
                for (int kk = 0; kk < 4; kk++)
                    tc::mma_bf16(tmem + kColS + i * 64, tc::sdesc_sw128(a_b + kk * 2048, kTile, 1024),
                                 tc::sdesc_sw128(a_xs + kk * 32, 16, 1024), id_st, kk > 0);
                tc::mma_commit(&s_done[i]);
            }

            // ---- mask: M[t][s] from the C B^T accumulator
            tc::mbar_wait(cb_done, par(q), s_abort, p.status, kStatusTimeout, p.wait_ns);
            tc::tc_fence_after();
            {
                const int t = r16;
                uint32_t r[16];
                tc::tmem_ld16_x2_32(tmem + lane_base + kColCB + half * 16, r);
                tc::tmem_wait_ld();
                float mv[16];
                if (c16 > t) {
#pragma unroll
                    for (int jj = 0; jj < 16; jj++) mv[jj] = 0.f;
                } else if ((cs->fast >> (c16 >> 4)) & 1u) {
                    // factored decay: 2^(a2_t - a2ref) per row times the column factor g_s
                    const float fr = ex2(fminf(cs->a2[t] - cs->a2ref[c16 >> 4], kMaskBlockRange));
                    float gs[16];
#pragma unroll
                    for (int j4 = 0; j4 < 4; j4++) {
                        const float4 v = *reinterpret_cast<const float4*>(cs->g + c16 + 4 * j4);
                        gs[4 * j4] = v.x; gs[4 * j4 + 1] = v.y; gs[4 * j4 + 2] = v.z; gs[4 * j4 + 3] = v.w;
                    }
                    const uint64_t frp = p2(fr, fr);
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 2) {
                        float m0v, m1v;
                        p2split(mul2(mul2(p2(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1])), frp),
                                     p2(gs[jj], gs[jj + 1])), m0v, m1v);
                        mv[jj] = c16 + jj <= t ? m0v : 0.f;
                        mv[jj + 1] = c16 + jj + 1 <= t ? m1v : 0.f;
                    }
                } else {
                    const float at = cs->a2[t];
                    float as[16], ds[16];
#pragma unroll
                    for (int j4 = 0; j4 < 4; j4++) {
                        const float4 v = *reinterpret_cast<const float4*>(cs->a2 + c16 + 4 * j4);
                        as[4 * j4] = v.x; as[4 * j4 + 1] = v.y; as[4 * j4 + 2] = v.z; as[4 * j4 + 3] = v.w;
                        const float4 d = *reinterpret_cast<const float4*>(cs->dt + c16 + 4 * j4);
                        ds[4 * j4] = d.x; ds[4 * j4 + 1] = d.y; ds[4 * j4 + 2] = d.z; ds[4 * j4 + 3] = d.w;
                    }
#pragma unroll
                    for (int jj = 0; jj < 16; jj++) ds[jj] *= __uint_as_float(r[jj]);   // C_t.B_s dt_s
                    if (quiet) {
#pragma unroll
                        for (int jj = 0; jj < 16; jj++)
                            mv[jj] = c16 + jj <= t ? ds[jj] * ex2(at - as[jj]) : 0.f;
                    } else {
                        const uint4 sv = *reinterpret_cast<const uint4*>(cs->seg + c16);
                        const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
                        const uint32_t segt = cs->seg[t];
#pragma unroll
                        for (int jj = 0; jj < 16; jj++) {
                            const uint32_t sj = (sw[jj >> 2] >> (8 * (jj & 3))) & 0xFFu;
                            const bool keep = c16 + jj <= t && sj == segt;
                            mv[jj] = keep ? ds[jj] * ex2(at - as[jj]) : 0.f;
                        }
                    }
                }
                const uint4 lo = make_uint4(pack_bf16(mv[0], mv[1]), pack_bf16(mv[2], mv[3]),
                                            pack_bf16(mv[4], mv[5]), pack_bf16(mv[6], mv[7]));
                const uint4 hi = make_uint4(pack_bf16(mv[8], mv[9]), pack_bf16(mv[10], mv[11]),
                                            pack_bf16(mv[12], mv[13]), pack_bf16(mv[14], mv[15]));
                *(uint4*)(mop + tc::sw128_offset(t, c16)) = lo;
                *(uint4*)(mop + tc::sw128_offset(t, c16 + 8)) = hi;
            }
            it.next();
            if (NORM && it.valid()) {
                // the next step's B and C tiles, before its C B^T and Yoff read them
                const int q1 = q + 1;
                tc::mbar_wait(&full[q1 % NST], par(q1 / NST), s_abort, p.status, kStatusTimeout, p.wait_ns);
                normalise(q1 % NST, it.h);
            }
            tc::fence_async_smem();
            tc::tc_fence_before();                 // the CB columns have been read
            const int aborted = bar_group_or(kBarA, *s_abort);
            if (issuer && !aborted) {
                // release: group B reads this step's Xb after it acquires y_done[i]
                tc::mbar_arrive(&y_done[i]);
                tc::tc_fence_after();
                // Ydiag = M u into Y[i] (K = s; u is [s][p], MN-major); its commit also
                // covers C B^T and S of this step
                const uint32_t a_mop = tc::smem_u32(mop), a_xb = tc::smem_u32(xb);
#pragma unroll
                for (int kk = 0; kk < 4; kk++)
                    tc::mma_bf16(tmem + kColY + i * 64, tc::sdesc_sw128(a_mop + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(a_xb + kk * 2048, 8192, 1024), id_mn, kk > 0);
                tc::mma_commit(&y_done[i]);
                // C B^T of the next step (the CB columns were read above)
                if (it.valid()) {
                    const int q1 = q + 1;
                    if (NORM) tc::mbar_arrive(&norm_done[q1 % NST]);
                    if (tc::mbar_wait(&full[q1 % NST], par(q1 / NST), s_abort, p.status, kStatusTimeout, p.wait_ns)) {
                        tc::tc_fence_after();
                        issue_cb(q1 % NST);
                    }
                }
            }
            if (aborted) break;
        }
        if (issuer) {
            tc::mma_commit(drain_a);
            tc::mbar_drain(drain_a, 0, p.status, kStatusTimeout, p.wait_ns);
        }
    } else if (warp < 2 * kGroupWarps) {
        // ------------------------------------------------------------ group B: state, epilogue
        // Warps 8-15.  Per step: h_c = k h_{c-1} + S(q-1) (or the entering state) ->
        // h^T; [thread 0: Yoff = C h^T]; out = (Ydiag + f Yoff + D u) SiLU(z) -> TMA store.
        const int half = (warp - kGroupWarps) >> 2;
        const int btid = tid - kGroupThreads;
        const bool issuer = btid == 0;
        const int r16 = 16 * sub + (lane & 15);
        const int c16 = half * 16 + (lane < 16 ? 0 : 32);
        // the carried state h: S^T[n][p] layout of the state MMA
        constexpr int HR = NS == 128 ? 32 : 16;
        const int nrow = NS == 128 ? 32 * sub + lane : r16;
        const int pcol = NS == 128 ? half * 32 : c16;
        const uint32_t id_yo = tc::idesc_bf16(64, 64, false, true);
        const uint32_t a_ht = tc::smem_u32(sm + LY::kHt);
        float hs[HR];
        float Dh = 0.f, carry_prev = 0.f;
        int cur_h = -1;
        auto load_S = [&](int bi, uint32_t (&r)[HR]) {
            const uint32_t col = kColS + bi * 64;
            if (NS == 128) {
                tc::tmem_ld16(tmem + lane_base + col + half * 32, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                tc::tmem_ld16(tmem + lane_base + col + half * 32 + 16,
                              *reinterpret_cast<uint32_t(*)[16]>(&r[16 % HR]));
            } else {
                tc::tmem_ld16_x2_32(tmem + lane_base + col + half * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            }
            tc::tmem_wait_ld();
        };

        int q = 0;
        for (StepIter it(p, nc); it.valid(); q++) {
            const int st = q % NST, i = q & 1;
            const int b = it.b, h = it.h, t0 = it.c * 64;
            const int64_t str = (int64_t)b * H + h;
            const bool first = it.first(), last = it.last();
            const bool stream_end = it.c == nc - 1;
            const int seg_k = it.k;
            if (h != cur_h) {
                cur_h = h;
                Dh = p.D[h];
            }
            tc::mbar_wait(&full[st], par(q / NST), s_abort, p.status, kStatusTimeout, p.wait_ns);
            const uint8_t* stg = sm + st * LY::kStage;
            const ChunkScalars* cs = &scal[st];
            const float carry = cs->carry;

            // ---- state entering this chunk -> bf16 h^T (the Yoff operand)
            if (first) {
                const float* src = nullptr;
                if (seg_k == 0) {
                    src = p.init_ssm ? p.init_ssm + str * 64 * NS : nullptr;
                } else {
                    // the previous segment's leaving state (an item started earlier)
                    const unsigned* fl = p.flags + str * p.nseg + (seg_k - 1);
                    if (issuer) {
                        const uint64_t tw = tc::global_ns();
                        unsigned v;
                        for (;;) {
                            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(fl) : "memory");
                            if (v == p.epoch || *s_abort) break;
                            if (tc::global_ns() - tw > p.wait_ns) {
                                *s_abort = 1;
                                atomicOr(p.status, kStatusTimeout);
                                break;
                            }
                            __nanosleep(128);
                        }
                    }
                    bar_group(kBarB);
                    src = p.hseg + (str * p.nseg + (seg_k - 1)) * 64 * NS;
                }
#pragma unroll
                for (int jj = 0; jj < HR; jj++) hs[jj] = src ? __ldcg(src + (int64_t)(pcol + jj) * NS + nrow) : 0.f;
            } else {
                // h_c = k_{c-1} h_{c-1} + S_{c-1}
                tc::mbar_wait(&s_done[i ^ 1], par((q - 1) >> 1), s_abort, p.status, kStatusTimeout, p.wait_ns);
                tc::tc_fence_after();
                uint32_t r[HR];
                load_S(i ^ 1, r);
                const float cm = carry_prev == kChunkReset ? 0.0f : carry_prev;
                const uint64_t cmp = p2(cm, cm);
#pragma unroll
                for (int jj = 0; jj < HR; jj += 2)
                    p2split(fma2(cmp, p2(hs[jj], hs[jj + 1]), p2(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1]))),
                            hs[jj], hs[jj + 1]);
            }
#pragma unroll
            for (int qq = 0; qq < HR / 8; qq++) {
                const uint4 v = make_uint4(pack_bf16(hs[8 * qq], hs[8 * qq + 1]),
                                           pack_bf16(hs[8 * qq + 2], hs[8 * qq + 3]),
                                           pack_bf16(hs[8 * qq + 4], hs[8 * qq + 5]),
                                           pack_bf16(hs[8 * qq + 6], hs[8 * qq + 7]));
                *(uint4*)(sm + LY::kHt + tc::sw128_offset(nrow, pcol + 8 * qq)) = v;
            }
            carry_prev = carry;
            tc::fence_async_smem();
            tc::tc_fence_before();                 // S(q-1) has been read
            if (issuer) tc::bulk_wait_read1();     // the out tile [i] of step q-2 has left
            bar_group(kBarB);
            if (issuer) {
                tc::tc_fence_after();
                // S[i^1] may be overwritten by S(q+1) now
                if (q >= 1) tc::mbar_arrive(&s_free[i ^ 1]);
                // NORM: group A has normalised this step's C tile
                if (NORM) tc::mbar_wait(&norm_done[st], par(q / NST), s_abort, p.status, kStatusTimeout, p.wait_ns);
                // Yoff = C h^T (K = n; h^T is MN-major: rows n, 64 p per row)
                const uint32_t a_c = tc::smem_u32(stg + 2 * kTile + LY::kBC);
#pragma unroll
                for (int kk = 0; kk < NS / 16; kk++) {
                    const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                    tc::mma_bf16(tmem + kColYO, tc::sdesc_sw128(a_c + off, 16, 1024),
                                 tc::sdesc_sw128(a_ht + kk * 2048, 8192, 1024), id_yo, kk > 0);
                }
                tc::mma_commit(yo_done);
            }

            // ---- epilogue: out = (Ydiag + f Yoff + D u) SiLU(z)
            tc::mbar_wait(&y_done[i], par(q >> 1), s_abort, p.status, kStatusTimeout, p.wait_ns);
            tc::mbar_wait(yo_done, par(q), s_abort, p.status, kStatusTimeout, p.wait_ns);
            tc::tc_fence_after();
            uint8_t* outt = sm + LY::kOut + i * kTile;
            {
                const int t = r16;
                const float f = cs->f[t];
                const uint64_t fp = p2(f, f), Dp = p2(Dh, Dh);
                const uint8_t* zt = stg + kTile;
                const uint8_t* xb = sm + LY::kXb + i * kTile;
                uint32_t ry[16], ro[16];
                tc::tmem_ld16_x2_32(tmem + lane_base + kColY + i * 64 + half * 16, ry);
                tc::tmem_ld16_x2_32(tmem + lane_base + kColYO + half * 16, ro);
                tc::tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const int col = c16 + hh * 8;
                    const uint4 xv = *(const uint4*)(xb + tc::sw128_offset(t, col));
                    const uint4 zv = *(const uint4*)(zt + tc::sw128_offset(t, col));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                    const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int jj = hh * 8 + e * 2;
                        uint64_t y = fma2(fp, p2(__uint_as_float(ro[jj]), __uint_as_float(ro[jj + 1])),
                                          p2(__uint_as_float(ry[jj]), __uint_as_float(ry[jj + 1])));
                        y = fma2(Dp, bf2(xw[e]), y);
                        ow[e] = pack_bf16_2(mul2(y, silu2(bf2(zw[e]))));
                    }
                    if (RAG && t >= (int)cs->nvalid) ow[0] = ow[1] = ow[2] = ow[3] = 0u;   // padding
                    *(uint4*)(outt + tc::sw128_offset(t, col)) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
            }
            // ---- leaving the segment: h_out = k_c h_c + S_c -> the next segment or the caller
            if (last) {
                tc::mbar_wait(&s_done[i], par(q >> 1), s_abort, p.status, kStatusTimeout, p.wait_ns);
                tc::tc_fence_after();
                uint32_t r[HR];
                load_S(i, r);
                const bool drop = carry == kChunkReset;
                float* dst = stream_end ? (p.final_ssm ? p.final_ssm + str * 64 * NS : nullptr)
                                        : p.hseg + (str * p.nseg + seg_k) * 64 * NS;
                if (dst != nullptr) {
#pragma unroll
                    for (int jj = 0; jj < HR; jj++)
                        dst[(int64_t)(pcol + jj) * NS + nrow] =
                            (drop ? 0.0f : carry * hs[jj]) + __uint_as_float(r[jj]);
                }
                if (!stream_end) {
                    bar_group(kBarB);
                    if (issuer && !(str == p.withhold && seg_k == 0)) {
                        __threadfence();
                        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.flags + str * p.nseg + seg_k),
                                     "r"(p.epoch) : "memory");
                    }
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();                 // Y[i], Yoff (and S[i]) have been read
            it.next();
            const int aborted = bar_group_or(kBarB, *s_abort);
            if (issuer) {
                tc::tc_fence_after();
                tc::mbar_arrive(&epi_done[i]);
                tc::tma_store_3d(&tm_out, outt, h * 64, t0, b);
                tc::bulk_commit();
                tc::mbar_arrive(&empty[st]);
            }
            if (aborted) break;
        }
        if (issuer) {
            tc::mma_commit(drain_b);
            tc::mbar_drain(drain_b, 0, p.status, kStatusTimeout, p.wait_ns);
            tc::bulk_wait0();
        }
    }

    // ---- teardown: every MMA has completed (drains above) before the tensor memory is freed
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
// (batch, seqlen, width) tensor whose rows lie ld elements apart (ld = width
// when contiguous; a column block of a packed in_proj row otherwise).
static bool encode_tile_map(CUtensorMap* m, const void* base, int width, int64_t ld, int seqlen,
                            int batch)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)seqlen, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * seqlen};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static_assert(Layout<64>::kAlloc <= 227 * 1024 && Layout<128>::kAlloc <= 227 * 1024,
              "the fused kernel's shared memory exceeds the per-CTA limit");

bool fused_path_available() { return tensor_map_encoder() != nullptr; }

size_t fused_flag_count(int max_streams, int sm_count)
{
    return (size_t)kItemsPerSm * sm_count + max_streams;
}
size_t fused_handoff_floats(int max_streams, int dstate, int sm_count)
{
    return fused_flag_count(max_streams, sm_count) * 64 * dstate;
}

// Segments per stream: the count that minimises the makespan in chunk steps
// within the hand-off buffers' capacity.  Items run in rounds of `grid`, but
// the segments of one stream follow each other, so the makespan is at least
// (segments) x (chunks per segment) as well; each step of a segment adds a
// small hand-off cost.
static void choose_segments(int streams, int nchunks, int grid, size_t cap_items, int& nseg, int& cps)
{
    double best = 1e300;
    nseg = 1;
    cps = nchunks;
    for (int sg = 1; sg <= nchunks && sg <= 64; sg++) {
        const int c = (nchunks + sg - 1) / sg;
        const int se = (nchunks + c - 1) / c;
        const size_t items = (size_t)streams * se;
        if (items > cap_items && se > 1) break;
        const double rounds = (double)((items + grid - 1) / grid);
        const double cost = (rounds > se ? rounds : (double)se) * (c + 0.5);
        if (cost < best - 1e-9) {
            best = cost;
            nseg = se;
            cps = c;
        }
    }
}

template <int NS, bool CONV, bool NORM, bool RAG>
static cudaError_t launch_t(const Shape& s, FusedParams fp, const CUtensorMap* maps, int sm_count,
                            size_t max_items, cudaStream_t st)
{
    auto kern = ssd_chunk_fused<NS, CONV, NORM, RAG>;
    const int smem = Layout<NS>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int streams = s.batch * s.nheads, nc = s.nchunks();
    int grid = sm_count * per_sm;                 // every CTA resident: hand-off waits end
    const size_t cap = max_items ? max_items : fused_flag_count(streams, sm_count);
    if (cap < (size_t)streams) return cudaErrorInvalidValue;
    choose_segments(streams, nc, grid, cap, fp.nseg, fp.cps);
    fp.nitems = streams * fp.nseg;
    if (grid > fp.nitems) grid = fp.nitems;
    // A launch captured into a CUDA graph keeps this call's epoch for every
    // replay, so the flags the previous replay published would already read
    // "ready".  Captured, the flag words are cleared in the graph itself, just
    // ahead of the kernel (zero is never an epoch).
    cudaStreamCaptureStatus cap_status = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cap_status);
    if (e != cudaSuccess) return e;
    if (cap_status != cudaStreamCaptureStatusNone) {
        e = cudaMemsetAsync(fp.flags, 0, (size_t)fp.nitems * sizeof(unsigned), st);
        if (e != cudaSuccess) return e;
    }
    // A cooperative launch makes co-residency of the whole grid a condition of
    // the launch: on a GPU shared with other work (another stream's kernels, a
    // reduced SM partition) it is refused with an error instead of starting CTAs
    // whose hand-off waits could only time out.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], fp);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_chunk_fused(const Shape& s, const FwdArgs& a, const void* ubc, const float* dt,
                               const float* acs, const float* rinv, int* status, const FusedWork& fw,
                               cudaStream_t st)
{
    if (!s.act_bf16 || s.headdim != 64 || (s.dstate != 64 && s.dstate != 128) || (s.bc_norm && !rinv))
        return cudaErrorNotSupported;
    const int HP = s.nheads * 64, GN = s.ngroups * s.dstate;
    CUtensorMap maps[5];
    bool ok = encode_tile_map(&maps[0], a.x, HP, a.ld_x, s.seqlen, s.batch) &&
              encode_tile_map(&maps[1], a.z, HP, a.ld_z, s.seqlen, s.batch) &&
              encode_tile_map(&maps[4], a.out, HP, HP, s.seqlen, s.batch);
    if (s.dconv == 4) {
        ok = ok && encode_tile_map(&maps[2], ubc, 2 * GN, 2 * GN, s.seqlen, s.batch);
        maps[3] = maps[2];
    } else {
        ok = ok && encode_tile_map(&maps[2], a.B, GN, a.ld_bc, s.seqlen, s.batch) &&
             encode_tile_map(&maps[3], a.C, GN, a.ld_bc, s.seqlen, s.batch);
    }
    if (!ok) return cudaErrorInvalidValue;
    FusedParams fp;
    fp.batch = s.batch;
    fp.seqlen = s.seqlen;
    fp.nheads = s.nheads;
    fp.ngroups = s.ngroups;
    fp.epoch = fw.epoch;
    fp.dt = dt;
    fp.acs = acs;
    fp.seq = a.seq_idx;
    fp.lengths = a.lengths;
    fp.D = a.D;
    fp.x = (const bf16*)a.x;
    fp.ld_x = a.ld_x;
    fp.conv_w = (const bf16*)a.conv_w;
    fp.conv_b = (const bf16*)a.conv_b;
    fp.init_conv = (const bf16*)a.init_conv;
    fp.init_ssm = a.init_ssm;
    fp.final_ssm = a.final_ssm;
    fp.hseg = fw.hseg;
    fp.flags = fw.flags;
    fp.status = status;
    fp.wait_ns = fw.wait_ns ? fw.wait_ns : tc::kWaitLimitNs;
    fp.withhold = fw.withhold;
    fp.rinv = rinv;
    fp.bn_w = a.bn_w;
    fp.cn_w = a.cn_w;
    fp.bn_bias = a.bn_bias;
    fp.cn_bias = a.cn_bias;
    const bool conv = s.dconv == 4, norm = s.bc_norm != 0, rag = a.lengths != nullptr;
#define SSD_FUSED_LAUNCH(NS_, CONV_, NORM_)                                                     \
    (rag ? launch_t<NS_, CONV_, NORM_, true>(s, fp, maps, fw.sm_count, fw.max_items, st)        \
         : launch_t<NS_, CONV_, NORM_, false>(s, fp, maps, fw.sm_count, fw.max_items, st))
    if (s.dstate == 64)
        return conv ? (norm ? SSD_FUSED_LAUNCH(64, true, true) : SSD_FUSED_LAUNCH(64, true, false))
                    : (norm ? SSD_FUSED_LAUNCH(64, false, true) : SSD_FUSED_LAUNCH(64, false, false));
    return conv ? (norm ? SSD_FUSED_LAUNCH(128, true, true) : SSD_FUSED_LAUNCH(128, true, false))
                : (norm ? SSD_FUSED_LAUNCH(128, false, true) : SSD_FUSED_LAUNCH(128, false, false));
#undef SSD_FUSED_LAUNCH
}

}  // namespace ssd
