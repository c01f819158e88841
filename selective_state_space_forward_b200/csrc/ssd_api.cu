// ssd_api.cu -- host layer of libssd.so: the C ABI declared in include/ssd.h.
//
// Every entry point validates its arguments on the host before enqueuing any
// work, names the bad argument in a thread-local message (the refuse-by-name
// convention of the mojolearn Mamba3Block docs: wrong inputs "are refused by
// name rather than converted"), and launches its kernels on the caller's
// stream.  Workspace is allocated once, at ssd_create, for the handle's
// maximum batch and sequence length.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "ssd.h"
#include "ssd_kernels.h"

using namespace ssd;

namespace {

thread_local std::string g_err;

ssd_status fail(ssd_status st, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

ssd_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

struct ssd_handle {
    ssd_desc d;
    int path;             // SSD_PATH_FUSED or SSD_PATH_STAGED
    int device;
    char* ws;             // one cudaMalloc'd block
    size_t ws_bytes;
    float* u;             // staged: conv output (B, L, conv_dim) fp32
    float* dt;            // (B, H, L)
    float* acs;           // (B, H, L)
    float* cdecay;        // staged: (B, H, nc)
    float* states;        // staged: (B, nc, H, P, N)
    void* ubc;            // fused: conv'd B|C (B, L, 2GN) bf16
    float* rinv;          // fused with bc_norm: 1/rms of every B and C row (B, L, 2G)
    int* status;          // device status word
    const float *bn_w, *cn_w, *bn_bias, *cn_bias;
    int gn_on, gn_group;             // gated RMSNorm after the scan (ssd_set_gated_norm)
    const float* gn_w;
    float gn_eps;
    cudaEvent_t ev_start, ev_stop;   // measurement hook (caller-owned), or null
    uint64_t launches;               // kernels launched since ssd_create
    FusedWork fw;                    // fused path: segment hand-off buffers, epoch, SM count
    // fused path: K2 runs on an auxiliary stream beside K1, forked from and joined
    // back into the caller's stream with events
    cudaStream_t aux;
    cudaEvent_t ev_fork, ev_join;
};

namespace {

int conv_dim(const ssd_desc& d) { return d.nheads * d.headdim + 2 * d.ngroups * d.dstate; }
size_t act_size(const ssd_desc& d) { return d.act_dtype == SSD_DTYPE_BF16 ? 2 : 4; }

Shape make_shape(const ssd_handle* h, int batch, int seqlen)
{
    Shape s;
    s.batch = batch;
    s.seqlen = seqlen;
    s.nheads = h->d.nheads;
    s.headdim = h->d.headdim;
    s.dstate = h->d.dstate;
    s.ngroups = h->d.ngroups;
    s.dconv = h->d.dconv;
    s.act_bf16 = h->d.act_dtype == SSD_DTYPE_BF16;
    s.a_per_token = h->d.a_mode == SSD_A_PER_TOKEN;
    s.bc_norm = h->d.bc_norm;
    return s;
}

size_t conv_offset(const ssd_desc& d, int batch)
{
    return align256((size_t)batch * d.nheads * d.headdim * d.dstate * sizeof(float));
}

bool fused_supported(const ssd_desc& d)
{
    return fused_path_available() && d.act_dtype == SSD_DTYPE_BF16 && d.headdim == 64 &&
           (d.dstate == 64 || d.dstate == 128);
}

ssd_status validate_desc(const ssd_desc* d)
{
    if (!d) return fail(SSD_ERR_INVALID_ARG, "desc is NULL");
    if (d->nheads < 1) return fail(SSD_ERR_INVALID_ARG, "nheads must be >= 1 (got %d)", d->nheads);
    if (d->headdim < 8 || d->headdim > 128 || d->headdim % 8)
        return fail(SSD_ERR_UNSUPPORTED, "headdim must be a multiple of 8 in [8, 128] (got %d)",
                    d->headdim);
    if (d->dstate < 8 || d->dstate > 256 || d->dstate % 8)
        return fail(SSD_ERR_UNSUPPORTED, "dstate must be a multiple of 8 in [8, 256] (got %d)",
                    d->dstate);
    if (d->ngroups < 1 || d->nheads % d->ngroups)
        return fail(SSD_ERR_INVALID_ARG, "ngroups (%d) must divide nheads (%d)", d->ngroups,
                    d->nheads);
    if (d->dconv != 1 && d->dconv != 4)
        return fail(SSD_ERR_UNSUPPORTED, "dconv must be 1 (no conv) or 4 (got %d)", d->dconv);
    if (d->chunk != 0 && d->chunk != 64)
        return fail(SSD_ERR_UNSUPPORTED, "chunk must be 0 or 64 (got %d)", d->chunk);
    if (d->act_dtype != SSD_DTYPE_F32 && d->act_dtype != SSD_DTYPE_BF16)
        return fail(SSD_ERR_INVALID_ARG, "act_dtype %d is not an ssd_dtype", d->act_dtype);
    if (d->a_mode != SSD_A_PER_HEAD && d->a_mode != SSD_A_PER_TOKEN)
        return fail(SSD_ERR_INVALID_ARG, "a_mode %d is not an ssd_a_mode", d->a_mode);
    if (d->bc_norm != 0 && d->bc_norm != 1)
        return fail(SSD_ERR_INVALID_ARG, "bc_norm must be 0 or 1 (got %d)", d->bc_norm);
    if (d->max_batch < 1 || d->max_seqlen < 1)
        return fail(SSD_ERR_INVALID_ARG, "max_batch and max_seqlen must be >= 1");
    if (d->path < SSD_PATH_AUTO || d->path > SSD_PATH_STAGED)
        return fail(SSD_ERR_INVALID_ARG, "path %d is not an ssd_path", d->path);
    if (d->validate_finite != 0 && d->validate_finite != 1)
        return fail(SSD_ERR_INVALID_ARG, "validate_finite must be 0 or 1 (got %d)", d->validate_finite);
    if (d->path == SSD_PATH_FUSED && !fused_supported(*d))
        return fail(SSD_ERR_UNSUPPORTED,
                    "the fused path needs bf16 activations, headdim 64 and dstate 64 or 128");
    return SSD_OK;
}

ssd_status check_ptr(const void* p, const char* name, size_t align, bool required)
{
    if (!p) return required ? fail(SSD_ERR_INVALID_ARG, "%s is NULL", name) : SSD_OK;
    if (!aligned(p, align))
        return fail(SSD_ERR_ALIGNMENT, "%s (%p) is not %zu-byte aligned", name, p, align);
    return SSD_OK;
}

#define SSD_TRY(expr)                     \
    do {                                  \
        ssd_status st_ = (expr);          \
        if (st_ != SSD_OK) return st_;    \
    } while (0)

#define SSD_CUDA(expr, what)                          \
    do {                                              \
        cudaError_t e_ = (expr);                      \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

// A kernel launch: counted, and reported as SSD_ERR_CUDA when it fails.
#define SSD_LAUNCH(h, expr, what)                     \
    do {                                              \
        (h)->launches++;                              \
        SSD_CUDA(expr, what);                         \
    } while (0)

// The main kernel of a call, bracketed by the caller's timing events when set.
#define SSD_MAIN_LAUNCH(h, st, expr, what)                                         \
    do {                                                                           \
        if ((h)->ev_start) SSD_CUDA(cudaEventRecord((h)->ev_start, st), "timing event"); \
        SSD_LAUNCH(h, expr, what);                                                 \
        if ((h)->ev_stop) SSD_CUDA(cudaEventRecord((h)->ev_stop, st), "timing event");   \
    } while (0)

ssd_status check_handle_dims(const ssd_handle* h, int batch, int seqlen)
{
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    if (batch < 0 || seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch (%d) and seqlen (%d) must be >= 0", batch, seqlen);
    if (batch > h->d.max_batch)
        return fail(SSD_ERR_SHAPE_EXCEEDS_MAX, "batch %d exceeds max_batch %d", batch,
                    h->d.max_batch);
    if (seqlen > h->d.max_seqlen)
        return fail(SSD_ERR_SHAPE_EXCEEDS_MAX, "seqlen %d exceeds max_seqlen %d", seqlen,
                    h->d.max_seqlen);
    return SSD_OK;
}

// Pointers shared by forward and step.
ssd_status check_common(const ssd_handle* h, const void* x, const void* z, const float* dt_raw,
                        const float* dt_bias, const float* A, const void* B, const void* C,
                        const float* D, const void* conv_w, const void* conv_b, const void* out)
{
    SSD_TRY(check_ptr(x, "x", 16, true));
    SSD_TRY(check_ptr(z, "z", 16, true));
    SSD_TRY(check_ptr(B, "B", 16, true));
    SSD_TRY(check_ptr(C, "C", 16, true));
    SSD_TRY(check_ptr(out, "out", 16, true));
    SSD_TRY(check_ptr(dt_raw, "dt_raw", 4, true));
    SSD_TRY(check_ptr(dt_bias, "dt_bias", 4, true));
    SSD_TRY(check_ptr(A, "A", 4, true));
    SSD_TRY(check_ptr(D, "D", 4, true));
    if (h->d.dconv == 4) {
        SSD_TRY(check_ptr(conv_w, "conv_w", 16, true));
        SSD_TRY(check_ptr(conv_b, "conv_b", 16, true));
    } else if (conv_w || conv_b) {
        return fail(SSD_ERR_INVALID_ARG, "conv_w/conv_b must be NULL when dconv is 1");
    }
    if (out == x || out == z || out == B || out == C)
        return fail(SSD_ERR_INVALID_ARG, "out may not alias an input");
    return SSD_OK;
}

// ---- scratch of ssd_forward_noalloc --------------------------------------------
// Callers that cannot allocate device memory (a fixed budget owned by someone
// else, or a loop that cannot take cudaFree's device-wide synchronisation)
// cannot create a handle; their forward keeps its workspace in a static device
// array of this module instead.  Layout: the hand-off flags at the head (a
// fixed place, so a flag word only ever holds an epoch), then per call the
// hand-off states, dt, the cumsum and the convolved B|C.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // per device
constexpr size_t kNoAllocMaxItems = 1024;                    // hand-off slots at most
constexpr size_t kNoAllocFlagBytes = kNoAllocMaxItems * sizeof(unsigned);
constexpr int kNoAllocMaxDevices = 64;
static_assert(kNoAllocFlagBytes % 256 == 0, "the hand-off states start 256-byte aligned");

struct NoAllocDevice {
    unsigned char* base = nullptr;   // device address of the scratch array on this device
    int sm_count = 0;
    unsigned epoch = 0;              // the last epoch handed to a call on this device
};
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

}  // namespace

// Zero when the module loads; the flag words are cleared once more at set-up.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// The current device's scratch, with a fresh epoch for this call.  The first
// call on a device (with that device current) looks the array's address up
// and clears its flag words on `st`, ahead of the call's kernels.
ssd_status noalloc_device(cudaStream_t st, NoAllocDevice& out)
{
    int dev = 0;
    SSD_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(SSD_ERR_UNSUPPORTED, "ssd_forward_noalloc serves devices 0 .. %d (current %d)",
                    kNoAllocMaxDevices - 1, dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice& d = g_noalloc_dev[dev];
    if (!d.base) {
        void* p = nullptr;
        SSD_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
        int sms = 0;
        SSD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev),
                 "cudaDeviceGetAttribute(SM count)");
        SSD_CUDA(cudaMemsetAsync(p, 0, kNoAllocFlagBytes, st), "scratch flag clear");
        d.base = (unsigned char*)p;
        d.sm_count = sms < 1 ? 1 : sms;
    }
    if (++d.epoch == 0) d.epoch = 1;   // flags hold earlier calls' epochs, never this one
    out = d;
    return SSD_OK;
}

// Workspace of ssd_backward: byte offsets of its buffers (256-byte aligned).
struct BwdPlan {
    size_t u, dt, acs, cdecay, hin, gs, gu, gbh, gch, pdtb, pA, pD, pconv, pnw, pnb, total;
};

BwdPlan bwd_plan(const ssd_desc& d, int batch, int seqlen)
{
    BwdPlan p;
    memset(&p, 0, sizeof p);
    const size_t B = batch, L = seqlen, H = d.nheads, P = d.headdim, N = d.dstate, G = d.ngroups;
    const size_t nc = (L + 63) / 64, cd = conv_dim(d), nseg = (L + 127) / 128;
    size_t off = 0;
    auto take = [&](size_t floats) { size_t o = off; off = align256(off + floats * sizeof(float)); return o; };
    if (d.dconv == 4) p.u = take(B * L * cd);
    p.dt = take(B * H * L);
    p.acs = take(B * H * L);
    p.cdecay = take(B * H * nc);
    p.hin = take(B * nc * H * P * N);
    p.gs = take(B * nc * H * P * N);
    p.gu = take(B * L * cd);
    p.gbh = take(B * L * H * N);
    p.gch = take(B * L * H * N);
    p.pdtb = take(B * nc * H);
    p.pA = take(B * nc * H);
    p.pD = take(B * nc * H);
    if (d.dconv == 4) p.pconv = take(B * nseg * cd * 5);
    if (d.bc_norm) {
        p.pnw = take(B * nc * G * 2 * N);
        p.pnb = take(B * nc * 2 * H * N);
    }
    p.total = off;
    return p;
}

}  // namespace

// ssd_forward and ssd_forward_ragged (lengths null: every row is seqlen long).
// ld_in > 0: x, z, B, C and dt_raw are column blocks of rows ld_in elements apart,
// dt_raw in the activation dtype (a packed in_proj output).
static ssd_status forward_impl(ssd_handle* h, int32_t batch, int32_t seqlen, const int32_t* lengths,
                               const void* x, const void* z, const void* dt_raw,
                               const float* dt_bias, const float* A, const void* B, const void* C,
                               const float* D, const void* conv_w, const void* conv_b,
                               const int32_t* seq_idx, const void* init_state, void* out,
                               void* final_state, struct CUstream_st* stream, int64_t ld_in = 0)
{
    g_err.clear();
    SSD_TRY(check_handle_dims(h, batch, seqlen));
    SSD_TRY(check_ptr(lengths, "lengths", 4, false));
    cudaStream_t st = (cudaStream_t)stream;
    if (batch == 0) return SSD_OK;
    SSD_TRY(check_ptr(init_state, "init_state", 16, false));
    SSD_TRY(check_ptr(final_state, "final_state", 16, false));
    if (seqlen == 0) {   // no token: the state passes through unchanged
        if (final_state && final_state != init_state) {
            const size_t n = ssd_state_bytes(h, batch);
            SSD_CUDA(init_state ? cudaMemcpyAsync(final_state, init_state, n,
                                                  cudaMemcpyDeviceToDevice, st)
                                : cudaMemsetAsync(final_state, 0, n, st),
                     "empty-sequence state copy");
        }
        return SSD_OK;
    }
    SSD_TRY(check_common(h, x, z, (const float*)dt_raw, dt_bias, A, B, C, D, conv_w, conv_b, out));
    SSD_TRY(check_ptr(seq_idx, "seq_idx", 4, false));
    if (out == init_state || out == final_state)
        return fail(SSD_ERR_INVALID_ARG, "out may not alias a state buffer");

    const Shape s = make_shape(h, batch, seqlen);
    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    if (ld_in > 0) {
        a.ld_x = a.ld_z = a.ld_bc = a.ld_dt = ld_in;
        a.dt_act = 1;
    }
    a.lengths = lengths;
    a.x = x; a.z = z; a.B = B; a.C = C; a.conv_w = conv_w; a.conv_b = conv_b;
    a.dt_raw = (const float*)dt_raw; a.dt_bias = dt_bias; a.A = A; a.D = D; a.seq_idx = seq_idx;
    a.init_ssm = (const float*)init_state;
    a.init_conv = (init_state && s.dconv == 4) ? (const char*)init_state + conv_offset(h->d, batch)
                                               : nullptr;
    a.out = out;
    a.final_ssm = (float*)final_state;
    a.final_conv = (final_state && s.dconv == 4) ? (char*)final_state + conv_offset(h->d, batch)
                                                 : nullptr;
    a.bn_w = h->bn_w; a.cn_w = h->cn_w; a.bn_bias = h->bn_bias; a.cn_bias = h->cn_bias;

    if (h->path == SSD_PATH_STAGED) {
        if (s.dconv == 4) SSD_LAUNCH(h, launch_conv_silu_all(s, a, h->u, st), "conv kernel");
        SSD_LAUNCH(h, launch_dt_cumsum(s, a, h->dt, h->acs, h->cdecay, st), "dt/cumsum kernel");
        SSD_LAUNCH(h, launch_chunk_state(s, a, h->u, h->dt, h->acs, h->states, st),
                   "chunk-state kernel");
        SSD_LAUNCH(h, launch_state_passing(s, a, h->cdecay, h->states, st), "state-passing kernel");
        SSD_MAIN_LAUNCH(h, st, launch_chunk_output(s, a, h->u, h->dt, h->acs, h->states, st),
                        "chunk-output kernel");
    } else {
        // K2 depends on nothing K1 writes: it runs on the auxiliary stream, which
        // starts after everything already on the caller's stream (so the last call's
        // fused kernel has read dt and acs) and which the caller's stream waits for
        // before the fused kernel.  (The final conv history stays after the fused
        // kernel: with the state updated in place it overwrites the history K1 and
        // the fused kernel read.)
        SSD_CUDA(cudaEventRecord(h->ev_fork, st), "cudaEventRecord(fork)");
        SSD_CUDA(cudaStreamWaitEvent(h->aux, h->ev_fork, 0), "cudaStreamWaitEvent(fork)");
        SSD_LAUNCH(h, launch_dt_cumsum(s, a, h->dt, h->acs, nullptr, h->aux), "dt/cumsum kernel");
        SSD_CUDA(cudaEventRecord(h->ev_join, h->aux), "cudaEventRecord(join)");
        if (s.dconv == 4) SSD_LAUNCH(h, launch_conv_silu_bc(s, a, h->ubc, st), "B|C conv kernel");
        if (s.bc_norm) SSD_LAUNCH(h, launch_bc_rms(s, a, h->ubc, h->rinv, st), "B/C rms kernel");
        SSD_CUDA(cudaStreamWaitEvent(st, h->ev_join, 0), "cudaStreamWaitEvent(join)");
        if (++h->fw.epoch == 0) h->fw.epoch = 1;      // flags hold the last call's epoch
        SSD_MAIN_LAUNCH(h, st,
                        launch_chunk_fused(s, a, h->ubc, h->dt, h->acs, h->rinv, h->status, h->fw, st),
                        "fused chunk kernel");
    }
    if (a.final_conv) SSD_LAUNCH(h, launch_conv_state(s, a, st), "conv-state kernel");
    if (h->gn_on)
        SSD_LAUNCH(h, launch_gated_norm(s, out, h->gn_w, h->gn_group, h->gn_eps, lengths, st),
                   "gated norm kernel");
    if (h->d.validate_finite) {
        const size_t ob = (size_t)batch * seqlen * h->d.nheads * h->d.headdim * act_size(h->d);
        SSD_LAUNCH(h, launch_finite_check(out, ob, s.act_bf16, h->status, st), "finite check");
        if (final_state)
            SSD_LAUNCH(h, launch_finite_check(final_state, (size_t)batch * h->d.nheads * h->d.headdim *
                                                               h->d.dstate * sizeof(float),
                                              false, h->status, st),
                       "finite check");
    }
    return SSD_OK;
}

extern "C" {

const char* ssd_last_error(void) { return g_err.c_str(); }

const char* ssd_status_string(ssd_status s)
{
    switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED";
    case SSD_ERR_ALIGNMENT: return "SSD_ERR_ALIGNMENT";
    case SSD_ERR_SHAPE_EXCEEDS_MAX: return "SSD_ERR_SHAPE_EXCEEDS_MAX";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA";
    case SSD_ERR_DEVICE: return "SSD_ERR_DEVICE";
    }
    return "SSD_ERR_UNKNOWN";
}

ssd_status ssd_create(const ssd_desc* d, ssd_handle** out)
{
    g_err.clear();
    if (!out) return fail(SSD_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    SSD_TRY(validate_desc(d));
    int path = d->path;
    if (path == SSD_PATH_AUTO) path = fused_supported(*d) ? SSD_PATH_FUSED : SSD_PATH_STAGED;

    ssd_desc dd = *d;
    dd.chunk = 64;
    dd.path = path;
    Shape s;
    s.batch = dd.max_batch; s.seqlen = dd.max_seqlen; s.nheads = dd.nheads;
    s.headdim = dd.headdim; s.dstate = dd.dstate; s.ngroups = dd.ngroups; s.dconv = dd.dconv;
    s.act_bf16 = dd.act_dtype == SSD_DTYPE_BF16; s.a_per_token = dd.a_mode; s.bc_norm = dd.bc_norm;
    if (path == SSD_PATH_STAGED) {
        const size_t lim = 227 * 1024;
        if (chunk_output_smem_bytes(s) > lim || chunk_state_smem_bytes(s) > lim)
            return fail(SSD_ERR_UNSUPPORTED,
                        "headdim %d x dstate %d needs more shared memory than the staged path has",
                        dd.headdim, dd.dstate);
    }

    const size_t BL = (size_t)dd.max_batch * dd.max_seqlen;
    const size_t nc = (size_t)(dd.max_seqlen + 63) / 64;
    const size_t H = dd.nheads, P = dd.headdim, N = dd.dstate, G = dd.ngroups;
    size_t off = 0, o_u = 0, o_dt, o_acs, o_cd = 0, o_st = 0, o_ubc = 0, o_status;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    if (path == SSD_PATH_STAGED && dd.dconv == 4) o_u = take(BL * conv_dim(dd) * sizeof(float));
    o_dt = take((size_t)dd.max_batch * H * dd.max_seqlen * sizeof(float));
    o_acs = take((size_t)dd.max_batch * H * dd.max_seqlen * sizeof(float));
    if (path == SSD_PATH_STAGED) {
        o_cd = take((size_t)dd.max_batch * H * nc * sizeof(float));
        o_st = take((size_t)dd.max_batch * nc * H * P * N * sizeof(float));
    }
    if (path == SSD_PATH_FUSED && dd.dconv == 4) o_ubc = take(BL * 2 * G * N * 2);
    size_t o_rinv = 0;
    if (path == SSD_PATH_FUSED && dd.bc_norm) o_rinv = take(BL * 2 * G * sizeof(float));
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms < 1) sms = 1;
    size_t o_hseg = 0, o_flags = 0, flag_bytes = 0;
    if (path == SSD_PATH_FUSED) {
        const int streams = dd.max_batch * dd.nheads;
        o_hseg = take(fused_handoff_floats(streams, dd.dstate, sms) * sizeof(float));
        flag_bytes = fused_flag_count(streams, sms) * sizeof(unsigned);
        o_flags = take(flag_bytes);
    }
    o_status = take(256);

    ssd_handle* h = new ssd_handle();
    h->d = dd;
    h->path = path;
    h->device = dev;
    h->fw.sm_count = sms;
    h->fw.epoch = 0;
    h->fw.wait_ns = 0;
    h->fw.withhold = -1;
    cudaError_t e = cudaMalloc(&h->ws, off);
    if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "cudaMalloc(workspace)");
    }
    e = cudaStreamCreateWithFlags(&h->aux, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        cudaFree(h->ws);
        delete h;
        return cuda_fail(e, "cudaStreamCreate / cudaEventCreate");
    }
    h->ws_bytes = off;
    h->u = (path == SSD_PATH_STAGED && dd.dconv == 4) ? (float*)(h->ws + o_u) : nullptr;
    h->dt = (float*)(h->ws + o_dt);
    h->acs = (float*)(h->ws + o_acs);
    h->cdecay = path == SSD_PATH_STAGED ? (float*)(h->ws + o_cd) : nullptr;
    h->states = path == SSD_PATH_STAGED ? (float*)(h->ws + o_st) : nullptr;
    h->ubc = (path == SSD_PATH_FUSED && dd.dconv == 4) ? (void*)(h->ws + o_ubc) : nullptr;
    h->rinv = (path == SSD_PATH_FUSED && dd.bc_norm) ? (float*)(h->ws + o_rinv) : nullptr;
    h->status = (int*)(h->ws + o_status);
    h->fw.hseg = path == SSD_PATH_FUSED ? (float*)(h->ws + o_hseg) : nullptr;
    h->fw.flags = path == SSD_PATH_FUSED ? (unsigned*)(h->ws + o_flags) : nullptr;
    e = cudaMemset(h->status, 0, 256);
    if (e == cudaSuccess && flag_bytes) e = cudaMemset(h->fw.flags, 0, flag_bytes);
    if (e != cudaSuccess) {
        cudaFree(h->ws);
        delete h;
        return cuda_fail(e, "cudaMemset(status)");
    }
    *out = h;
    return SSD_OK;
}

void ssd_destroy(ssd_handle* h)
{
    if (!h) return;
    if (h->aux) {
        cudaStreamSynchronize(h->aux);
        cudaStreamDestroy(h->aux);
    }
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    cudaFree(h->ws);
    delete h;
}

int32_t ssd_get_path(const ssd_handle* h) { return h ? h->path : -1; }

ssd_status ssd_set_bc_norm(ssd_handle* h, const float* B_norm_w, const float* C_norm_w,
                           const float* B_bias, const float* C_bias)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    if (!h->d.bc_norm) return fail(SSD_ERR_INVALID_ARG, "handle was created with bc_norm = 0");
    SSD_TRY(check_ptr(B_norm_w, "B_norm_w", 4, false));
    SSD_TRY(check_ptr(C_norm_w, "C_norm_w", 4, false));
    SSD_TRY(check_ptr(B_bias, "B_bias", 4, false));
    SSD_TRY(check_ptr(C_bias, "C_bias", 4, false));
    h->bn_w = B_norm_w;
    h->cn_w = C_norm_w;
    h->bn_bias = B_bias;
    h->cn_bias = C_bias;
    return SSD_OK;
}

ssd_status ssd_set_gated_norm(ssd_handle* h, int32_t enable, const float* weight,
                              int32_t group_size, float eps)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    if (enable != 0 && enable != 1) return fail(SSD_ERR_INVALID_ARG, "enable must be 0 or 1 (got %d)", enable);
    if (!enable) {
        h->gn_on = 0;
        return SSD_OK;
    }
    const int HP = h->d.nheads * h->d.headdim;
    const int gs = group_size == 0 ? HP : group_size;
    if (!ssd::gated_norm_group_ok(HP, gs))
        return fail(SSD_ERR_INVALID_ARG,
                    "group_size %d must divide H*P = %d, be a multiple of 8 and at most 16384",
                    group_size, HP);
    if (!(eps >= 0.0f) || eps > 1.0f) return fail(SSD_ERR_INVALID_ARG, "eps must lie in [0, 1] (got %g)", (double)eps);
    SSD_TRY(check_ptr(weight, "weight", 16, false));
    h->gn_on = 1;
    h->gn_w = weight;
    h->gn_group = gs;
    h->gn_eps = eps;
    return SSD_OK;
}

size_t ssd_state_conv_offset(const ssd_handle* h, int32_t batch)
{
    if (!h || batch < 0) return 0;
    return conv_offset(h->d, batch);
}

size_t ssd_state_bytes(const ssd_handle* h, int32_t batch)
{
    if (!h || batch < 0) return 0;
    size_t b = conv_offset(h->d, batch);
    if (h->d.dconv == 4) b += (size_t)batch * 3 * conv_dim(h->d) * act_size(h->d);
    return align256(b);
}

ssd_status ssd_forward(ssd_handle* h, int32_t batch, int32_t seqlen, const void* x, const void* z,
                       const float* dt_raw, const float* dt_bias, const float* A, const void* B,
                       const void* C, const float* D, const void* conv_w, const void* conv_b,
                       const int32_t* seq_idx, const void* init_state, void* out,
                       void* final_state, struct CUstream_st* stream)
{
    return forward_impl(h, batch, seqlen, nullptr, x, z, dt_raw, dt_bias, A, B, C, D, conv_w, conv_b,
                        seq_idx, init_state, out, final_state, stream);
}

ssd_status ssd_forward_ragged(ssd_handle* h, int32_t batch, int32_t seqlen, const int32_t* lengths,
                              const void* x, const void* z, const float* dt_raw,
                              const float* dt_bias, const float* A, const void* B, const void* C,
                              const float* D, const void* conv_w, const void* conv_b,
                              const int32_t* seq_idx, const void* init_state, void* out,
                              void* final_state, struct CUstream_st* stream)
{
    if (!lengths) {
        g_err.clear();
        return fail(SSD_ERR_INVALID_ARG, "lengths is NULL");
    }
    return forward_impl(h, batch, seqlen, lengths, x, z, dt_raw, dt_bias, A, B, C, D, conv_w,
                        conv_b, seq_idx, init_state, out, final_state, stream);
}

ssd_status ssd_forward_packed(ssd_handle* h, int32_t batch, int32_t seqlen, const void* zxbcdt,
                              int64_t ld, const float* dt_bias, const float* A, const float* D,
                              const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                              const void* init_state, void* out, void* final_state,
                              struct CUstream_st* stream)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    const int64_t HP = (int64_t)h->d.nheads * h->d.headdim, GN = (int64_t)h->d.ngroups * h->d.dstate;
    const int64_t need = 2 * HP + 2 * GN + h->d.nheads;
    const size_t es = act_size(h->d);
    if (ld < need)
        return fail(SSD_ERR_INVALID_ARG, "ld %lld is below the packed row width 2*H*P + 2*G*N + H = %lld",
                    (long long)ld, (long long)need);
    if ((ld * (int64_t)es) % 16)
        return fail(SSD_ERR_ALIGNMENT, "ld * element size (%lld bytes) must be a multiple of 16",
                    (long long)(ld * (int64_t)es));
    if (batch > 0 && seqlen > 0) SSD_TRY(check_ptr(zxbcdt, "zxbcdt", 16, true));
    const char* base = (const char*)zxbcdt;
    const void* z = base;
    const void* x = base ? base + HP * es : nullptr;
    const void* B = base ? base + 2 * HP * es : nullptr;
    const void* C = base ? base + (2 * HP + GN) * es : nullptr;
    const void* dt = base ? base + (2 * HP + 2 * GN) * es : nullptr;
    return forward_impl(h, batch, seqlen, nullptr, x, z, dt, dt_bias, A, B, C, D, conv_w, conv_b,
                        seq_idx, init_state, out, final_state, stream, ld);
}

ssd_status ssd_step(ssd_handle* h, int32_t batch, const void* x, const void* z,
                    const float* dt_raw, const float* dt_bias, const float* A, const void* B,
                    const void* C, const float* D, const void* conv_w, const void* conv_b,
                    void* state, void* out, struct CUstream_st* stream)
{
    g_err.clear();
    SSD_TRY(check_handle_dims(h, batch, 1));
    if (batch == 0) return SSD_OK;
    SSD_TRY(check_common(h, x, z, dt_raw, dt_bias, A, B, C, D, conv_w, conv_b, out));
    SSD_TRY(check_ptr(state, "state", 16, true));
    if (out == state) return fail(SSD_ERR_INVALID_ARG, "out may not alias the state");
    const Shape s = make_shape(h, batch, 1);
    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    a.x = x; a.z = z; a.B = B; a.C = C; a.conv_w = conv_w; a.conv_b = conv_b;
    a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.D = D; a.out = out;
    a.bn_w = h->bn_w; a.cn_w = h->cn_w; a.bn_bias = h->bn_bias; a.cn_bias = h->cn_bias;
    void* hist = s.dconv == 4 ? (char*)state + conv_offset(h->d, batch) : nullptr;
    SSD_MAIN_LAUNCH(h, (cudaStream_t)stream,
                    launch_decode_step(s, a, (float*)state, hist, h->status, h->fw.wait_ns, h->fw.withhold,
                                       (cudaStream_t)stream),
                    "decode kernel");
    if (h->gn_on)
        SSD_LAUNCH(h, launch_gated_norm(s, out, h->gn_w, h->gn_group, h->gn_eps, nullptr,
                                        (cudaStream_t)stream),
                   "gated norm kernel");
    if (h->d.validate_finite) {
        const size_t ob = (size_t)batch * h->d.nheads * h->d.headdim * act_size(h->d);
        SSD_LAUNCH(h, launch_finite_check(out, ob, s.act_bf16, h->status, (cudaStream_t)stream),
                   "finite check");
        SSD_LAUNCH(h, launch_finite_check(state, (size_t)batch * h->d.nheads * h->d.headdim *
                                                     h->d.dstate * sizeof(float),
                                          false, h->status, (cudaStream_t)stream),
                   "finite check");
    }
    return SSD_OK;
}

ssd_status ssd_stage_conv(ssd_handle* h, int32_t batch, int32_t seqlen, const void* x,
                          const void* B, const void* C, const void* conv_w, const void* conv_b,
                          const int32_t* seq_idx, const void* init_state, float* u,
                          struct CUstream_st* stream)
{
    g_err.clear();
    SSD_TRY(check_handle_dims(h, batch, seqlen));
    if (h->d.dconv != 4) return fail(SSD_ERR_UNSUPPORTED, "the handle has no conv (dconv is 1)");
    if (batch == 0 || seqlen == 0) return SSD_OK;
    SSD_TRY(check_ptr(x, "x", 16, true));
    SSD_TRY(check_ptr(B, "B", 16, true));
    SSD_TRY(check_ptr(C, "C", 16, true));
    SSD_TRY(check_ptr(conv_w, "conv_w", 16, true));
    SSD_TRY(check_ptr(conv_b, "conv_b", 16, true));
    SSD_TRY(check_ptr(u, "u", 16, true));
    SSD_TRY(check_ptr(seq_idx, "seq_idx", 4, false));
    SSD_TRY(check_ptr(init_state, "init_state", 16, false));
    const Shape s = make_shape(h, batch, seqlen);
    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    a.x = x; a.B = B; a.C = C; a.conv_w = conv_w; a.conv_b = conv_b; a.seq_idx = seq_idx;
    a.init_conv = init_state ? (const char*)init_state + conv_offset(h->d, batch) : nullptr;
    SSD_LAUNCH(h, launch_conv_silu_all(s, a, u, (cudaStream_t)stream), "conv kernel");
    return SSD_OK;
}

ssd_status ssd_stage_dt(ssd_handle* h, int32_t batch, int32_t seqlen, const float* dt_raw,
                        const float* dt_bias, const float* A, const int32_t* seq_idx, float* dt,
                        float* acs, struct CUstream_st* stream)
{
    g_err.clear();
    SSD_TRY(check_handle_dims(h, batch, seqlen));
    if (batch == 0 || seqlen == 0) return SSD_OK;
    SSD_TRY(check_ptr(dt_raw, "dt_raw", 4, true));
    SSD_TRY(check_ptr(dt_bias, "dt_bias", 4, true));
    SSD_TRY(check_ptr(A, "A", 4, true));
    SSD_TRY(check_ptr(seq_idx, "seq_idx", 4, false));
    SSD_TRY(check_ptr(dt, "dt", 4, true));
    SSD_TRY(check_ptr(acs, "acs", 4, true));
    const Shape s = make_shape(h, batch, seqlen);
    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.seq_idx = seq_idx;
    SSD_LAUNCH(h, launch_dt_cumsum(s, a, dt, acs, nullptr, (cudaStream_t)stream),
               "dt/cumsum kernel");
    return SSD_OK;
}

ssd_status ssd_set_timing_events(ssd_handle* h, void* start, void* stop)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    if ((start == nullptr) != (stop == nullptr))
        return fail(SSD_ERR_INVALID_ARG, "start and stop must both be set or both be NULL");
    h->ev_start = (cudaEvent_t)start;
    h->ev_stop = (cudaEvent_t)stop;
    return SSD_OK;
}

uint64_t ssd_launch_count(const ssd_handle* h) { return h ? h->launches : 0; }

ssd_status ssd_set_wait_test(ssd_handle* h, uint64_t wait_limit_ns, int32_t withhold_stream)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    if (withhold_stream < -1)
        return fail(SSD_ERR_INVALID_ARG, "withhold_stream must be -1 or a stream index (got %d)",
                    withhold_stream);
    if (wait_limit_ns != 0 && wait_limit_ns < 100000)
        return fail(SSD_ERR_INVALID_ARG, "wait_limit_ns must be 0 (the default) or at least 100000");
    h->fw.wait_ns = wait_limit_ns;
    h->fw.withhold = withhold_stream;
    return SSD_OK;
}

ssd_status ssd_check(ssd_handle* h, struct CUstream_st* stream)
{
    g_err.clear();
    if (!h) return fail(SSD_ERR_INVALID_ARG, "handle is NULL");
    SSD_CUDA(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize");
    int word = 0;
    SSD_CUDA(cudaMemcpy(&word, h->status, sizeof word, cudaMemcpyDeviceToHost), "status read");
    if (word == 0) return SSD_OK;
    SSD_CUDA(cudaMemset(h->status, 0, sizeof word), "status clear");
    return fail(SSD_ERR_DEVICE, "device status 0x%x:%s%s%s", word,
                (word & kStatusTimeout) ? " a bounded wait timed out;" : "",
                (word & kStatusBadLaunch) ? " a kernel rejected its launch shape;" : "",
                (word & kStatusNonFinite) ? " a non-finite value in the results;" : "");
}

ssd_status ssd_s6_forward(int32_t batch, int32_t seqlen, int32_t d_inner, int32_t dstate,
                          int32_t act_dtype, const void* u, const float* delta,
                          const float* delta_bias, const float* A_log, const void* B,
                          const void* C, const float* D, const void* z, const float* init_state,
                          void* out, float* final_state, struct CUstream_st* stream)
{
    g_err.clear();
    if (batch < 0 || seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch (%d) and seqlen (%d) must be >= 0", batch, seqlen);
    if (d_inner < 1) return fail(SSD_ERR_INVALID_ARG, "d_inner must be >= 1 (got %d)", d_inner);
    if (dstate != 8 && dstate != 16 && dstate != 32)
        return fail(SSD_ERR_UNSUPPORTED, "dstate must be 8, 16 or 32 (got %d)", dstate);
    if (act_dtype != SSD_DTYPE_F32 && act_dtype != SSD_DTYPE_BF16)
        return fail(SSD_ERR_INVALID_ARG, "act_dtype %d is not an ssd_dtype", act_dtype);
    const size_t ea = act_dtype == SSD_DTYPE_BF16 ? 2 : 4;
    SSD_TRY(check_ptr(init_state, "init_state", 4, false));
    SSD_TRY(check_ptr(final_state, "final_state", 4, false));
    cudaStream_t st = (cudaStream_t)stream;
    if (batch == 0) return SSD_OK;
    if (seqlen == 0) {   // no token: the state passes through unchanged
        if (final_state && final_state != init_state) {
            const size_t n = (size_t)batch * d_inner * dstate * sizeof(float);
            SSD_CUDA(init_state ? cudaMemcpyAsync(final_state, init_state, n, cudaMemcpyDeviceToDevice, st)
                                : cudaMemsetAsync(final_state, 0, n, st),
                     "empty-sequence state copy");
        }
        return SSD_OK;
    }
    SSD_TRY(check_ptr(u, "u", ea, true));
    SSD_TRY(check_ptr(delta, "delta", 4, true));
    SSD_TRY(check_ptr(delta_bias, "delta_bias", 4, true));
    SSD_TRY(check_ptr(A_log, "A_log", 4, true));
    SSD_TRY(check_ptr(B, "B", ea, true));
    SSD_TRY(check_ptr(C, "C", ea, true));
    SSD_TRY(check_ptr(D, "D", 4, true));
    SSD_TRY(check_ptr(z, "z", ea, false));
    SSD_TRY(check_ptr(out, "out", ea, true));
    if (out == u || out == z || out == B || out == C)
        return fail(SSD_ERR_INVALID_ARG, "out may not alias an input");
    S6Args s;
    s.batch = batch; s.seqlen = seqlen; s.d_inner = d_inner; s.dstate = dstate;
    s.bf16 = act_dtype == SSD_DTYPE_BF16;
    s.u = u; s.B = B; s.C = C; s.z = z;
    s.delta = delta; s.delta_bias = delta_bias; s.A_log = A_log; s.D = D;
    s.init = init_state; s.out = out; s.fin = final_state;
    SSD_CUDA(launch_s6_scan(s, st), "S6 scan kernel");
    return SSD_OK;
}

size_t ssd_backward_workspace_bytes(const ssd_handle* h, int32_t batch, int32_t seqlen)
{
    if (!h || batch < 0 || seqlen < 0) return 0;
    return bwd_plan(h->d, batch, seqlen).total;
}

ssd_status ssd_backward(ssd_handle* h, int32_t batch, int32_t seqlen, const int32_t* lengths,
                        const void* x, const void* z, const float* dt_raw, const float* dt_bias,
                        const float* A, const void* B, const void* C, const float* D,
                        const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                        const void* gout, const ssd_grads* grads, void* workspace,
                        size_t workspace_bytes, struct CUstream_st* stream)
{
    g_err.clear();
    SSD_TRY(check_handle_dims(h, batch, seqlen));
    if (!grads) return fail(SSD_ERR_INVALID_ARG, "grads is NULL");
    SSD_TRY(check_ptr(lengths, "lengths", 4, false));
    const Shape s = make_shape(h, batch, seqlen);
    if (!bwd_supported(s))
        return fail(SSD_ERR_UNSUPPORTED, "the backward serves headdim <= 64 and dstate <= 128 "
                                         "(got headdim %d, dstate %d)", s.headdim, s.dstate);
    if (batch == 0 || seqlen == 0) return SSD_OK;
    SSD_TRY(check_ptr(gout, "gout", 16, true));
    SSD_TRY(check_common(h, x, z, dt_raw, dt_bias, A, B, C, D, conv_w, conv_b, gout));
    SSD_TRY(check_ptr(seq_idx, "seq_idx", 4, false));
    SSD_TRY(check_ptr(grads->x, "grads->x", 16, true));
    SSD_TRY(check_ptr(grads->z, "grads->z", 16, true));
    SSD_TRY(check_ptr(grads->B, "grads->B", 16, true));
    SSD_TRY(check_ptr(grads->C, "grads->C", 16, true));
    SSD_TRY(check_ptr(grads->dt_raw, "grads->dt_raw", 4, true));
    SSD_TRY(check_ptr(grads->dt_bias, "grads->dt_bias", 4, false));
    SSD_TRY(check_ptr(grads->A, "grads->A", 4, false));
    SSD_TRY(check_ptr(grads->D, "grads->D", 4, false));
    SSD_TRY(check_ptr(grads->conv_w, "grads->conv_w", 4, false));
    SSD_TRY(check_ptr(grads->conv_b, "grads->conv_b", 4, false));
    SSD_TRY(check_ptr(grads->B_norm_w, "grads->B_norm_w", 4, false));
    SSD_TRY(check_ptr(grads->C_norm_w, "grads->C_norm_w", 4, false));
    SSD_TRY(check_ptr(grads->B_bias, "grads->B_bias", 4, false));
    SSD_TRY(check_ptr(grads->C_bias, "grads->C_bias", 4, false));
    if (h->d.dconv == 1 && (grads->conv_w || grads->conv_b))
        return fail(SSD_ERR_INVALID_ARG, "grads->conv_w/conv_b must be NULL when dconv is 1");
    if (!h->d.bc_norm && (grads->B_norm_w || grads->C_norm_w || grads->B_bias || grads->C_bias))
        return fail(SSD_ERR_INVALID_ARG, "norm gradients need a handle created with bc_norm = 1");
    SSD_TRY(check_ptr(workspace, "workspace", 256, true));
    const BwdPlan pl = bwd_plan(h->d, batch, seqlen);
    if (workspace_bytes < pl.total)
        return fail(SSD_ERR_INVALID_ARG, "workspace_bytes %zu is below the %zu bytes the call needs "
                    "(ssd_backward_workspace_bytes)", workspace_bytes, pl.total);
    cudaStream_t st = (cudaStream_t)stream;

    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    a.lengths = lengths;
    a.x = x; a.z = z; a.B = B; a.C = C; a.conv_w = conv_w; a.conv_b = conv_b;
    a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.D = D; a.seq_idx = seq_idx;
    a.bn_w = h->bn_w; a.cn_w = h->cn_w; a.bn_bias = h->bn_bias; a.cn_bias = h->cn_bias;
    char* ws = (char*)workspace;
    BwdBufs w;
    memset(&w, 0, sizeof w);
    float* u = s.dconv == 4 ? (float*)(ws + pl.u) : nullptr;
    float* dt = (float*)(ws + pl.dt);
    float* acs = (float*)(ws + pl.acs);
    float* cdecay = (float*)(ws + pl.cdecay);
    float* hin = (float*)(ws + pl.hin);
    w.u = u; w.dt = dt; w.acs = acs; w.cdecay = cdecay; w.hin = hin;
    w.gs = (float*)(ws + pl.gs);
    w.gout = gout;
    w.gu = (float*)(ws + pl.gu);
    w.gbh = (float*)(ws + pl.gbh);
    w.gch = (float*)(ws + pl.gch);
    w.p_dtb = (float*)(ws + pl.pdtb);
    w.p_A = (float*)(ws + pl.pA);
    w.p_D = (float*)(ws + pl.pD);
    w.p_conv = s.dconv == 4 ? (float*)(ws + pl.pconv) : nullptr;
    w.p_nw = s.bc_norm ? (float*)(ws + pl.pnw) : nullptr;
    w.p_nb = s.bc_norm ? (float*)(ws + pl.pnb) : nullptr;
    w.gx = grads->x; w.gz = grads->z; w.gB = grads->B; w.gC = grads->C;
    w.gdt_raw = grads->dt_raw; w.gA = grads->A;
    w.g_dt_bias = grads->dt_bias; w.g_D = grads->D;
    w.gconv_w = grads->conv_w; w.gconv_b = grads->conv_b;
    w.g_bnw = grads->B_norm_w; w.g_cnw = grads->C_norm_w;
    w.g_bnb = grads->B_bias; w.g_cnb = grads->C_bias;
    if (s.dconv == 4 && (!w.gconv_w) != (!w.gconv_b))
        return fail(SSD_ERR_INVALID_ARG, "grads->conv_w and grads->conv_b must both be set or both be NULL");

    // forward recompute on the staged kernels: conv output, dt and the cumsum, the
    // states entering every chunk (zero initial state)
    if (s.dconv == 4) SSD_LAUNCH(h, launch_conv_silu_all(s, a, u, st), "conv kernel");
    SSD_LAUNCH(h, launch_dt_cumsum(s, a, dt, acs, cdecay, st), "dt/cumsum kernel");
    SSD_LAUNCH(h, launch_chunk_state(s, a, u, dt, acs, hin, st), "chunk-state kernel");
    SSD_LAUNCH(h, launch_state_passing(s, a, cdecay, hin, st), "state-passing kernel");
    int nl = 0;
    if (h->ev_start) SSD_CUDA(cudaEventRecord(h->ev_start, st), "timing event");
    const cudaError_t e = launch_backward(s, a, w, &nl, st);
    h->launches += nl;
    if (e != cudaSuccess) return cuda_fail(e, "backward kernels");
    if (h->ev_stop) SSD_CUDA(cudaEventRecord(h->ev_stop, st), "timing event");
    return SSD_OK;
}

ssd_status ssd_forward_noalloc(const ssd_desc* d, int32_t batch, int32_t seqlen, const void* x,
                               const void* z, const float* dt_raw, const float* dt_bias,
                               const float* A, const void* B, const void* C, const float* D,
                               const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                               const void* init_state, void* out, void* final_state,
                               int32_t* status, struct CUstream_st* stream)
{
    g_err.clear();
    SSD_TRY(validate_desc(d));
    if (d->path == SSD_PATH_STAGED || !fused_supported(*d) || d->bc_norm)
        return fail(SSD_ERR_UNSUPPORTED,
                    "ssd_forward_noalloc runs the fused path only: bf16 activations, headdim 64, "
                    "dstate 64 or 128, no B/C norm");
    ssd_handle h{};   // holds the descriptor for the shared checks; owns no memory
    h.d = *d;
    h.d.chunk = 64;
    h.d.path = SSD_PATH_FUSED;
    h.path = SSD_PATH_FUSED;
    SSD_TRY(check_handle_dims(&h, batch, seqlen));
    SSD_TRY(check_ptr(status, "status", 4, true));
    cudaStream_t st = (cudaStream_t)stream;
    if (batch == 0) return SSD_OK;
    SSD_TRY(check_ptr(init_state, "init_state", 16, false));
    SSD_TRY(check_ptr(final_state, "final_state", 16, false));
    if (seqlen == 0) {   // no token: the state passes through unchanged
        if (final_state && final_state != init_state) {
            const size_t n = ssd_state_bytes(&h, batch);
            SSD_CUDA(init_state ? cudaMemcpyAsync(final_state, init_state, n,
                                                  cudaMemcpyDeviceToDevice, st)
                                : cudaMemsetAsync(final_state, 0, n, st),
                     "empty-sequence state copy");
        }
        return SSD_OK;
    }
    SSD_TRY(check_common(&h, x, z, dt_raw, dt_bias, A, B, C, D, conv_w, conv_b, out));
    SSD_TRY(check_ptr(seq_idx, "seq_idx", 4, false));
    if (out == init_state || out == final_state)
        return fail(SSD_ERR_INVALID_ARG, "out may not alias a state buffer");

    // Scratch plan: the token buffers first, then as many hand-off slots as
    // the rest holds (at least one per stream, at most kNoAllocMaxItems).
    const size_t H = h.d.nheads, N = h.d.dstate, G = h.d.ngroups;
    const size_t streams = (size_t)batch * H;
    const size_t slot = 64 * N * sizeof(float);
    const size_t dt_bytes = align256((size_t)batch * H * seqlen * sizeof(float));
    const size_t ubc_bytes = h.d.dconv == 4 ? align256((size_t)batch * seqlen * 2 * G * N * 2) : 0;
    const size_t fixed = kNoAllocFlagBytes + 2 * dt_bytes + ubc_bytes;
    if (streams > kNoAllocMaxItems || fixed + streams * slot > kNoAllocScratchBytes)
        return fail(SSD_ERR_SHAPE_EXCEEDS_MAX,
                    "batch %d x seqlen %d needs %zu bytes of scratch for %zu (row, head) streams; "
                    "ssd_forward_noalloc's static scratch holds %zu bytes and %zu streams",
                    batch, seqlen, fixed + streams * slot, streams, kNoAllocScratchBytes,
                    kNoAllocMaxItems);
    size_t items = (kNoAllocScratchBytes - fixed) / slot;
    if (items > kNoAllocMaxItems) items = kNoAllocMaxItems;

    NoAllocDevice dev;
    SSD_TRY(noalloc_device(st, dev));
    unsigned char* p = dev.base;
    FusedWork fw;
    fw.flags = (unsigned*)p;
    fw.hseg = (float*)(p + kNoAllocFlagBytes);
    fw.epoch = dev.epoch;
    fw.sm_count = dev.sm_count;
    fw.max_items = items;
    fw.wait_ns = 0;
    fw.withhold = -1;
    size_t off = kNoAllocFlagBytes + items * slot;   // slot is a multiple of 256 bytes
    float* dt = (float*)(p + off);
    off += dt_bytes;
    float* acs = (float*)(p + off);
    off += dt_bytes;
    void* ubc = h.d.dconv == 4 ? (void*)(p + off) : nullptr;

    const Shape s = make_shape(&h, batch, seqlen);
    FwdArgs a;
    memset(&a, 0, sizeof a);
    default_strides(a, s);
    a.x = x; a.z = z; a.B = B; a.C = C; a.conv_w = conv_w; a.conv_b = conv_b;
    a.dt_raw = dt_raw; a.dt_bias = dt_bias; a.A = A; a.D = D; a.seq_idx = seq_idx;
    a.init_ssm = (const float*)init_state;
    a.init_conv = (init_state && s.dconv == 4) ? (const char*)init_state + conv_offset(h.d, batch)
                                               : nullptr;
    a.out = out;
    a.final_ssm = (float*)final_state;
    a.final_conv = (final_state && s.dconv == 4) ? (char*)final_state + conv_offset(h.d, batch)
                                                 : nullptr;
    if (s.dconv == 4) SSD_LAUNCH(&h, launch_conv_silu_bc(s, a, ubc, st), "B|C conv kernel");
    SSD_LAUNCH(&h, launch_dt_cumsum(s, a, dt, acs, nullptr, st), "dt/cumsum kernel");
    SSD_LAUNCH(&h, launch_chunk_fused(s, a, ubc, dt, acs, nullptr, status, fw, st), "fused chunk kernel");
    if (a.final_conv) SSD_LAUNCH(&h, launch_conv_state(s, a, st), "conv-state kernel");
    if (h.d.validate_finite) {
        SSD_LAUNCH(&h, launch_finite_check(out, (size_t)batch * seqlen * H * 64 * 2, true, status, st),
                   "finite check");
        if (final_state)
            SSD_LAUNCH(&h, launch_finite_check(final_state, streams * 64 * N * sizeof(float), false,
                                               status, st),
                       "finite check");
    }
    return SSD_OK;
}

}  // extern "C"
