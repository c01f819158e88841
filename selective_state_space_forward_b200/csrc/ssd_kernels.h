// ssd_kernels.h -- host-side launch functions of the libssd kernels (internal).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define SSD_HD __host__ __device__
#else
#define SSD_HD
#endif

namespace ssd {

// Device status word bits (read and cleared by ssd_check).
constexpr int kStatusTimeout = 1;   // a bounded wait gave up
constexpr int kStatusBadLaunch = 2; // a kernel saw a launch shape it cannot serve
constexpr int kStatusNonFinite = 4; // validate_finite: a result holds a NaN or an infinity

// Shapes of one call, resolved by the host layer.
struct Shape {
    int batch, seqlen, nheads, headdim, dstate, ngroups, dconv;
    int act_bf16;     // activations are bf16 (else fp32)
    int a_per_token;  // A is (batch, seqlen, H)
    int bc_norm;      // B/C RMSNorm + per-head bias
    SSD_HD int nchunks() const { return (seqlen + 63) / 64; }
    SSD_HD int conv_dim() const { return nheads * headdim + 2 * ngroups * dstate; }
};

// Pointers of one forward call (device memory).
struct FwdArgs {
    const void *x, *z, *B, *C, *conv_w, *conv_b;
    const float *dt_raw, *dt_bias, *A, *D;
    const int32_t* seq_idx;
    const float* init_ssm;   // (batch, H, P, N) or null
    const void* init_conv;   // (batch, dconv-1, conv_dim) act or null
    void* out;
    float* final_ssm;        // or null
    void* final_conv;        // or null
    const float *bn_w, *cn_w, *bn_bias, *cn_bias;  // B/C norm parameters (nullable)
    const int32_t* lengths;  // (batch) real tokens per row of a ragged batch, or null
    // Row strides in elements of the token-major inputs (a packed in_proj output
    // holds x, z, B, C and dt_raw as column blocks of one row): x, z, B and C,
    // and dt_raw; dt_act: dt_raw has the activation dtype instead of fp32.
    int64_t ld_x, ld_z, ld_bc, ld_dt;
    int dt_act;
};

// Contiguous inputs: every row stride is the tensor's width.
inline void default_strides(FwdArgs& a, const Shape& s)
{
    a.ld_x = a.ld_z = (int64_t)s.nheads * s.headdim;
    a.ld_bc = (int64_t)s.ngroups * s.dstate;
    a.ld_dt = s.nheads;
    a.dt_act = 0;
}

// K1: conv + SiLU of every x|B|C channel into u (batch, seqlen, conv_dim) fp32.
cudaError_t launch_conv_silu_all(const Shape& s, const FwdArgs& a, float* u, cudaStream_t st);
// K1 (fused path): conv + SiLU of the B|C channels only, bf16 (batch, seqlen, 2*G*N).
cudaError_t launch_conv_silu_bc(const Shape& s, const FwdArgs& a, void* ubc, cudaStream_t st);
// Final conv history (batch, dconv-1, conv_dim) from the raw inputs / initial history.
cudaError_t launch_conv_state(const Shape& s, const FwdArgs& a, cudaStream_t st);
// K2: dt = softplus(dt_raw + dt_bias), acs = per-chunk cumsum of dt*a (batch, H, seqlen),
// and the per-chunk carry factor cdecay (batch, H, nchunks): exp(sum of the chunk's dt*a)
// when the chunk holds no document boundary, else 0.  cdecay may be null.
cudaError_t launch_dt_cumsum(const Shape& s, const FwdArgs& a, float* dt, float* acs,
                             float* cdecay, cudaStream_t st);
// K3 (staged): chunk states (batch, nchunks, H, P, N) fp32.
cudaError_t launch_chunk_state(const Shape& s, const FwdArgs& a, const float* u,
                               const float* dt, const float* acs, float* states, cudaStream_t st);
// K4: states -> per-chunk entering states, in place; writes final_ssm.
cudaError_t launch_state_passing(const Shape& s, const FwdArgs& a, const float* cdecay,
                                 float* states, cudaStream_t st);
// K5 (staged): chunk outputs with the D skip and SiLU(z) gate.
cudaError_t launch_chunk_output(const Shape& s, const FwdArgs& a, const float* u,
                                const float* dt, const float* acs, const float* hin,
                                cudaStream_t st);
size_t chunk_output_smem_bytes(const Shape& s);
size_t chunk_state_smem_bytes(const Shape& s);
// KF: the fused chunk sweep (persistent; segments of a stream hand their
// leaving state to the next segment through `hseg`, tagged in `flags` with
// the call's epoch).
struct FusedWork {
    float* hseg;        // fused_handoff_floats(...) floats
    unsigned* flags;    // fused_flag_count(...) words, zero at creation
    unsigned epoch;     // distinct per call (never 0)
    int sm_count;
    size_t max_items;   // hand-off slots in hseg/flags; 0: fused_flag_count(streams, sm_count)
    uint64_t wait_ns;   // limit of the kernel's bounded waits; 0: the default (1 s)
    int withhold;       // testing: stream whose first hand-off is never published; -1: none
};
bool fused_path_available();
size_t fused_handoff_floats(int max_streams, int dstate, int sm_count);
size_t fused_flag_count(int max_streams, int sm_count);
// rinv: with bc_norm, (batch, seqlen, 2G) fp32 from launch_bc_rms, else null.
cudaError_t launch_chunk_fused(const Shape& s, const FwdArgs& a, const void* ubc, const float* dt,
                               const float* acs, const float* rinv, int* status, const FusedWork& fw,
                               cudaStream_t st);
// Fused path with bc_norm: 1/sqrt(mean(row^2) + eps) of every B and C row,
// rinv (batch, seqlen, 2G) fp32: B of group g at g, C at G + g.  Reads the
// convolved B|C (ubc) when dconv = 4, else the raw B and C.
cudaError_t launch_bc_rms(const Shape& s, const FwdArgs& a, const void* ubc, float* rinv,
                          cudaStream_t st);
// validate_finite: OR kStatusNonFinite into *status when the `bytes` bytes at
// data (bf16 or fp32 values; 16-byte aligned, a multiple of 16 bytes) hold a
// NaN or an infinity.
cudaError_t launch_finite_check(const void* data, size_t bytes, bool bf16, int* status, cudaStream_t st);
// Mamba-1 selective scan (S6): device pointers of one call.
struct S6Args {
    int batch, seqlen, d_inner, dstate, bf16;
    const void *u, *B, *C, *z;          // act dtype; z may be null
    const float *delta, *delta_bias, *A_log, *D;
    const float* init;                  // (batch, d_inner, dstate) or null
    void* out;
    float* fin;                         // or null
};
cudaError_t launch_s6_scan(const S6Args& s, cudaStream_t st);
// Backward of a zero-state prefill (chunk_bwd.cu).  Forward quantities recomputed
// by the staged kernels (u, dt, acs, cdecay, hin), the workspace buffers and the
// caller's gradient outputs (fp32; a NULL weight-gradient pointer skips it).
struct BwdBufs {
    const float* u;        // (B, L, conv_dim) conv output, or null when dconv = 1
    const float *dt, *acs; // (B, H, L)
    const float* cdecay;   // (B, H, nc)
    const float* hin;      // (B, nc, H, P, N) states entering each chunk
    float* gs;             // (B, nc, H, P, N) gradient of each chunk state
    const void* gout;      // (B, L, H*P) act dtype
    float* gu;             // (B, L, conv_dim) gradient of the conv output
    float *gbh, *gch;      // (B, L, H, N) per-head gradients of B^, C^
    float *p_dtb, *p_A, *p_D;   // (B, nc, H) partial sums
    float* p_conv;         // (B, nseg, conv_dim, 5) partial sums
    float *p_nw, *p_nb;    // (B, nc, G, 2, N), (B, nc, 2, H, N) partial sums
    // outputs
    float *gx, *gz, *gB, *gC, *gdt_raw, *gA;
    float *g_dt_bias, *g_D, *gconv_w, *gconv_b, *g_bnw, *g_cnw, *g_bnb, *g_cnb;
};
bool bwd_supported(const Shape& s);
size_t bwd_chunk_smem_bytes(const Shape& s);
// Enqueue the backward kernels after the forward recompute; *launches counts them.
cudaError_t launch_backward(const Shape& s, const FwdArgs& a, const BwdBufs& w, int* launches,
                            cudaStream_t st);
// Gated RMSNorm of the scan output, in place: each group of gs consecutive channels
// of every real token is scaled by weight / sqrt(mean(out^2) + eps) (weight null:
// ones).  gs must divide H*P, be a multiple of 8 and at most 16384.
bool gated_norm_group_ok(int d_inner, int gs);
cudaError_t launch_gated_norm(const Shape& s, void* out, const float* weight, int gs, float eps,
                              const int32_t* lengths, cudaStream_t st);
// K6: one decode token per row, state updated in place.  status: the handle's
// device status word (kStatusTimeout when a bounded wait of the kernel gave up);
// wait_ns: the bound of its waits (0: the default); withhold: testing, the
// (row * G + group) block that never requests its first state piece (-1: none).
cudaError_t launch_decode_step(const Shape& s, const FwdArgs& a, float* ssm, void* conv_hist,
                               int* status, uint64_t wait_ns, int withhold, cudaStream_t st);

}  // namespace ssd
